"""The device-trace summary (persistent_sm_decode_02_b200.trace) on hand-built records."""
import numpy as np

from persistent_sm_decode_02_b200 import trace

PLAN = """0 a layer=0 kind=0 tasks=2 K=8 Kpad=8 kcb=32 R=64 S=1 nst=1 segs=1 dep=-1,-1 pdep=-1 nch=0
1 b layer=0 kind=0 tasks=2 K=8 Kpad=8 kcb=32 R=64 S=1 nst=1 segs=1 dep=0,-1 pdep=-1 nch=0
2 a layer=1 kind=0 tasks=1 K=8 Kpad=8 kcb=32 R=64 S=1 nst=1 segs=1 dep=1,-1 pdep=-1 nch=0
ctas=2 smem=1 stages=5 stage_bytes=32768
"""


def rec(cta, op, task, start, ready, data, done, pub):
    key = (cta << 48) | (op << 32) | task
    base = 10_000  # ns; times below in microseconds
    return [key] + [base + int(1000 * x) for x in (start, ready, data, done, pub)]


def test_summary_of_a_three_op_chain():
    records = np.array([
        rec(0, 0, 0, 0.0, 1.0, 1.5, 5.0, 6.0),
        rec(1, 0, 1, 0.0, 1.0, 1.5, 7.0, 8.0),   # op 0 published at 8
        rec(0, 1, 0, 8.5, 9.0, 9.0, 12.0, 13.0),
        rec(1, 1, 1, 9.0, 10.0, 10.0, 12.0, 14.0),  # op 1 published at 14
        rec(0, 2, 0, 15.0, 16.0, 16.0, 19.0, 20.0),  # op 2 published at 20
        [0, 0, 0, 0, 0, 0],  # an unused record slot
    ], dtype=np.uint64)
    rows, totals = trace.summarize(records, PLAN)
    assert [r["name"] for r in rows] == ["a", "b", "a"]
    r0, r1, r2 = rows
    assert r0["critical"] == 8.0 and r0["detect"] == 0.0 and r0["tasks"] == 2
    assert r0["pro"] == 1.0 and r0["cmp"] == 4.5 and r0["tail"] == 1.0 and r0["pub"] == 1.0
    assert r1["critical"] == 6.0 and r1["detect"] == 0.5            # 14 - 8; 8.5 - 8
    assert r1["pro"] == 0.75 and r1["cmp"] == 2.5 and r1["pub"] == 1.5
    assert r2["critical"] == 6.0 and r2["detect"] == 1.0            # 20 - 14; 15 - 14
    assert totals == {"a": [2, 14.0], "b": [1, 6.0]}
    table = trace.format_table(rows, totals)
    assert "| 1 | `b` | 2 | 6.0 | 0.5 | 0.8 | 2.5 | 0.0 | 1.5 |" in table
    assert "| `a` | 2 | 14.0 |" in table


def test_parse_plan_skips_the_footer():
    ops = trace.parse_plan(PLAN)
    assert [o[0] for o in ops] == ["a", "b", "a"] and ops[1][1]["dep"] == "0,-1"
