"""Per-op timeline of one decode step from the device trace (DEC_FLAG_TRACE).

A decoder created with DEC_FLAG_TRACE records, for every task of the last step,
{cta<<48 | op<<32 | task, start, input ready, first stage available, compute done,
published} (DEC_DUMP_TRACE, %globaltimer ns).  `summarize` turns those records into
the critical path of the step: for each op, the time from the publication of its
last dependency to its own last publication, split into

  detect   first task start - dependency published (the dependency poll)
  pro      median input-ready - start (the prologue building the input vector)
  cmp      median done - first stage (the task's stages and arithmetic)
  tail     last done - median done (imbalance and last-task work)
  pub      median published - done (hand-off to the signaller and counter release)

    python -m persistent_sm_decode_02_b200.trace moe_mla_fp8_1k [first_op last_op]

runs the workload (seeded weights and cache draw) for a few persistent steps on
cuda:0 and prints the table for the last one.
"""
from __future__ import annotations

import sys

import numpy as np


def parse_plan(plan_text: str):
    """[(name, {field: value})] per op, from dec_debug_dump(DEC_DUMP_PLAN)."""
    ops = []
    for line in plan_text.splitlines():
        p = line.split()
        if len(p) < 2 or not p[0].isdigit():
            continue
        ops.append((p[1], dict(x.split("=", 1) for x in p[2:] if "=" in x)))
    return ops


def summarize(records: np.ndarray, plan_text: str):
    """Per-op rows and per-op-name totals of the critical path (microseconds)."""
    tr = np.asarray(records, dtype=np.uint64).reshape(-1, 6)
    tr = tr[tr[:, 1] > 0]
    ops = parse_plan(plan_text)
    key = tr[:, 0]
    op = ((key >> np.uint64(32)) & np.uint64(0xFFFF)).astype(np.int64)
    t0 = float(tr[:, 1].min())
    us = [(tr[:, i].astype(np.float64) - t0) / 1e3 for i in range(1, 6)]
    st, pr, da, dn, pb = us
    pub_at, rows, totals = {}, [], {}
    for i, (name, kv) in enumerate(ops):
        m = op == i
        if not m.any():
            continue
        deps = [int(x) for x in kv.get("dep", "-1,-1").split(",") if int(x) >= 0]
        ready = max([pub_at.get(d, 0.0) for d in deps], default=0.0)
        pub_at[i] = float(pb[m].max())
        row = dict(op=i, name=name, tasks=int(m.sum()), start=float(st[m].min()), published=pub_at[i],
                   critical=pub_at[i] - ready, detect=float(st[m].min()) - ready,
                   pro=float(np.median(pr[m] - st[m])), cmp=float(np.median(dn[m] - da[m])),
                   tail=float(dn[m].max() - np.median(dn[m])), pub=float(np.median(pb[m] - dn[m])))
        rows.append(row)
        t = totals.setdefault(name, [0, 0.0])
        t[0] += 1
        t[1] += row["critical"]
    return rows, totals


def format_table(rows, totals, first=0, last=10 ** 9) -> str:
    out = ["| op | name | tasks | critical | detect | pro | cmp | tail | pub |", "|---|---|---|---|---|---|---|---|---|"]
    for r in rows:
        if first <= r["op"] <= last:
            out.append("| %d | `%s` | %d | %.1f | %.1f | %.1f | %.1f | %.1f | %.1f |" % (
                r["op"], r["name"].replace("|", "\\|"), r["tasks"], r["critical"], r["detect"], r["pro"], r["cmp"],
                r["tail"], r["pub"]))
    out += ["", "| op name | ops | critical path total (us) |", "|---|---|---|"]
    for name, (c, d) in sorted(totals.items(), key=lambda x: -x[1][1]):
        out.append("| `%s` | %d | %.1f |" % (name.replace("|", "\\|"), c, d))
    return "\n".join(out)


def collect(workload: str, steps: int = 6):
    """Decode `steps` persistent steps of a workload with tracing on; (records, plan text, step ms)."""
    import torch

    import synth
    from synth import device as sdev
    from synth import workloads

    from . import dec
    from .dec import Decoder, config_from_workload

    w = workloads.get(workload)
    d = Decoder(config_from_workload(w, flags=dec.DEC_FLAG_TRACE))
    try:
        sdev.load_weights(d, w)
        k, v = sdev.synthetic_cache_device(w)
        d.set_kv_cache(k.data_ptr(), v.data_ptr(), w["ctx"])
        s = torch.cuda.Stream()
        d.set_stream(s.cuda_stream)
        d.step(int(synth.tokens(w["seed"], synth.TOKENS_FIRST, 1, w["vocab"])[0]))
        ms = []
        for _ in range(steps):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(s)
            d.step_async(-1)
            e1.record(s)
            d.sync()
            ms.append(e0.elapsed_time(e1))
        rec = np.frombuffer(d.dump(dec.DEC_DUMP_TRACE), np.uint64).copy()
        return rec, d.plan_text(), ms
    finally:
        d.close()


def main(argv):
    workload = argv[1] if len(argv) > 1 else "moe_mla_fp8_1k"
    first = int(argv[2]) if len(argv) > 2 else 0
    last = int(argv[3]) if len(argv) > 3 else 10 ** 9
    rec, plan, ms = collect(workload)
    rows, totals = summarize(rec, plan)
    print("traced step ms:", " ".join("%.3f" % x for x in ms))
    print("step span us: %.1f" % max(r["published"] for r in rows))
    print(format_table(rows, totals, first, last))


if __name__ == "__main__":
    main(sys.argv)
