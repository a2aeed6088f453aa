"""bench.py on the GPU: one JSON line with the keys and the arithmetic its readers rely on.

Runs the tiny dense workload (seconds) from both contexts: the default prefill-by-decode
and the seeded cache draw.
"""
import json
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def run_bench(*extra):
    cmd = [sys.executable, os.path.join(ROOT, "bench.py"), "--workload", "tiny_dense_f32", "--steps", "8",
           "--warmup", "3", "--e2e-steps", "4", "--no-cpu-baseline", *extra]
    out = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, out.stdout
    return json.loads(lines[0])


@pytest.mark.parametrize("cache", ["prefill", "synthetic"])
def test_bench_line(cache):
    d = run_bench("--cache", cache)
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
              "vs_baseline", "dtype", "data", "config", "roofline", "clocks", "e2e", "gpu_launches", "ablation"):
        assert k in d, k
    assert d["n_gpus"] == 1 and d["steps"] == 8 and d["warmup"] == 3 and d["gpu_launches"] == 8
    assert d["config"]["workload"] == "tiny_dense_f32"
    assert abs(d["value"] - 1e3 / d["ms_per_step"]) < 1e-6 * d["value"]
    r = d["roofline"]
    assert r["bound"] == "hbm" and r["unit"] == "GB/s" and abs(r["frac"] - r["achieved"] / r["peak"]) < 1e-9
    assert abs(r["achieved"] - r["bytes_per_step"] / (d["ms_per_step"] * 1e-3) / 1e9) < 1e-6 * r["achieved"]
    e = d["e2e"]
    assert e["unit"] == "tokens/s" and e["value"] > 0 and e["h2d_bytes_per_step"] == 4
    a = d["ablation"]
    for k in ("per_op_launches", "per_op_cuda_graph", "persistent", "generation_one_launch"):
        assert a[k]["tokens_per_s"] > 0, k
    assert a["generation_one_launch"]["launches"] == 1
    assert ("decoded on the GPU" in d["data"]) == (cache == "prefill")
