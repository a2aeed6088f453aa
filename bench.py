#!/usr/bin/env python
"""Batch-1 decode benchmark: tokens/s/user (TPOT) and achieved HBM bandwidth on one B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--workload NAME]

Prints one JSON line.  The default workload is the 12-layer MoE + MLA FP8 model
with a 1k context (decode 1k), the shape the roofline target is set on; the
context is decoded on the GPU from its token ids before anything is timed
(--cache synthetic installs the seeded cache draw instead).  Timing: W untimed
warm-up steps, then K decode steps chained on the
device (each step feeds back its own greedy token) between CUDA events on the
decoder's stream; the step reads ~8 GB of weights, far more than the 126 MB L2,
so no flush is needed.  `e2e` repeats the measurement through the synchronous
C-ABI call dec_step with the token passed from the host and the greedy token
read back every step.  `ablation` runs the same tiles as one kernel per op
(plain launches and a CUDA graph), and the K steps as one launch of a whole
generation (dec_generate).  `cpu_baseline` times the CPU oracle.
Under torchrun each rank runs an independent replica of the decoder on its own
GPU (batch-1 decode does not shard here); value = all ranks' tokens / max time.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "tokens/s/user at batch 1 (TPOT us); achieved HBM GB/s vs ~8 TB/s roofline"
DEFAULT_WORKLOAD = "moe_mla_fp8_1k"
SOURCES = ["persistent_sm_decode_02_b200/csrc/engine.cuh", "persistent_sm_decode_02_b200/csrc/dec_api.cu",
           "persistent_sm_decode_02_b200/csrc/dec_types.h", "persistent_sm_decode_02_b200/csrc/ptx.cuh"]


def source_hash() -> str:
    h = hashlib.sha256()
    for s in SOURCES:
        with open(os.path.join(ROOT, s), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def recorded_traffic(bytes_step: float):
    """DRAM bytes per step of the engine kernel, scaled from the committed ncu record of the one-layer
    profiling case (its traffic / algorithmic-bytes ratio times this workload's algorithmic bytes),
    if the record was taken on this kernel source; else None."""
    p = os.path.join(ROOT, "profiles", "engine_kernel_traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    # A record stays valid across the later source states it lists as leaving the kernel, the
    # task plan and the launch as captured (host-only or comment-only changes).
    valid = {d.get("source_hash")} | {x["source_hash"] for x in d.get("same_kernel_sources", [])}
    if source_hash() not in valid:
        return None
    return bytes_step * d["dram_bytes_per_step"] / d["algorithmic_bytes_per_step"]


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.file = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=self.file, stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            time.sleep(0.2)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        self.file.flush()
        self.file.seek(0)
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.file.read().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        os.unlink(self.file.name)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"]}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm)}


# --------------------------------------------------------------------------- CPU oracle
def oracle_steps(w, n_steps: int, budget_s: float):
    """Time the CPU oracle decoding `w` (all layers).  Weight generation on the host is
    excluded from the timed compute (reported separately)."""
    import numpy as np

    import synth
    from oracle import model as om

    om.set_threads(os.cpu_count() or 1)
    weights = om.Weights(w)
    gen_time = [0.0]
    orig = weights._generate

    def timed_gen(spec):
        t0 = time.perf_counter()
        r = orig(spec)
        gen_time[0] += time.perf_counter() - t0
        return r

    weights._generate = timed_gen
    dec = om.OracleDecoder(w, weights)
    dec.set_cache(om.synthetic_cache(w), w["ctx"])
    tok = int(synth.tokens(w["seed"], synth.TOKENS_FIRST, 1, w["vocab"])[0])
    out = dec.step(tok)  # warm-up: generates the dense weights
    tok = out["next"]
    total, steps = 0.0, 0
    t_start = time.perf_counter()
    while steps < n_steps and time.perf_counter() - t_start < budget_s:
        g0 = gen_time[0]
        t0 = time.perf_counter()
        out = dec.step(tok)
        total += (time.perf_counter() - t0) - (gen_time[0] - g0)
        tok = out["next"]
        steps += 1
    return dict(value=steps / total if total > 0 else None, steps=steps, seconds=total, gen_s=gen_time[0],
                cores=om.get_threads())


# --------------------------------------------------------------------------- ranks
L2_BYTES = 126 * 2**20


def l2_note(bytes_step: float) -> str:
    """How the timed steps relate to the 126 MB L2 (no flush between steps in either case)."""
    if bytes_step > 4 * L2_BYTES:
        return "no flush: every step streams ~%.1f GB of weights, far above the 126 MB L2" % (bytes_step / 1e9)
    return ("no flush: a step's %.1f MB fit in the 126 MB L2, so steps run warm (a latency-bound "
            "case, not an HBM measurement)" % (bytes_step / 1e6))


def max_over_ranks(x: float, dist=None, device: str = "cuda") -> float:
    """The largest value of x over all ranks (every rank gets it); x itself without a process group."""
    if dist is None:
        return x
    import torch

    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def tpot_stats(per_step_ms):
    """Median, p99 and max of the per-step times (ms) in microseconds (this rank's steps)."""
    xs = sorted(per_step_ms)
    if not xs:
        return None
    pick = lambda q: xs[min(len(xs) - 1, int(round(q * (len(xs) - 1))))]  # nearest rank
    return {"p50": pick(0.5) * 1e3, "p99": pick(0.99) * 1e3, "max": xs[-1] * 1e3, "steps": len(xs)}


def job_throughput(world: int, steps_per_rank: int, seconds_max: float) -> float:
    """Whole-job tokens/s: every rank decodes steps_per_rank tokens of its own replica; the job
    takes as long as its slowest rank."""
    return world * steps_per_rank / seconds_max


# --------------------------------------------------------------------------- GPU arm
def run_ours(args, rank, world, local_rank):
    import torch

    import persistent_sm_decode_02_b200 as pkg
    import synth
    from synth import device as sdev
    from synth import workloads

    torch.cuda.set_device(local_rank)
    dist = None
    if world > 1:
        import torch.distributed as dist  # noqa: F811
    w = workloads.get(args.workload)
    if args.warmup + args.steps > w["n_decode"] or args.e2e_steps + 3 > w["n_decode"]:
        raise SystemExit("steps + warmup must fit the workload's decode length")
    dec = pkg.Decoder(pkg.config_from_workload(w, device=local_rank))
    sdev.load_weights(dec, w)
    t_pf = time.perf_counter()
    if args.cache == "prefill":  # the context decoded on the GPU from its token ids (untimed setup)
        k, v = sdev.prefill_by_decode(dec, w, device=f"cuda:{local_rank}")
    else:
        k, v = sdev.synthetic_cache_device(w, device=f"cuda:{local_rank}")
    t_pf = time.perf_counter() - t_pf
    first = int(synth.tokens(w["seed"], synth.TOKENS_FIRST, 1, w["vocab"])[0])
    stream = torch.cuda.Stream()
    dec.set_stream(stream.cuda_stream)

    per_step = {}

    def timed_chain(mode):
        dec.set_kv_cache(k.data_ptr(), v.data_ptr(), w["ctx"])
        dec.set_exec_mode(mode)
        dec.step(first)
        for _ in range(max(args.warmup - 1, 0)):
            dec.step_async(-1)
        dec.sync()
        torch.cuda.synchronize()
        if dist is not None:
            dist.barrier()
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps + 1)]
        ev[0].record(stream)
        for i in range(args.steps):
            dec.step_async(-1)
            ev[i + 1].record(stream)  # per-step boundaries for the TPOT distribution
        dec.sync()
        torch.cuda.synchronize()
        per_step[mode] = [ev[i].elapsed_time(ev[i + 1]) for i in range(args.steps)]
        ms = max_over_ranks(ev[0].elapsed_time(ev[-1]), dist)
        if dist is not None:
            dist.barrier()
        return ms

    with ClockSampler(local_rank) as clocks:
        ms_main = timed_chain(pkg.dec.DEC_PERSISTENT)
    clk = clocks.summary()
    ablation = {}
    if args.ablation:
        for name, mode in (("per_op_launches", pkg.dec.DEC_PER_OP), ("per_op_cuda_graph", pkg.dec.DEC_PER_OP_GRAPH)):
            ms = timed_chain(mode)
            ablation[name] = {"ms_per_step": ms / args.steps, "tokens_per_s": args.steps / (ms / 1e3)}
        ablation["persistent"] = {"ms_per_step": ms_main / args.steps, "tokens_per_s": args.steps / (ms_main / 1e3)}
        dec.set_exec_mode(pkg.dec.DEC_PERSISTENT)
        # one launch for the whole generation: dec_generate_async runs args.steps steps in a single
        # persistent kernel (greedy feedback and the token ring on the device)
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
        for timed in (False, True):
            dec.set_kv_cache(k.data_ptr(), v.data_ptr(), w["ctx"])
            if dist is not None:
                dist.barrier()
            if timed:
                ev[0].record(stream)
            dec.generate_async(first, args.steps)
            if timed:
                ev[1].record(stream)
            got = dec.generate_wait(args.steps)
            torch.cuda.synchronize()
            if len(got) != args.steps:
                raise RuntimeError(f"generation ended after {len(got)} of {args.steps} steps")
        ms = max_over_ranks(ev[0].elapsed_time(ev[1]), dist)
        ablation["generation_one_launch"] = {"ms_per_step": ms / args.steps, "tokens_per_s": args.steps / (ms / 1e3),
                                             "launches": 1, "steps": args.steps}

    # e2e: the synchronous public call, token in from the host, greedy token out to the host
    dec.set_kv_cache(k.data_ptr(), v.data_ptr(), w["ctx"])
    tok = dec.step(first)
    for _ in range(2):
        tok = dec.step(tok)
    if dist is not None:
        dist.barrier()
    t0 = time.perf_counter()
    for _ in range(args.e2e_steps):
        tok = dec.step(tok)
    e2e_s = max_over_ranks(time.perf_counter() - t0, dist)

    T_mean = w["ctx"] + args.warmup + args.steps / 2.0
    bytes_step = workloads.active_bytes_per_token(w, T_mean)["total"]
    ms_step = ms_main / args.steps
    peak, peak_kind = measured_peaks()
    achieved = bytes_step / (ms_step * 1e-3) / 1e9
    result = None
    if rank == 0:
        result = {
            "metric": METRIC,
            "value": job_throughput(world, args.steps, ms_main / 1e3),
            "unit": "tokens/s",
            "n_gpus": world,
            "steps": args.steps,
            "warmup": args.warmup,
            "ms_per_step": ms_step,
            "tpot_us": ms_step * 1e3,
            "tpot_us_dist": tpot_stats(per_step[pkg.dec.DEC_PERSISTENT]),
            "higher_is_better": True,
            "scaling": "weak",
            "vs_baseline": None,
            "dtype": "fp8-e4m3 weights (128x128 block scales), bf16 activations, fp32 accumulate"
            if w["weight_dtype"] == "fp8" else w["weight_dtype"],
            "data": "synthetic: seeded random-init weights of the named shape; " + (
                f"context of {w['ctx']} seeded uniform-random token ids decoded on the GPU from an empty cache "
                f"({t_pf:.1f} s, untimed)" if args.cache == "prefill" else "seeded random cache draw"),
            "config": {"workload": args.workload, "context": w["ctx"], "decode_positions": [
                w["ctx"] + args.warmup, w["ctx"] + args.warmup + args.steps], "users": world,
                "parallelism": f"replicas{world}", "exec_mode": "persistent",
                "l2": l2_note(bytes_step)},
            "achieved_hbm_gbs": achieved,
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "peak_kind": peak_kind, "unit": "GB/s",
                         "frac": achieved / peak, "traffic": recorded_traffic(bytes_step),
                         "bytes_per_step": bytes_step, "frac_of_8tbs": achieved / 8000.0,
                         "kernel": "engine_kernel (one persistent launch per step)"},
            "clocks": clk,
            "e2e": {"value": job_throughput(world, args.e2e_steps, e2e_s), "unit": "tokens/s", "h2d_bytes_per_step": 4,
                    "d2h_bytes_per_step": 32, "note": "dec_step: token id in, status + step state (greedy token) out"},
            "gpu_launches": args.steps,
            "ablation": ablation or None,
            "source_hash": source_hash(),
        }
    dec.close()
    return result


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=256)
    ap.add_argument("--warmup", type=int, default=8)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--e2e-steps", type=int, default=64)
    ap.add_argument("--no-ablation", dest="ablation", action="store_false")
    ap.add_argument("--cache", choices=("prefill", "synthetic"), default="prefill",
                    help="context cache: decoded on the GPU from the workload's context ids (default), "
                         "or drawn directly from the seeded generator")
    ap.add_argument("--no-cpu-baseline", dest="cpu_baseline", action="store_false")
    ap.add_argument("--cpu-budget-s", type=float, default=30.0)
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    from synth import workloads

    w = workloads.get(args.workload)

    if args.impl == "reference":
        # The reference arm is the CPU oracle; rank 0 alone runs it.
        if rank != 0:
            return
        r = oracle_steps(w, max(1, args.steps), budget_s=max(30.0, 4 * args.cpu_budget_s))
        line = {
            "impl": "reference", "metric": METRIC, "value": r["value"], "unit": "tokens/s", "n_gpus": 0,
            "steps": r["steps"], "warmup": 1, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f64 (bf16 rounding points of the model definition)",
            "data": "synthetic: seeded weights and seeded cache draw (an oracle step costs the same for any "
                    "cache values, so this times the same work as a decoded context)",
            "config": {"workload": args.workload, "context": w["ctx"]},
            "cpu_baseline": {"value": r["value"], "unit": "tokens/s", "cores": r["cores"], "kind": "oracle",
                             "sample": f"{r['steps']} full oracle decode steps (all layers), host weight "
                                       f"generation excluded ({r['gen_s']:.1f} s)"},
            "e2e": {"value": r["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        }
        print(json.dumps(line))
        return

    if world > 1:
        import datetime

        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    result = run_ours(args, rank, world, local_rank)
    if rank == 0 and args.cpu_baseline:
        r = oracle_steps(w, 8, budget_s=args.cpu_budget_s)
        result["cpu_baseline"] = {"value": r["value"], "unit": "tokens/s", "cores": r["cores"], "kind": "oracle",
                                  "sample": f"{r['steps']} full oracle decode steps of {args.workload} after one "
                                            f"warm-up; host weight generation excluded ({r['gen_s']:.1f} s)"}
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(result))


if __name__ == "__main__":
    main()
