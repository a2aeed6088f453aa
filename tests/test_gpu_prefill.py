"""Prefill by decode: the cache the GPU builds from the workload's context ids, against the oracle.

The large configs' context is a run of uniform-random token ids; the pages hand
prefill to another engine, so here the decoder itself builds it: from an empty
cache, dec_step_async once per context id (synth.device.prefill_by_decode, which
bench.py uses for the timed workloads).  The oracle decodes the same ids from an
empty cache (its own steps, no GPU value), and the two caches are compared:

  * layer 0: a row of position p depends only on token p (embedding, RMSNorm,
    rounding, one GEMV, RoPE / latent norm, rounding), so nothing spreads across
    positions or layers: max|d| <= 2^-7 max|ref| for bf16 caches (one rounding of an
    8-bit significand at the layer's scale), 1e-5 max|ref| for float32 caches.  (Not
    per element: a flipped rounding of the normalised input moves a small, cancelling
    output by several of its own ulps.);
  * every layer: max|d| <= max(bar, band) * max|ref| of that layer, where bar is the
    model's logits bar (2e-2 FP8, 5e-3 bf16, 1e-4 float32 weights) and band is twice
    the deviation of the oracle's float32-accumulation twin (gemv_acc32) decoding the
    same ids: deeper rows attend to earlier ones, so rounding flips spread as in
    test_gpu_fullsize_e2e.py.

Small workloads: the whole context.  The full-size MoE + MLA model: its first 16
context positions (the oracle takes about 2 s per step there).
"""
import numpy as np
import pytest
import torch

from oracle import model as om
from synth import device as sdev
from synth import workloads

pytestmark = pytest.mark.gpu

SMALL = ["tiny_dense_f32", "small_dense_bf16", "small_dense_fp8", "small_dense_g8_bf16", "small_dense_g8_fp8_hd64",
         "small_mla_moe_fp8"]


def bar(w):
    return {"fp8": 2e-2, "bf16": 5e-3, "f32": 1e-4}[w["weight_dtype"]]


def oracle_cache(w, Wt, ids, gemv=None):
    """Cache of an oracle decoder that decoded `ids` from an empty cache (float64, cache_specs layout)."""
    orig = om.gemv
    if gemv is not None:
        om.gemv = gemv
    try:
        od = om.OracleDecoder(w, Wt)
        for t in ids:
            od.step(int(t))
        return od.export_cache()
    finally:
        om.gemv = orig


def gpu_cache(w, a, b, n):
    """Device cache tensors (install layout, cache dtype bits) -> float64 arrays shaped like the oracle's."""
    def f64(t):
        t = t.cpu()
        if t.dtype == torch.int16:
            t = t.view(torch.bfloat16)
        return t.to(torch.float64).numpy()
    L = w["n_layers"]
    if w["arch"] == "dense":
        shp = (L, w["n_kv_heads"], n, w["head_dim"])
        return dict(k=f64(a).reshape(shp), v=f64(b).reshape(shp))
    return dict(latent=f64(a).reshape(L, n, w["kv_lora"]), pe=f64(b).reshape(L, n, w["qk_rope"]))


def check(w, got, ref, twin):
    rel0 = 2.0 ** -7 if workloads.act_dtype(w) != "f32" else 1e-5
    lines, failures = [], []
    for part in ref:
        for l in range(w["n_layers"]):
            g, r, t = got[part][l], ref[part][l], twin[part][l]
            scale = np.max(np.abs(r))
            dev = np.max(np.abs(g - r)) / scale
            band = 2.0 * np.max(np.abs(t - r)) / scale
            lim = max(bar(w), band)
            lines.append(f"{part} L{l}: max|d|/max|ref| = {dev:.2e} (twin band {band:.2e}, bound {lim:.2e})")
            if dev > lim:
                failures.append(lines[-1])
            if l == 0 and dev > rel0:
                failures.append(f"{part} L0: {dev:.2e} of max|ref| exceeds one rounding ({rel0:.2e})")
    report = f"{w['name']} prefill-by-decode cache:\n  " + "\n  ".join(lines)
    print("\n" + report)
    assert not failures, "\n".join(failures) + "\n" + report


def run(w, n):
    import persistent_sm_decode_02_b200 as pkg

    d = pkg.Decoder(pkg.config_from_workload(w))
    try:
        sdev.load_weights(d, w)
        a, b = sdev.prefill_by_decode(d, w, n)
        assert d.position() == n
        got = gpu_cache(w, a, b, n)
    finally:
        d.close()
        torch.cuda.empty_cache()
    Wt = om.Weights(w, cache_bytes=16 << 30)
    ids = sdev.context_ids(w, n)
    return got, oracle_cache(w, Wt, ids), oracle_cache(w, Wt, ids, gemv=om.gemv_acc32)


@pytest.mark.parametrize("name", SMALL)
def test_prefill_by_decode_small(name):
    w = workloads.get(name)
    check(w, *run(w, w["ctx"]))


def test_prefill_by_decode_fullsize_prefix():
    w = workloads.get("moe_mla_fp8_1k")
    check(w, *run(w, 16))
