"""GPU decode step vs the CPU oracle, teacher-forced, through the C ABI.

Small workloads (several tiles per op, ragged rows and columns, GQA groups of
1, 2, 3 and 8 with head_dim 64 and 128, MLA + routed MoE) run every decode step of the workload in all
three execution modes; the persistent kernel, the per-op launches and the CUDA
graph must agree bit for bit, and each must match the oracle within the
tolerances of the model definition:
  logits: max|d| <= 2e-2 * max|logit| (FP8 weights), <= 5e-3 * max|logit| (bf16 / fp32);
  greedy token and router top-k: exact unless the oracle's margin is below 1e-4.
"""
import numpy as np
import pytest
import torch

from oracle import model as om
from oracle import numerics as nm
from synth import device as sdev
from synth import workloads

pytestmark = pytest.mark.gpu

# cases beyond the named workloads: name -> (workload, overrides).  The long-context MLA case has
# 40 cache blocks, so the MLA attention runs two tasks per block (half of O's columns each); the
# named small MLA case (2 blocks) runs four, and the full-size 8k workloads one.
# The long-context dense case spreads 10,000 positions over 64 chunks per kv head, so each attention
# task streams several ring stages and the last task of a kv head combines many chunks.
VARIANTS = {"small_mla_moe_fp8_ctx2500": ("small_mla_moe_fp8", dict(ctx=2500, cache_from="synthetic")),
            "small_dense_fp8_ctx10000": ("small_dense_fp8", dict(ctx=10000, cache_from="synthetic"))}
SMALL = ["tiny_dense_f32", "small_dense_bf16", "small_dense_fp8", "small_dense_g8_bf16", "small_dense_g8_fp8_hd64",
         "small_mla_moe_fp8", "small_mla_moe_fp8_ctx2500", "small_dense_fp8_ctx10000"]
MARGIN = 1e-4


def tol(w):
    return 2e-2 if w["weight_dtype"] == "fp8" else 5e-3


@pytest.fixture(scope="module")
def pkg():
    import persistent_sm_decode_02_b200 as p
    assert torch.cuda.is_available()
    return p


_REF = {}


def reference(name):
    """Oracle run of the workload: context, then n_decode teacher-forced steps."""
    if name not in _REF:
        base, over = VARIANTS.get(name, (name, {}))
        w = workloads.get(base, **over)
        dec, first, _ = om.build_context(w)
        cache = dec.export_cache()
        steps, tok = [], first
        for _ in range(w["n_decode"]):
            out = dec.step(tok)
            steps.append(dict(tok=tok, logits=out["logits"], next=out["next"],
                              routes=[(r["idx"], r["logits"]) for r in out["routes"]]))
            tok = out["next"]
        _REF[name] = (w, cache, steps, dec.export_cache())
    return _REF[name]


def make_decoder(pkg, w, cache, mode):
    d = pkg.Decoder(pkg.config_from_workload(w, exec_mode=mode))
    sdev.load_weights(d, w)
    k, v = sdev.host_cache_arrays(w, cache)
    d.set_kv_cache(k.ctypes.data, v.ctypes.data, w["ctx"])
    return d


def run_steps(pkg, d, w, steps):
    logits, toks, routes = [], [], []
    buf = np.empty(w["vocab"], dtype=np.float32)
    for s in steps:
        toks.append(d.step(s["tok"], buf.ctypes.data))
        logits.append(buf.copy())
        if w["arch"] != "dense" and w["n_dense_layers"] < w["n_layers"]:
            r = np.frombuffer(d.dump(pkg.dec.DEC_DUMP_ROUTES), dtype=np.int32)
            routes.append(r.reshape(-1, w["top_k"]).copy())
    return logits, toks, routes


def check_against_oracle(w, steps, logits, toks, routes):
    t = tol(w)
    for i, s in enumerate(steps):
        ref = s["logits"]
        err = np.max(np.abs(logits[i] - ref)) / np.max(np.abs(ref))
        assert err <= t, f"step {i}: logits error {err:.3e} > {t}"
        if toks[i] != s["next"]:
            assert nm.margin_topk(ref, 1) < MARGIN, f"step {i}: greedy token {toks[i]} != {s['next']}"
        for j, (idx, rlog) in enumerate(s["routes"]):
            if not np.array_equal(np.sort(routes[i][j]), np.sort(idx)):
                assert nm.margin_topk(rlog, w["top_k"]) < MARGIN, f"step {i} layer {j}: routes differ"
            else:
                assert np.array_equal(routes[i][j], idx), "route order differs"


@pytest.mark.parametrize("name", SMALL)
def test_persistent_matches_oracle(pkg, name):
    w, cache, steps, _ = reference(name)
    d = make_decoder(pkg, w, cache, pkg.dec.DEC_PERSISTENT)
    try:
        logits, toks, routes = run_steps(pkg, d, w, steps)
        check_against_oracle(w, steps, logits, toks, routes)
        assert d.position() == w["ctx"] + w["n_decode"]
    finally:
        d.close()


@pytest.mark.parametrize("name", SMALL)
def test_modes_are_bit_identical(pkg, name):
    w, cache, steps, _ = reference(name)
    d = make_decoder(pkg, w, cache, pkg.dec.DEC_PERSISTENT)
    try:
        outs = {}
        for mode in (pkg.dec.DEC_PERSISTENT, pkg.dec.DEC_PER_OP, pkg.dec.DEC_PER_OP_GRAPH):
            k, v = sdev.host_cache_arrays(w, cache)
            d.set_kv_cache(k.ctypes.data, v.ctypes.data, w["ctx"])
            d.set_exec_mode(mode)
            outs[mode] = run_steps(pkg, d, w, steps)
        base = outs[pkg.dec.DEC_PERSISTENT]
        for mode, o in outs.items():
            for i in range(len(steps)):
                assert np.array_equal(o[0][i], base[0][i]), f"mode {mode} step {i} logits differ"
            assert o[1] == base[1]
    finally:
        d.close()


@pytest.mark.parametrize("name", SMALL)
def test_cache_append_matches_oracle(pkg, name):
    """The rows the decode steps appended (K/V or latent/pe) match the oracle's cache."""
    w, cache, steps, final_cache = reference(name)
    d = make_decoder(pkg, w, cache, pkg.dec.DEC_PERSISTENT)
    try:
        run_steps(pkg, d, w, steps)
        raw = d.dump(pkg.dec.DEC_DUMP_KV)
    finally:
        d.close()
    n = w["ctx"] + w["n_decode"]
    if workloads.act_dtype(w) == "f32":
        vals = np.frombuffer(raw, dtype=np.float32).astype(np.float64)
    else:
        vals = nm.bf16_bits_to_f64(np.frombuffer(raw, dtype=np.uint16))
    L = w["n_layers"]
    if w["arch"] == "dense":
        shp = (L, w["n_kv_heads"], n, w["head_dim"])
        half = int(np.prod(shp))
        got = dict(k=vals[:half].reshape(shp), v=vals[half:].reshape(shp))
        new = (slice(None), slice(None), slice(w["ctx"], n))
        keys = ("k", "v")
    else:
        nl = L * n * w["kv_lora"]
        got = dict(latent=vals[:nl].reshape(L, n, w["kv_lora"]), pe=vals[nl:].reshape(L, n, w["qk_rope"]))
        new = (slice(None), slice(w["ctx"], n))
        keys = ("latent", "pe")
    for k in keys:
        ref = final_cache[k][new]
        g = got[k][new]
        scale = np.max(np.abs(ref))
        assert np.max(np.abs(g - ref)) <= 2 * tol(w) * scale, k
        # the prefilled part is returned untouched
        old = (slice(None), slice(None), slice(0, w["ctx"])) if w["arch"] == "dense" else (slice(None), slice(0, w["ctx"]))
        assert np.array_equal(got[k][old], final_cache[k][old]), k


def test_feedback_chain_matches_host_tokens(pkg):
    """dec_step_async(-1) feeds the device's own greedy token back: same tokens as host-driven steps."""
    w, cache, steps, _ = reference("small_dense_bf16")
    d = make_decoder(pkg, w, cache, pkg.dec.DEC_PERSISTENT)
    try:
        first = steps[0]["tok"]
        host = [d.step(first)]
        for _ in range(4):
            host.append(d.step(host[-1]))
        k, v = sdev.host_cache_arrays(w, cache)
        d.set_kv_cache(k.ctypes.data, v.ctypes.data, w["ctx"])
        dev = []
        d.step_async(first)
        dev.append(d.sync())
        for _ in range(4):
            d.step_async(-1)
            dev.append(d.sync())
        assert dev == host
    finally:
        d.close()
