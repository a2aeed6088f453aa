"""Model-level pins of the oracle: invariants that any correct decoder must satisfy."""
import numpy as np
import pytest

import synth
from oracle import model as om
from oracle import numerics as nm
from synth import workloads


def _incremental_vs_full(name, n_tok, **over):
    w = workloads.get(name, **over)
    Wt = om.Weights(w)
    toks = synth.tokens(w["seed"], 0x77, n_tok, w["vocab"])
    full = om.forward_full(w, Wt, toks, exact=True)
    dec = om.OracleDecoder(w, Wt, exact=True)
    inc = np.stack([dec.step(int(t))["logits"] for t in toks])
    np.testing.assert_allclose(inc, full, rtol=1e-9, atol=1e-10 * np.max(np.abs(full)))


def test_incremental_equals_full_recompute_dense_f32():
    _incremental_vs_full("tiny_dense_f32", 12)


def test_incremental_equals_full_recompute_dense_gqa():
    _incremental_vs_full("small_dense_bf16", 10)


def test_incremental_equals_full_recompute_mla_moe():
    _incremental_vs_full("small_mla_moe_fp8", 8, n_layers=2)


def test_context_length_one_returns_v_dense():
    w = workloads.get("small_dense_bf16")
    dec = om.OracleDecoder(w, exact=True)
    rng = np.random.default_rng(0)
    a = rng.normal(size=w["d_model"])
    o = dec._dense_attention(0, a, 0).reshape(w["n_heads"], w["head_dim"])
    v = dec.Wt.mv("wv", 0, a).reshape(w["n_kv_heads"], w["head_dim"])
    for i in range(w["n_heads"]):
        np.testing.assert_array_equal(o[i], v[(i * w["n_kv_heads"]) // w["n_heads"]])


def test_context_length_one_returns_v_mla():
    w = workloads.get("small_mla_moe_fp8")
    dec = om.OracleDecoder(w, exact=True)
    a = np.random.default_rng(1).normal(size=w["d_model"])
    o = dec._mla_attention(0, a, 0).reshape(w["n_heads"], w["v_head"])
    kvb = om.dense_matrix(dec.Wt.get("kv_b", 0)).reshape(w["n_heads"], w["qk_nope"] + w["v_head"], w["kv_lora"])
    ref = np.einsum("hvc,c->hv", kvb[:, w["qk_nope"]:], dec.C[0, 0])
    np.testing.assert_allclose(o, ref, rtol=1e-12, atol=1e-14)


def test_one_expert_top1_equals_dense_mlp():
    w = workloads.get("small_mla_moe_fp8", n_experts=1, top_k=1, n_shared=0)
    dec = om.OracleDecoder(w, exact=True)
    m = np.random.default_rng(2).normal(size=w["d_model"])
    f, route = dec._moe(1, m)
    assert list(route["idx"]) == [0] and route["weights"][0] == 1.0
    G = om.dense_matrix(dec.Wt.get("exp_gate", 1, 0))
    U = om.dense_matrix(dec.Wt.get("exp_up", 1, 0))
    D = om.dense_matrix(dec.Wt.get("exp_down", 1, 0))
    ref = D @ (nm.silu(G @ m) * (U @ m))
    np.testing.assert_allclose(f, ref, rtol=1e-11, atol=1e-13)


def test_router_weights_sum_to_one_in_step():
    w = workloads.get("small_mla_moe_fp8")
    dec = om.OracleDecoder(w)
    out = dec.step(3)
    assert len(out["routes"]) == w["n_layers"] - w["n_dense_layers"]
    for r in out["routes"]:
        assert r["weights"].sum() == pytest.approx(1.0, abs=1e-13)
        assert np.array_equal(r["idx"], nm.topk_lowest_index(r["logits"], w["top_k"]))


def test_rounding_points_are_on_grid():
    """With bf16 activations every cached value lies on the bf16 grid."""
    w = workloads.get("small_dense_bf16")
    dec = om.OracleDecoder(w)
    for t in (5, 9, 11):
        dec.step(t)
    k = dec.K[:, :, :3]
    np.testing.assert_array_equal(nm.round_bf16(k), k)


def test_first_token_after_context_is_greedy():
    w = workloads.get("tiny_dense_f32", ctx=8)
    dec, first, ids = om.build_context(w)
    assert dec.T == 8 and len(ids) == 8
    dec2 = om.OracleDecoder(w, dec.Wt)
    for t in ids:
        out = dec2.step(int(t))
    assert first == out["next"] == nm.argmax_first(out["logits"])
