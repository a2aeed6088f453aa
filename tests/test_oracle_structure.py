"""Structural pins of the oracle step: special cases whose result has a closed form that does not
go through the oracle's own step code, so that a dropped residual add, a norm gain used in the
wrong place, a wrong attention scale or a router weight left out fails here even though the
incremental step and the full recompute (which share the model's structure) would still agree."""
import math

import numpy as np

from oracle import model as om
from oracle import numerics as nm
from synth import workloads


class _ZeroedWeights(om.Weights):
    """The workload's weights with the named matrices replaced by zeros (codes 0 for FP8)."""

    def __init__(self, w, zero):
        super().__init__(w)
        self.zero = set(zero)

    def get(self, name, layer=-1, expert=-1):
        t = super().get(name, layer, expert)
        if name in self.zero:
            t = dict(t, data=np.zeros_like(t["data"]))
        return t


def _rms(x, g, eps):
    return x / math.sqrt(float(np.dot(x, x)) / x.size + eps) * g


def _sig(x):
    return 1.0 / (1.0 + math.exp(-x))


def _logits_of_embedding(w, Wt, tok):
    e = Wt.embed_row(tok)
    return om.dense_matrix(Wt.get("lm_head")) @ _rms(e, Wt.vector("final_norm"), w["norm_eps"])


def test_zeroed_blocks_pass_the_embedding_through_dense():
    """Every block's output projection zero: the residual stream is the embedding row, and the
    logits are the LM head applied to its final RMSNorm (pre-norm residual decoder)."""
    w = workloads.get("tiny_dense_f32")
    Wt = _ZeroedWeights(w, ("wo", "w_down"))
    dec = om.OracleDecoder(w, Wt, exact=True)
    for tok in (5, 900, 17):
        out = dec.step(tok)
        np.testing.assert_array_equal(out["h"], Wt.embed_row(tok))
        np.testing.assert_allclose(out["logits"], _logits_of_embedding(w, Wt, tok), rtol=1e-12, atol=1e-13)


def test_zeroed_blocks_pass_the_embedding_through_mla_moe():
    w = workloads.get("small_mla_moe_fp8", n_layers=2)
    Wt = _ZeroedWeights(w, ("wo", "w_down", "exp_down", "sh_down"))
    dec = om.OracleDecoder(w, Wt, exact=True)
    for tok in (3, 999):
        out = dec.step(tok)
        np.testing.assert_array_equal(out["h"], Wt.embed_row(tok))
        np.testing.assert_allclose(out["logits"], _logits_of_embedding(w, Wt, tok), rtol=1e-12, atol=1e-13)


def test_one_layer_ffn_only_is_pre_norm_residual():
    """One layer, attention output zero: h = e + W_down(silu(W_gate m) * W_up m) with m the
    RMSNorm of e under the FFN gain (not the attention gain, not un-normalised)."""
    w = workloads.get("tiny_dense_f32", n_layers=1)
    Wt = _ZeroedWeights(w, ("wo",))
    dec = om.OracleDecoder(w, Wt, exact=True)
    tok = 77
    out = dec.step(tok)
    e = Wt.embed_row(tok)
    m = _rms(e, Wt.vector("ffn_norm", 0), w["norm_eps"])
    G, U, D = (om.dense_matrix(Wt.get(n, 0)) for n in ("w_gate", "w_up", "w_down"))
    g = G @ m
    h = e + D @ (g / (1.0 + np.exp(-g)) * (U @ m))
    np.testing.assert_allclose(out["h"], h, rtol=1e-11, atol=1e-12)
    z = om.dense_matrix(Wt.get("lm_head")) @ _rms(h, Wt.vector("final_norm"), w["norm_eps"])
    np.testing.assert_allclose(out["logits"], z, rtol=1e-10, atol=1e-11)


def test_dense_attention_two_positions_is_a_sigmoid_mix():
    """Two cached positions: o = s(d) v0 + (1 - s(d)) v1 with d = q.(k0 - k1) / sqrt(head_dim) and
    s the logistic function; query head i reads kv head i // (n_heads / n_kv_heads).  Also checks
    that position 1's RoPE'd key and its value are appended to the cache."""
    w = workloads.get("small_dense_bf16")
    hq, hkv, hd, th = w["n_heads"], w["n_kv_heads"], w["head_dim"], w["rope_theta"]
    dec = om.OracleDecoder(w, exact=True)
    rng = np.random.default_rng(21)
    k0, v0 = rng.normal(size=(hkv, hd)), rng.normal(size=(hkv, hd))
    dec.K[0, :, 0], dec.V[0, :, 0] = k0, v0
    a = rng.normal(size=w["d_model"])
    o = dec._dense_attention(0, a, 1).reshape(hq, hd)
    Wq, Wk, Wv = (om.dense_matrix(dec.Wt.get(n, 0)) for n in ("wq", "wk", "wv"))
    q = nm.rope((Wq @ a).reshape(hq, hd), 1, th)
    k1 = nm.rope((Wk @ a).reshape(hkv, hd), 1, th)
    v1 = (Wv @ a).reshape(hkv, hd)
    np.testing.assert_allclose(dec.K[0, :, 1], k1, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(dec.V[0, :, 1], v1, rtol=1e-12, atol=1e-12)
    per_group = hq // hkv
    for i in range(hq):
        g = i // per_group
        p0 = _sig(float(q[i] @ (k0[g] - k1[g])) / math.sqrt(hd))
        np.testing.assert_allclose(o[i], p0 * v0[g] + (1 - p0) * v1[g], rtol=1e-10, atol=1e-12)


def test_mla_two_positions_is_a_sigmoid_mix():
    """MLA over two cached positions written per head without absorption: the key of position t
    is [W_UK c_t ; pe_t], its value W_UV c_t, and the score scale 1/sqrt(qk_nope + qk_rope).
    Position 1's latent (RMSNorm of the kv_a output's first kv_lora values under the kv_a gain)
    and its RoPE'd pe part are appended to the cache."""
    w = workloads.get("small_mla_moe_fp8")
    H, nope, rdim, vdim, kvl, th = w["n_heads"], w["qk_nope"], w["qk_rope"], w["v_head"], w["kv_lora"], \
        w["rope_theta"]
    dec = om.OracleDecoder(w, exact=True)
    rng = np.random.default_rng(22)
    c0, pe0 = rng.normal(size=kvl), rng.normal(size=rdim)
    dec.C[0, 0], dec.PE[0, 0] = c0, pe0
    a = rng.normal(size=w["d_model"])
    o = dec._mla_attention(0, a, 1).reshape(H, vdim)
    Wt, eps = dec.Wt, w["norm_eps"]
    cq = om.dense_matrix(Wt.get("q_a", 0)) @ a
    q = (om.dense_matrix(Wt.get("q_b", 0)) @ _rms(cq, Wt.vector("q_a_norm", 0), eps)).reshape(H, nope + rdim)
    ckv = om.dense_matrix(Wt.get("kv_a", 0)) @ a
    c1 = _rms(ckv[:kvl], Wt.vector("kv_a_norm", 0), eps)
    pe1 = nm.rope(ckv[kvl:], 1, th)
    np.testing.assert_allclose(dec.C[0, 1], c1, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(dec.PE[0, 1], pe1, rtol=1e-12, atol=1e-12)
    kvb = om.dense_matrix(Wt.get("kv_b", 0)).reshape(H, nope + vdim, kvl)
    for h in range(H):
        qh = np.concatenate([q[h, :nope], nm.rope(q[h, nope:], 1, th)])
        key0 = np.concatenate([kvb[h, :nope] @ c0, pe0])
        key1 = np.concatenate([kvb[h, :nope] @ c1, pe1])
        p0 = _sig(float(qh @ (key0 - key1)) / math.sqrt(nope + rdim))
        ref = p0 * (kvb[h, nope:] @ c0) + (1 - p0) * (kvb[h, nope:] @ c1)
        np.testing.assert_allclose(o[h], ref, rtol=1e-9, atol=1e-11)


def _expert(Wt, l, e, m, pre):
    G, U, D = (om.dense_matrix(Wt.get(pre + n, l, e)) for n in ("_gate", "_up", "_down"))
    g = G @ m
    return D @ (g / (1.0 + np.exp(-g)) * (U @ m))


def test_moe_two_of_two_experts_weights_are_a_sigmoid_pair():
    """Two experts, both chosen: the weights are s(r0 - r1) and s(r1 - r0) of the router logits r,
    and the shared expert is added with weight 1."""
    w = workloads.get("small_mla_moe_fp8", n_experts=2, top_k=2, n_shared=1)
    dec = om.OracleDecoder(w, exact=True)
    m = np.random.default_rng(23).normal(size=w["d_model"])
    f, route = dec._moe(1, m)
    r = om.dense_matrix(dec.Wt.get("router", 1)) @ m
    w0 = _sig(float(r[0] - r[1]))
    ref = w0 * _expert(dec.Wt, 1, 0, m, "exp") + (1 - w0) * _expert(dec.Wt, 1, 1, m, "exp") + \
        _expert(dec.Wt, 1, -1, m, "sh")
    np.testing.assert_allclose(f, ref, rtol=1e-10, atol=1e-12)


def test_moe_renormalised_weights_are_the_softmax_of_the_chosen_logits():
    """Renormalising the softmax over the top-k equals a softmax over the k chosen logits alone;
    the chosen experts are the k largest logits (softmax is monotone)."""
    w = workloads.get("small_mla_moe_fp8", n_shared=0)
    dec = om.OracleDecoder(w, exact=True)
    m = np.random.default_rng(24).normal(size=w["d_model"])
    f, route = dec._moe(2, m)
    r = om.dense_matrix(dec.Wt.get("router", 2)) @ m
    chosen = np.argsort(-r, kind="stable")[: w["top_k"]]
    assert sorted(route["idx"].tolist()) == sorted(chosen.tolist())
    e = np.exp(r[chosen] - r[chosen].max())
    wts = e / e.sum()
    ref = sum(wts[j] * _expert(dec.Wt, 2, int(x), m, "exp") for j, x in enumerate(chosen))
    np.testing.assert_allclose(f, ref, rtol=1e-10, atol=1e-12)
