"""Full-size parity: the four large workloads in the configuration bench.py times.

A whole oracle step over 8-32 layers is too slow for every workload and, after
many bf16 layers, amplifies rounding-point flips; so each op of three sampled
layers (first, middle, last) and the LM head is checked against the oracle op
evaluated on the GPU's own inputs (rebuilt from the step's dumps), which holds
at any size: all ops agree to ~1e-7 relative except where a bf16 rounding flips.
The router's chosen experts must be the top-k of the GPU's router logits
(exempt below a 1e-4 margin).  End-to-end parity of the same workloads, teacher
forced over several steps, is in test_gpu_fullsize_e2e.py.
"""
import math

import numpy as np
import pytest
import torch

import synth
from oracle import model as om
from oracle.numerics import argmax_first, bf16_bits_to_f64, margin_topk, rmsnorm, rope, rounder, silu
from synth import device as sdev
from synth import workloads

pytestmark = pytest.mark.gpu

LOCAL_TOL = 2e-3  # relative to max |reference| of the op


def _cmp(label, got, ref, tol=LOCAL_TOL):
    err = np.max(np.abs(got - ref)) / max(np.max(np.abs(ref)), 1e-30)
    assert err <= tol, f"{label}: local error {err:.3e}"
    return err


class Step:
    """One GPU step plus accessors for its dumped op outputs."""

    def __init__(self, pkg, w):
        self.pkg, self.w = pkg, w
        self.d = pkg.Decoder(pkg.config_from_workload(w))
        sdev.load_weights(self.d, w)
        k, v = sdev.synthetic_cache_device(w)
        self.d.set_kv_cache(k.data_ptr(), v.data_ptr(), w["ctx"])
        del k, v
        self.first = int(synth.tokens(w["seed"], synth.TOKENS_FIRST, 1, w["vocab"])[0])
        self.logits = np.empty(w["vocab"], np.float32)
        self.next = self.d.step(self.first, self.logits.ctypes.data)
        self.plan = [(l.split()[1], dict(f.split("=") for f in l.split()[2:] if "=" in f))
                     for l in self.d.plan_text().splitlines()[:-1]]
        self.by_layer = {}
        for i, (name, f) in enumerate(self.plan):
            self.by_layer.setdefault(int(f["layer"]), {})[name] = i
        self.kv = self.d.dump(pkg.dec.DEC_DUMP_KV)
        self.routes = np.frombuffer(self.d.dump(pkg.dec.DEC_DUMP_ROUTES), np.int32) if w["arch"] != "dense" else None

    def raw(self, i):
        return np.frombuffer(self.d.dump(self.pkg.dec.DEC_DUMP_OP + i), np.float32).astype(np.float64)

    def out(self, layer, name):
        i = self.by_layer[layer][name]
        return self.raw(i).reshape(int(self.plan[i][1]["S"]), -1).sum(0)

    def combine(self, layer, name, heads, dim):
        i = self.by_layer[layer][name]
        nch = int(self.plan[i][1]["nch"])
        r = self.raw(i)
        m = r[: heads * nch].reshape(heads, nch)
        l_ = r[heads * nch: 2 * heads * nch].reshape(heads, nch)
        o = r[2 * heads * nch:].reshape(heads, nch, dim)
        M = np.max(np.where(l_ > 0, m, -np.inf), axis=1, keepdims=True)
        wg = np.where(l_ > 0, np.exp(m - M), 0.0)
        return (wg[:, :, None] * o).sum(1) / (wg * l_).sum(1, keepdims=True)

    def close(self):
        self.d.close()


def _ffn_out(st, w, l, moe_l):
    """GPU FFN output of layer l (dense down sum, or routed + shared experts with router weights)."""
    if w["arch"] == "dense" or l < w["n_dense_layers"]:
        return st.out(l, "down")
    d = w["d_model"]
    r = st.out(l, "router")
    idx, wts = om.route_topk(r, w["top_k"])
    dn = st.out(l, "exp_down")
    f = sum(wts[j] * dn[j * d:(j + 1) * d] for j in range(w["top_k"]))
    if w["n_shared"]:
        f = f + dn[w["top_k"] * d:(w["top_k"] + 1) * d]
    return f


@pytest.mark.parametrize("name", ["dense_gqa_bf16_1k", "dense_gqa_fp8_8k", "moe_mla_fp8_1k", "moe_mla_fp8_8k"])
def test_fullsize_sampled_ops(name):
    import persistent_sm_decode_02_b200 as pkg

    w = workloads.get(name)
    st = Step(pkg, w)
    try:
        Wt = om.Weights(w, cache_bytes=8 << 30)
        R = rounder(workloads.act_dtype(w))
        eps, th, L, d = w["norm_eps"], w["rope_theta"], w["n_layers"], w["d_model"]
        p = w["ctx"]
        n = p + 1
        kv = bf16_bits_to_f64(np.frombuffer(st.kv, np.uint16))
        sample = sorted({0, L // 2, L - 1})
        h = Wt.embed_row(st.first)
        moe_l = 0
        for l in range(L):
            a = R(rmsnorm(h, Wt.vector("attn_norm", l), eps))
            check = l in sample
            if w["arch"] == "dense":
                hq, hkv, hd = w["n_heads"], w["n_kv_heads"], w["head_dim"]
                qkv = st.out(l, "qkv")
                og = st.combine(l, "attn", hq, hd)
                if check:
                    ref = np.concatenate([Wt.mv("wq", l, a), Wt.mv("wk", l, a), Wt.mv("wv", l, a)])
                    _cmp(f"L{l} qkv", qkv, ref)
                    K = kv[: kv.size // 2].reshape(L, hkv, n, hd)[l]
                    V = kv[kv.size // 2:].reshape(L, hkv, n, hd)[l]
                    q = R(rope(qkv[: hq * hd].reshape(hq, hd), p, th))
                    o = np.stack([om.attention_split_lse(q[i], K[i * hkv // hq], V[i * hkv // hq], [(0, n)])
                                  for i in range(hq)])
                    _cmp(f"L{l} attn", og, o)
                O = st.out(l, "o_proj")
                if check:
                    _cmp(f"L{l} o_proj", O, Wt.mv("wo", l, R(og.reshape(-1))))
            else:
                H, nope, rd, vh, kvl = w["n_heads"], w["qk_nope"], w["qk_rope"], w["v_head"], w["kv_lora"]
                s1 = st.out(l, "q_a|kv_a")
                qb = st.out(l, "q_b")
                ql = st.out(l, "absorb_q")
                olat = st.combine(l, "mla_attn", H, kvl)
                uv = st.out(l, "uv")
                O = st.out(l, "o_proj")
                if check:
                    _cmp(f"L{l} q_a|kv_a", s1, np.concatenate([Wt.mv("q_a", l, a), Wt.mv("kv_a", l, a)]))
                    cqn = R(rmsnorm(s1[: w["q_lora"]], Wt.vector("q_a_norm", l), eps))
                    _cmp(f"L{l} q_b", qb, Wt.mv("q_b", l, cqn))
                    kvb = om.dense_matrix(Wt.get("kv_b", l)).reshape(H, nope + vh, kvl)
                    q = qb.reshape(H, nope + rd)
                    _cmp(f"L{l} absorb", ql, om.mla_absorb_query(R(q[:, :nope]), kvb[:, :nope]).reshape(-1))
                    nl = L * n * kvl
                    C = kv[:nl].reshape(L, n, kvl)[l]
                    PE = kv[nl:].reshape(L, n, rd)[l]
                    qpe = R(rope(q[:, nope:], p, th))
                    olat_ref = om.mla_latent_attention(R(ql.reshape(H, kvl)), qpe, C, PE, 1.0 / math.sqrt(nope + rd))
                    _cmp(f"L{l} mla_attn", olat, olat_ref)
                    _cmp(f"L{l} uv", uv, om.mla_up_value(R(olat), kvb[:, nope:]).reshape(-1))
                    _cmp(f"L{l} o_proj", O, Wt.mv("wo", l, R(uv)))
            h = h + O
            m = R(rmsnorm(h, Wt.vector("ffn_norm", l), eps))
            if check:
                if w["arch"] == "dense" or l < w["n_dense_layers"]:
                    gu = st.out(l, "gate|up")
                    ff = w["ffn_hidden"]
                    _cmp(f"L{l} gate|up", gu, np.concatenate([Wt.mv("w_gate", l, m), Wt.mv("w_up", l, m)]))
                    _cmp(f"L{l} down", st.out(l, "down"), Wt.mv("w_down", l, R(silu(gu[:ff]) * gu[ff:])))
                else:
                    r = st.out(l, "router")
                    _cmp(f"L{l} router", r, Wt.mv("router", l, m))
                    idx, _ = om.route_topk(r, w["top_k"])
                    got = st.routes.reshape(-1, w["top_k"])[moe_l]
                    if not np.array_equal(got, idx):
                        assert margin_topk(r, w["top_k"]) < 1e-4, f"L{l}: routes {got} vs {idx}"
                    eh, gu, ref = w["expert_hidden"], st.out(l, "exp_gate|up"), []
                    for e in got:
                        ref += [Wt.mv("exp_gate", l, m, int(e)), Wt.mv("exp_up", l, m, int(e))]
                    if w["n_shared"]:
                        ref += [Wt.mv("sh_gate", l, m), Wt.mv("sh_up", l, m)]
                    _cmp(f"L{l} experts gate|up", gu, np.concatenate(ref))
                    dn, ref = st.out(l, "exp_down"), []
                    for j, e in enumerate(list(got) + ([-1] if w["n_shared"] else [])):
                        g_, u_ = gu[2 * j * eh:(2 * j + 1) * eh], gu[(2 * j + 1) * eh:(2 * j + 2) * eh]
                        nm = ("sh_down", -1) if e < 0 else ("exp_down", int(e))
                        ref.append(Wt.mv(nm[0], l, R(silu(g_) * u_), nm[1]))
                    _cmp(f"L{l} experts down", dn, np.concatenate(ref))
            if w["arch"] != "dense" and l >= w["n_dense_layers"]:
                moe_l += 1
            h = h + _ffn_out(st, w, l, moe_l)
        z = Wt.mv("lm_head", -1, R(rmsnorm(h, Wt.vector("final_norm"), eps)))
        _cmp("lm_head", st.logits.astype(np.float64), z)
        if margin_topk(z, 1) >= 1e-4:
            assert st.next == argmax_first(z)
    finally:
        st.close()
        torch.cuda.empty_cache()
