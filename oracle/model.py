"""Oracle decoder: one batch-1 decode step of a dense GQA or an MLA + MoE transformer, float64.

TEST INFRASTRUCTURE ONLY (see the package docstring).

The step follows the model family the pages name (TileRT 是什么, §五 5.2 模型结构
支持: MLA attention, MoE with routed experts and 8 active per token, dense first
layers; §五 5.3 内存管理: the latent kv_cache and the RoPE-key pe_cache) and the
decode-only split of work (SemiAnalysis TileRT InferenceX article, PD
disaggregation section: prefill runs elsewhere and hands its KV cache to the
decode engine).  Formulas are the textbook ones (see numerics.py).  Rounding
points (the activation dtype of the model definition; identity in the
exactness pins):
  * every GEMV input vector, q/k/v after RoPE, the cached latent and RoPE key,
    the absorbed query q_lat, the attention output, the SwiGLU product;
  * GEMV outputs, router logits, logits and the residual stream stay float64.
"""
from __future__ import annotations

import ctypes
import math
import os
from collections import OrderedDict

import numpy as np

import synth
from synth import workloads

from .numerics import (E4M3_TABLE, argmax_first, bf16_bits_to_f64, dequant_fp8_b128, identity, rmsnorm,
                       rope, rounder, silu, softmax, topk_lowest_index)

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB = os.path.join(_HERE, "liboracle.so")
_lib = None


def lib():
    global _lib
    if _lib is None:
        if not os.path.exists(LIB):
            raise RuntimeError(f"{LIB} missing: run __graft_entry__.build()")
        L = ctypes.CDLL(LIB)
        i64, vp = ctypes.c_int64, ctypes.c_void_p
        L.oracle_gemv_f32.argtypes = [vp, i64, i64, vp, vp]
        L.oracle_gemv_bf16.argtypes = [vp, i64, i64, vp, vp]
        L.oracle_gemv_fp8.argtypes = [vp, vp, i64, i64, vp, vp, vp]
        L.oracle_gemv_f32_acc32.argtypes = [vp, i64, i64, vp, vp]
        L.oracle_gemv_bf16_acc32.argtypes = [vp, i64, i64, vp, vp]
        L.oracle_gemv_fp8_acc32.argtypes = [vp, vp, i64, i64, vp, vp, vp]
        L.oracle_set_threads.argtypes = [ctypes.c_int]
        L.oracle_get_threads.restype = ctypes.c_int
        _lib = L
    return _lib


def set_threads(n: int) -> None:
    lib().oracle_set_threads(int(n))


def get_threads() -> int:
    return int(lib().oracle_get_threads())


_TABLE = np.ascontiguousarray(E4M3_TABLE)


def gemv(t: dict, x: np.ndarray) -> np.ndarray:
    """y = W x in float64 for a host weight `t` (dtype f32 / bf16 bits / fp8 codes + scales)."""
    x = np.ascontiguousarray(x, dtype=np.float64)
    N, K = t["data"].shape
    assert x.shape == (K,), (x.shape, K)
    y = np.empty(N, dtype=np.float64)
    d = t["data"]
    if t["dtype"] == "f32":
        lib().oracle_gemv_f32(d.ctypes.data, N, K, x.ctypes.data, y.ctypes.data)
    elif t["dtype"] == "bf16":
        lib().oracle_gemv_bf16(d.ctypes.data, N, K, x.ctypes.data, y.ctypes.data)
    else:
        lib().oracle_gemv_fp8(d.ctypes.data, t["scales"].ctypes.data, N, K, _TABLE.ctypes.data, x.ctypes.data,
                              y.ctypes.data)
    return y


def gemv_acc32(t: dict, x: np.ndarray) -> np.ndarray:
    """Float32-accumulation twin of gemv: NOT the definition.  The same products summed in
    float32 (per 128-column block, then across blocks), as a float32-accumulating
    implementation would.  Tests swap it in for gemv only to measure how far such an
    implementation lands from the float64 definition on a chaotic random-init model."""
    x = np.ascontiguousarray(x, dtype=np.float64)
    N, K = t["data"].shape
    assert x.shape == (K,), (x.shape, K)
    y = np.empty(N, dtype=np.float64)
    d = t["data"]
    if t["dtype"] == "f32":
        lib().oracle_gemv_f32_acc32(d.ctypes.data, N, K, x.ctypes.data, y.ctypes.data)
    elif t["dtype"] == "bf16":
        lib().oracle_gemv_bf16_acc32(d.ctypes.data, N, K, x.ctypes.data, y.ctypes.data)
    else:
        lib().oracle_gemv_fp8_acc32(d.ctypes.data, t["scales"].ctypes.data, N, K, _TABLE.ctypes.data,
                                    x.ctypes.data, y.ctypes.data)
    return y


def dense_matrix(t: dict) -> np.ndarray:
    """Float64 value of a host weight (small tensors only)."""
    if t["dtype"] == "f32":
        return t["data"].astype(np.float64)
    if t["dtype"] == "bf16":
        return bf16_bits_to_f64(t["data"])
    return dequant_fp8_b128(t["data"], t["scales"])


class Weights:
    """Host weights of a workload, drawn on demand from the seeded generator (CPU side).

    Tensors are kept in an LRU store bounded by `cache_bytes`, so full-size
    workloads regenerate what does not fit.
    """

    def __init__(self, w: dict, cache_bytes: int = 24 << 30):
        self.w = w
        self.seed = w["seed"]
        self.specs = {(s["name"], s["layer"], s["expert"]): s for s in workloads.weight_specs(w)}
        self.cache_bytes = cache_bytes
        self._store: OrderedDict = OrderedDict()
        self._bytes = 0

    def spec(self, name, layer=-1, expert=-1):
        return self.specs[(name, layer, expert)]

    def get(self, name, layer=-1, expert=-1) -> dict:
        key = (name, layer, expert)
        if key in self._store:
            self._store.move_to_end(key)
            return self._store[key]
        s = self.specs[key]
        t = self._generate(s)
        nb = t["data"].nbytes + (t["scales"].nbytes if t.get("scales") is not None else 0)
        self._store[key] = t
        self._bytes += nb
        while self._bytes > self.cache_bytes and len(self._store) > 1:
            _, old = self._store.popitem(last=False)
            self._bytes -= old["data"].nbytes + (old["scales"].nbytes if old.get("scales") is not None else 0)
        return t

    def _generate(self, s) -> dict:
        n = int(np.prod(s["shape"]))
        if s["dtype"] == "f32":
            data = synth.normal_f32(self.seed, s["tid"], n, s["std"], s["offset"]).reshape(s["shape"])
            return dict(dtype="f32", data=data, scales=None)
        if s["dtype"] == "bf16":
            data = synth.normal_bf16_bits(self.seed, s["tid"], n, s["std"], s["offset"]).reshape(s["shape"])
            return dict(dtype="bf16", data=data, scales=None)
        q, sc = synth.fp8_b128(self.seed, s["tid"], s["shape"][0], s["shape"][1], s["std"])
        return dict(dtype="fp8", data=q, scales=sc)

    def vector(self, name, layer=-1) -> np.ndarray:
        return self.get(name, layer)["data"].astype(np.float64)

    def embed_row(self, tok: int) -> np.ndarray:
        """Row `tok` of the embedding table (generated alone: its stream offset is tok * d_model)."""
        s = self.specs[("embed", -1, -1)]
        d = s["shape"][1]
        if s["dtype"] == "f32":
            return synth.normal_f32(self.seed, s["tid"], d, s["std"], s["offset"], start=tok * d).astype(np.float64)
        return bf16_bits_to_f64(synth.normal_bf16_bits(self.seed, s["tid"], d, s["std"], s["offset"], start=tok * d))

    def mv(self, name, layer, x, expert=-1) -> np.ndarray:
        return gemv(self.get(name, layer, expert), x)


class OracleDecoder:
    """Batch-1 decoder holding its own copy of the KV cache (values already in the cache dtype)."""

    def __init__(self, w: dict, weights: Weights | None = None, exact: bool = False):
        self.w = w
        self.Wt = weights if weights is not None else Weights(w)
        # exact=True drops every rounding point (used by the exactness pins).
        self.R = identity if exact else rounder(workloads.act_dtype(w))
        self.eps = w["norm_eps"]
        self.theta = w["rope_theta"]
        L, S = w["n_layers"], w["max_seq"]
        if w["arch"] == "dense":
            shp = (L, w["n_kv_heads"], S, w["head_dim"])
            self.K = np.zeros(shp)
            self.V = np.zeros(shp)
        else:
            self.C = np.zeros((L, S, w["kv_lora"]))
            self.PE = np.zeros((L, S, w["qk_rope"]))
        self.T = 0

    # -------------------------------------------------------------- context
    def set_cache(self, parts: dict, n: int) -> None:
        """Take a prefilled cache of n positions (float64 values, one array per part as in cache_specs)."""
        if self.w["arch"] == "dense":
            self.K[:, :, :n] = parts["k"]
            self.V[:, :, :n] = parts["v"]
        else:
            self.C[:, :n] = parts["latent"]
            self.PE[:, :n] = parts["pe"]
        self.T = n

    def export_cache(self, n: int | None = None) -> dict:
        n = self.T if n is None else n
        if self.w["arch"] == "dense":
            return dict(k=self.K[:, :, :n].copy(), v=self.V[:, :, :n].copy())
        return dict(latent=self.C[:, :n].copy(), pe=self.PE[:, :n].copy())

    # ----------------------------------------------------------------- step
    def step(self, tok: int) -> dict:
        """Decode one token at position p = T; appends to the cache and returns the logits and extras."""
        w, R, Wt = self.w, self.R, self.Wt
        p = self.T
        if p >= w["max_seq"]:
            raise ValueError("cache full")
        h = Wt.embed_row(int(tok))
        routes = []
        for l in range(w["n_layers"]):
            a = R(rmsnorm(h, Wt.vector("attn_norm", l), self.eps))
            if w["arch"] == "dense":
                o = self._dense_attention(l, a, p)
            else:
                o = self._mla_attention(l, a, p)
            h = h + Wt.mv("wo", l, o)
            m = R(rmsnorm(h, Wt.vector("ffn_norm", l), self.eps))
            if w["arch"] == "dense" or l < w["n_dense_layers"]:
                h = h + self._swiglu(("w_gate", "w_up", "w_down"), l, -1, m)
            else:
                f, route = self._moe(l, m)
                h = h + f
                routes.append(route)
        z = Wt.mv("lm_head", -1, R(rmsnorm(h, Wt.vector("final_norm"), self.eps)))
        self.T = p + 1
        return dict(logits=z, next=argmax_first(z), routes=routes, h=h)

    def _dense_attention(self, l, a, p):
        """GQA attention of one new token over positions 0..p (Vaswani et al. 2017; Ainslie et al. 2023)."""
        w, R, Wt = self.w, self.R, self.Wt
        hq, hkv, hd = w["n_heads"], w["n_kv_heads"], w["head_dim"]
        q = R(rope(Wt.mv("wq", l, a).reshape(hq, hd), p, self.theta))
        k = R(rope(Wt.mv("wk", l, a).reshape(hkv, hd), p, self.theta))
        v = R(Wt.mv("wv", l, a).reshape(hkv, hd))
        self.K[l, :, p] = k
        self.V[l, :, p] = v
        o = np.empty((hq, hd))
        for i in range(hq):
            g = (i * hkv) // hq
            s = self.K[l, g, : p + 1] @ q[i] / math.sqrt(hd)
            o[i] = softmax(s) @ self.V[l, g, : p + 1]
        return R(o.reshape(-1))

    def _mla_attention(self, l, a, p):
        """MLA in the absorbed form: the query is mapped into the latent space, scores and the
        weighted sum run over the cached latent, then W_UV maps back per head."""
        w, R, Wt = self.w, self.R, self.Wt
        H, nope, rdim, vdim, kvl = w["n_heads"], w["qk_nope"], w["qk_rope"], w["v_head"], w["kv_lora"]
        cq = Wt.mv("q_a", l, a)
        ckv = Wt.mv("kv_a", l, a)
        cqn = R(rmsnorm(cq, Wt.vector("q_a_norm", l), self.eps))
        q = Wt.mv("q_b", l, cqn).reshape(H, nope + rdim)
        self.C[l, p] = R(rmsnorm(ckv[:kvl], Wt.vector("kv_a_norm", l), self.eps))
        self.PE[l, p] = R(rope(ckv[kvl:], p, self.theta))
        qn = R(q[:, :nope])
        qpe = R(rope(q[:, nope:], p, self.theta))
        kvb = dense_matrix(Wt.get("kv_b", l)).reshape(H, nope + vdim, kvl)
        o = mla_absorbed(qn, qpe, self.C[l, : p + 1], self.PE[l, : p + 1], kvb[:, :nope], kvb[:, nope:], R)
        return R(o.reshape(-1))

    def _swiglu(self, names, l, e, m):
        """SwiGLU FFN (Shazeer 2020): W_down (silu(W_gate m) * (W_up m))."""
        g = self.Wt.mv(names[0], l, m, e)
        u = self.Wt.mv(names[1], l, m, e)
        return self.Wt.mv(names[2], l, self.R(silu(g) * u), e)

    def _moe(self, l, m):
        """Softmax router, top-k with ties to the lower expert id, weights renormalised over the
        chosen k; weighted routed experts plus the shared expert(s) with weight 1."""
        w = self.w
        r = self.Wt.mv("router", l, m)
        idx, wts = route_topk(r, w["top_k"])
        f = np.zeros(w["d_model"])
        for j, e in enumerate(idx):
            f = f + wts[j] * self._swiglu(("exp_gate", "exp_up", "exp_down"), l, int(e), m)
        if w["n_shared"] > 0:
            f = f + self._swiglu(("sh_gate", "sh_up", "sh_down"), l, -1, m)
        return f, dict(layer=l, logits=r, idx=idx, weights=wts)


def route_topk(router_logits: np.ndarray, k: int):
    """pi = softmax(r); S = top-k of pi (ties to the lower index); w_i = pi_i / sum_S pi."""
    pi = softmax(router_logits)
    idx = topk_lowest_index(pi, k)
    wts = pi[idx] / np.sum(pi[idx])
    return idx, wts


def mla_absorb_query(qn, W_UK):
    """q_lat^h = W_UK^h^T q_nope^h: the query mapped into the latent space (qn [H, nope], W_UK [H, nope, kv_lora])."""
    return np.einsum("hjc,hj->hc", W_UK, qn)


def mla_latent_attention(q_lat, qpe, C, PE, scale):
    """s_h(t) = (q_lat^h . c_t + q_pe^h . kpe_t) * scale; O_lat^h = sum_t softmax(s_h)_t c_t."""
    s = (q_lat @ C.T + qpe @ PE.T) * scale
    return softmax(s, axis=1) @ C


def mla_up_value(O_lat, W_UV):
    """o^h = W_UV^h O_lat^h (O_lat [H, kv_lora], W_UV [H, v, kv_lora])."""
    return np.einsum("hvc,hc->hv", W_UV, O_lat)


def mla_absorbed(qn, qpe, C, PE, W_UK, W_UV, R=identity):
    """Absorbed MLA for one token: q_lat^h = W_UK^h^T q_nope^h; s_h(t) = (q_lat^h . c_t + q_pe^h . kpe_t)
    / sqrt(d_nope + d_rope); O_lat^h = sum_t softmax(s_h)_t c_t; o^h = W_UV^h O_lat^h.

    qn [H, nope], qpe [H, rope], C [T, kv_lora], PE [T, rope], W_UK [H, nope, kv_lora], W_UV [H, v, kv_lora].
    """
    scale = 1.0 / math.sqrt(qn.shape[1] + qpe.shape[1])
    q_lat = R(mla_absorb_query(qn, W_UK))
    O_lat = mla_latent_attention(q_lat, qpe, C, PE, scale)
    return mla_up_value(R(O_lat), W_UV)


def mla_unabsorbed(qn, qpe, C, PE, W_UK, W_UV):
    """MLA written without absorption: per head, k_t = [W_UK c_t ; kpe_t], v_t = W_UV c_t,
    o = sum_t softmax(q . k_t / sqrt(d_nope + d_rope)) v_t."""
    H = qn.shape[0]
    scale = 1.0 / math.sqrt(qn.shape[1] + qpe.shape[1])
    out = np.empty((H, W_UV.shape[1]))
    for h in range(H):
        k_nope = C @ W_UK[h].T  # [T, nope]
        v = C @ W_UV[h].T  # [T, v]
        s = (k_nope @ qn[h] + PE @ qpe[h]) * scale
        out[h] = softmax(s) @ v
    return out


def attention_split_lse(q, K, V, bounds):
    """Split-KV attention for one query: each chunk [t0, t1) yields (m, l, o) = (max score,
    sum e^(s-m), sum e^(s-m) v); the combine rescales every chunk to the global max M:
    out = sum_c e^(m_c-M) o_c / sum_c e^(m_c-M) l_c."""
    scale = 1.0 / math.sqrt(q.shape[0])
    parts = []
    for t0, t1 in bounds:
        s = K[t0:t1] @ q * scale
        m = np.max(s)
        e = np.exp(s - m)
        parts.append((m, np.sum(e), e @ V[t0:t1]))
    M = max(pm for pm, _, _ in parts)
    num = sum(math.exp(pm - M) * po for pm, _, po in parts)
    den = sum(math.exp(pm - M) * pl for pm, pl, _ in parts)
    return num / den


# ------------------------------------------------------------------ full recompute


def forward_full(w: dict, Wt: Weights, tokens, exact: bool = True) -> np.ndarray:
    """Causal forward pass over a whole token sequence without a cache (no incremental state):
    every layer processes all positions at once with a causal mask.  Returns logits [T, vocab].
    Used to pin the incremental step (the two must agree)."""
    R = identity if exact else rounder(workloads.act_dtype(w))
    eps, theta = w["norm_eps"], w["rope_theta"]
    T = len(tokens)
    pos = np.arange(T)
    h = np.stack([Wt.embed_row(int(t)) for t in tokens])
    mask = np.tril(np.ones((T, T), dtype=bool))

    def mm(name, l, X, e=-1):
        return X @ dense_matrix(Wt.get(name, l, e)).T

    for l in range(w["n_layers"]):
        a = R(rmsnorm(h, Wt.vector("attn_norm", l), eps))
        if w["arch"] == "dense":
            hq, hkv, hd = w["n_heads"], w["n_kv_heads"], w["head_dim"]
            q = R(rope(mm("wq", l, a).reshape(T, hq, hd), pos[:, None], theta))
            k = R(rope(mm("wk", l, a).reshape(T, hkv, hd), pos[:, None], theta))
            v = R(mm("wv", l, a).reshape(T, hkv, hd))
            o = np.empty((T, hq, hd))
            for i in range(hq):
                g = (i * hkv) // hq
                s = q[:, i] @ k[:, g].T / math.sqrt(hd)
                s = np.where(mask, s, -np.inf)
                o[:, i] = softmax(s, axis=1) @ v[:, g]
        else:
            H, nope, rdim, vdim, kvl = w["n_heads"], w["qk_nope"], w["qk_rope"], w["v_head"], w["kv_lora"]
            cq = mm("q_a", l, a)
            ckv = mm("kv_a", l, a)
            q = mm("q_b", l, R(rmsnorm(cq, Wt.vector("q_a_norm", l), eps))).reshape(T, H, nope + rdim)
            c = R(rmsnorm(ckv[:, :kvl], Wt.vector("kv_a_norm", l), eps))
            kpe = R(rope(ckv[:, kvl:], pos, theta))
            qn = R(q[:, :, :nope])
            qpe = R(rope(q[:, :, nope:], pos[:, None], theta))
            kvb = dense_matrix(Wt.get("kv_b", l)).reshape(H, nope + vdim, kvl)
            o = np.empty((T, H, vdim))
            for h_ in range(H):
                k_nope = c @ kvb[h_, :nope].T
                vv = c @ kvb[h_, nope:].T
                s = (qn[:, h_] @ k_nope.T + qpe[:, h_] @ kpe.T) / math.sqrt(nope + rdim)
                s = np.where(mask, s, -np.inf)
                o[:, h_] = softmax(s, axis=1) @ vv
        h = h + mm("wo", l, R(o.reshape(T, -1)))
        m = R(rmsnorm(h, Wt.vector("ffn_norm", l), eps))
        if w["arch"] == "dense" or l < w["n_dense_layers"]:
            h = h + mm("w_down", l, R(silu(mm("w_gate", l, m)) * mm("w_up", l, m)))
        else:
            f = np.zeros_like(h)
            for t in range(T):
                idx, wts = route_topk(mm("router", l, m[t:t + 1])[0], w["top_k"])
                for j, e in enumerate(idx):
                    g = mm("exp_gate", l, m[t:t + 1], int(e))
                    u = mm("exp_up", l, m[t:t + 1], int(e))
                    f[t] += wts[j] * mm("exp_down", l, R(silu(g) * u), int(e))[0]
            if w["n_shared"] > 0:
                f = f + mm("sh_down", l, R(silu(mm("sh_gate", l, m)) * mm("sh_up", l, m)))
            h = h + f
    return mm("lm_head", -1, R(rmsnorm(h, Wt.vector("final_norm"), eps)))


# ------------------------------------------------------------------ context set-up


def synthetic_cache(w: dict) -> dict:
    """Prefilled cache drawn directly from the generator (workloads whose context forward pass
    is too large for the host); values are bf16 (returned as float64)."""
    parts = {}
    L, ctx = w["n_layers"], w["ctx"]
    for s in workloads.cache_specs(w):
        n = int(np.prod(s["shape"]))
        vals = bf16_bits_to_f64(synth.normal_bf16_bits(w["seed"], s["tid"], n, s["std"])).reshape(s["shape"])
        key = {"k_cache": "k", "v_cache": "v", "latent_cache": "latent", "pe_cache": "pe"}[s["name"]]
        parts.setdefault(key, np.empty((L,) + s["shape"]))[s["layer"]] = vals
    return parts


def build_context(w: dict, weights: Weights | None = None):
    """Oracle decoder with the context of workload `w` in its cache, and the first decode token.

    cache_from == 'oracle': the decoder steps through the seeded context ids and its greedy
    token after the last one is the first decode token.  'synthetic': the cache is drawn
    directly and the first decode token is a seeded id.
    """
    dec = OracleDecoder(w, weights)
    ctx_ids = synth.tokens(w["seed"], synth.TOKENS_CONTEXT, w["ctx"], w["vocab"])
    if w["cache_from"] == "oracle":
        out = None
        for t in ctx_ids:
            out = dec.step(int(t))
        first = out["next"]
    else:
        dec.set_cache(synthetic_cache(w), w["ctx"])
        first = int(synth.tokens(w["seed"], synth.TOKENS_FIRST, 1, w["vocab"])[0])
    return dec, first, ctx_ids
