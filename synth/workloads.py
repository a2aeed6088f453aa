"""Synthetic decode workloads: model shapes, seeds and the recipe of every input.

Each workload names a decoder shape (dense GQA or MLA+MoE), its weight dtype,
the prefilled context length handed to the decoder and the number of decode
steps.  The five full-size workloads follow the model structure of the pages
(TileRT 是什么, §五 5.2: 61-layer DeepSeek-V3.2-Exp with MLA, 256 routed experts
with 8 active, d_model 7168, vocab 129,280; cut to 12 layers here) and the
InferenceX 1k/1k and 8k/1k decode shapes (SemiAnalysis TileRT InferenceX
article, results section).  The small workloads are parity cases sized so the
CPU oracle finishes in seconds while every kernel still runs several tiles
and a ragged tail.

Recipe (all values from the seeded generator in this package):
  * linear weights ~ N(0, 0.02^2); FP8 configs quantise per 128x128 block;
  * norm gains = 1 + N(0, 0.1^2) (fp32);
  * embeddings ~ N(0, 0.02^2) in the activation dtype (fp32 or bf16);
  * context token ids uniform in [0, vocab) (stream TOKENS_CONTEXT);
  * prefilled caches: where the oracle can run the context forward pass in
    seconds (tiny configs) the cache comes from that pass; otherwise each
    cache entry is drawn directly with the statistics of such a cache:
    keys/values and the RoPE key ~ N(0, (0.02*sqrt(d_model))^2) (a projection
    of a unit-RMS vector by N(0, 0.02^2) weights), MLA latent ~ N(0, 1) (an
    RMS-normalised vector).
"""
from __future__ import annotations

import copy
import math

from . import tensor_id

WEIGHT_STD = 0.02
GAIN_STD = 0.1

_BASE_DENSE = dict(arch="dense", rope_theta=10000.0, norm_eps=1e-6,
                   q_lora=0, kv_lora=0, qk_nope=0, qk_rope=0, v_head=0,
                   n_dense_layers=0, n_experts=0, top_k=0, n_shared=0, expert_hidden=0)
_BASE_MLA = dict(arch="mla_moe", rope_theta=10000.0, norm_eps=1e-6,
                 kv_lora=512, qk_nope=128, qk_rope=64, v_head=128, n_kv_heads=0, head_dim=0, n_shared=1)

WORKLOADS = {
    # --- the five full-size workloads
    "tiny_dense_f32": dict(_BASE_DENSE, n_layers=2, d_model=256, n_heads=4, n_kv_heads=4, head_dim=64,
                           ffn_hidden=688, vocab=1024, weight_dtype="f32", ctx=64, n_decode=16, seed=1001,
                           cache_from="oracle"),
    "dense_gqa_bf16_1k": dict(_BASE_DENSE, n_layers=16, d_model=2048, n_heads=32, n_kv_heads=8, head_dim=64,
                              ffn_hidden=8192, vocab=32000, weight_dtype="bf16", ctx=1024, n_decode=1024,
                              seed=1002, cache_from="synthetic"),
    "dense_gqa_fp8_8k": dict(_BASE_DENSE, n_layers=32, d_model=4096, n_heads=32, n_kv_heads=8, head_dim=128,
                             ffn_hidden=14336, vocab=128256, weight_dtype="fp8", ctx=8192, n_decode=1024,
                             seed=1003, cache_from="synthetic"),
    "moe_mla_fp8_1k": dict(_BASE_MLA, n_layers=12, d_model=7168, n_heads=128, q_lora=1536, n_dense_layers=3,
                           ffn_hidden=18432, n_experts=256, top_k=8, expert_hidden=2048, vocab=129280,
                           weight_dtype="fp8", ctx=1024, n_decode=1024, seed=1004, cache_from="synthetic"),
    "moe_mla_fp8_8k": dict(_BASE_MLA, n_layers=12, d_model=7168, n_heads=128, q_lora=1536, n_dense_layers=3,
                           ffn_hidden=18432, n_experts=256, top_k=8, expert_hidden=2048, vocab=129280,
                           weight_dtype="fp8", ctx=8192, n_decode=1024, seed=1004, cache_from="synthetic"),
    # --- profiling case: one MoE layer of the full-size MLA model with 16 experts and a
    # short vocabulary (~1.1 GB of weights, ~0.7 GB streamed per step: above the L2, small
    # enough for an ncu capture that saves and restores device memory between passes)
    "prof_mla_moe_fp8": dict(_BASE_MLA, n_layers=1, d_model=7168, n_heads=128, q_lora=1536, n_dense_layers=0,
                             ffn_hidden=18432, n_experts=16, top_k=8, expert_hidden=2048, vocab=8192,
                             weight_dtype="fp8", ctx=1024, n_decode=64, seed=3004, cache_from="synthetic"),
    # --- small parity cases (several tiles, ragged tails, all code paths)
    "small_dense_bf16": dict(_BASE_DENSE, n_layers=2, d_model=384, n_heads=6, n_kv_heads=2, head_dim=64,
                             ffn_hidden=1000, vocab=1000, weight_dtype="bf16", ctx=77, n_decode=6, seed=2002,
                             cache_from="oracle"),
    "small_dense_fp8": dict(_BASE_DENSE, n_layers=2, d_model=384, n_heads=4, n_kv_heads=2, head_dim=128,
                            ffn_hidden=1040, vocab=1000, weight_dtype="fp8", ctx=150, n_decode=6, seed=2003,
                            cache_from="oracle"),
    "small_dense_g8_bf16": dict(_BASE_DENSE, n_layers=2, d_model=512, n_heads=16, n_kv_heads=2, head_dim=128,
                                ffn_hidden=1024, vocab=1000, weight_dtype="bf16", ctx=90, n_decode=6, seed=2005,
                                cache_from="oracle"),
    "small_dense_g8_fp8_hd64": dict(_BASE_DENSE, n_layers=2, d_model=512, n_heads=8, n_kv_heads=1, head_dim=64,
                                    ffn_hidden=1024, vocab=1000, weight_dtype="fp8", ctx=70, n_decode=6, seed=2006,
                                    cache_from="oracle"),
    "small_mla_moe_fp8": dict(_BASE_MLA, n_layers=3, d_model=512, n_heads=16, q_lora=384, n_dense_layers=1,
                              ffn_hidden=1024, n_experts=16, top_k=4, expert_hidden=256, vocab=1000,
                              weight_dtype="fp8", ctx=100, n_decode=6, seed=2004, cache_from="oracle"),
}


def get(name: str, **overrides) -> dict:
    w = copy.deepcopy(WORKLOADS[name])
    w.update(overrides)
    w["name"] = name
    w["max_seq"] = w["ctx"] + w["n_decode"]
    return w


def act_dtype(w) -> str:
    return "f32" if w["weight_dtype"] == "f32" else "bf16"


def weight_specs(w):
    """Every weight tensor of workload `w`, in load order.

    Each spec: dict(name, layer, expert, shape, dtype ('f32'|'bf16'|'fp8'),
    std, offset, tid).  Vectors (norm gains) are always fp32; the embedding
    table uses the activation dtype; all matrices use the weight dtype.
    """
    d, L, V = w["d_model"], w["n_layers"], w["vocab"]
    wd, ad = w["weight_dtype"], act_dtype(w)
    specs = []

    def add(name, shape, dtype, layer=-1, expert=-1, std=WEIGHT_STD, offset=0.0):
        specs.append(dict(name=name, layer=layer, expert=expert, shape=tuple(shape), dtype=dtype, std=std,
                          offset=offset, tid=tensor_id(name, layer, expert)))

    def gain(name, n, layer=-1):
        add(name, (n,), "f32", layer, std=GAIN_STD, offset=1.0)

    add("embed", (V, d), ad)
    for l in range(L):
        gain("attn_norm", d, l)
        if w["arch"] == "dense":
            hq, hkv, hd = w["n_heads"], w["n_kv_heads"], w["head_dim"]
            add("wq", (hq * hd, d), wd, l)
            add("wk", (hkv * hd, d), wd, l)
            add("wv", (hkv * hd, d), wd, l)
            add("wo", (d, hq * hd), wd, l)
        else:
            H = w["n_heads"]
            add("q_a", (w["q_lora"], d), wd, l)
            gain("q_a_norm", w["q_lora"], l)
            add("q_b", (H * (w["qk_nope"] + w["qk_rope"]), w["q_lora"]), wd, l)
            add("kv_a", (w["kv_lora"] + w["qk_rope"], d), wd, l)
            gain("kv_a_norm", w["kv_lora"], l)
            add("kv_b", (H * (w["qk_nope"] + w["v_head"]), w["kv_lora"]), wd, l)
            add("wo", (d, H * w["v_head"]), wd, l)
        gain("ffn_norm", d, l)
        if w["arch"] == "dense" or l < w["n_dense_layers"]:
            ff = w["ffn_hidden"]
            add("w_gate", (ff, d), wd, l)
            add("w_up", (ff, d), wd, l)
            add("w_down", (d, ff), wd, l)
        else:
            eh = w["expert_hidden"]
            add("router", (w["n_experts"], d), wd, l)
            for e in range(w["n_experts"]):
                add("exp_gate", (eh, d), wd, l, e)
                add("exp_up", (eh, d), wd, l, e)
                add("exp_down", (d, eh), wd, l, e)
            if w["n_shared"] > 0:
                sh = eh * w["n_shared"]
                add("sh_gate", (sh, d), wd, l)
                add("sh_up", (sh, d), wd, l)
                add("sh_down", (d, sh), wd, l)
    gain("final_norm", d)
    add("lm_head", (V, d), wd)
    return specs


def cache_specs(w):
    """Synthetic prefilled-cache tensors per layer (used when cache_from == 'synthetic').

    Dense: k_cache, v_cache [n_kv_heads][ctx][head_dim].  MLA: latent_cache
    [ctx][kv_lora] and pe_cache [ctx][qk_rope].  Stored in the activation dtype.
    """
    d, ctx = w["d_model"], w["ctx"]
    proj_std = WEIGHT_STD * math.sqrt(d)
    specs = []
    for l in range(w["n_layers"]):
        if w["arch"] == "dense":
            shp = (w["n_kv_heads"], ctx, w["head_dim"])
            specs.append(dict(name="k_cache", layer=l, shape=shp, std=proj_std, tid=tensor_id("k_cache", l)))
            specs.append(dict(name="v_cache", layer=l, shape=shp, std=proj_std, tid=tensor_id("v_cache", l)))
        else:
            specs.append(dict(name="latent_cache", layer=l, shape=(ctx, w["kv_lora"]), std=1.0,
                              tid=tensor_id("latent_cache", l)))
            specs.append(dict(name="pe_cache", layer=l, shape=(ctx, w["qk_rope"]), std=proj_std,
                              tid=tensor_id("pe_cache", l)))
    return specs


def active_bytes_per_token(w, T_mean: float) -> dict:
    """Algorithmic HBM bytes one decode step must read (weights actually used, FP8 scales, KV read).

    The embedding contributes one row; the routed experts contribute top_k of n_experts.
    """
    d, L, V = w["d_model"], w["n_layers"], w["vocab"]
    wb = {"f32": 4, "bf16": 2, "fp8": 1}[w["weight_dtype"]]
    ab = 4 if w["weight_dtype"] == "f32" else 2
    mats = []  # (rows, cols) of every matrix read in one step
    for l in range(L):
        if w["arch"] == "dense":
            hq, hkv, hd = w["n_heads"], w["n_kv_heads"], w["head_dim"]
            mats += [((hq + 2 * hkv) * hd, d), (d, hq * hd)]
        else:
            H = w["n_heads"]
            mats += [(w["q_lora"], d), (H * (w["qk_nope"] + w["qk_rope"]), w["q_lora"]),
                     (w["kv_lora"] + w["qk_rope"], d), (H * (w["qk_nope"] + w["v_head"]), w["kv_lora"]),
                     (d, H * w["v_head"])]
        if w["arch"] == "dense" or l < w["n_dense_layers"]:
            ff = w["ffn_hidden"]
            mats += [(2 * ff, d), (d, ff)]
        else:
            eh = w["expert_hidden"]
            n_act = w["top_k"] + w["n_shared"]
            mats += [(w["n_experts"], d)] + [(2 * eh, d), (d, eh)] * n_act
    mats.append((V, d))
    weights = sum(r * c for r, c in mats) * wb
    scales = sum(((r + 127) // 128) * ((c + 127) // 128) for r, c in mats) * 4 if wb == 1 else 0
    if w["arch"] == "dense":
        kv = L * 2 * w["n_kv_heads"] * w["head_dim"] * ab * T_mean
    else:
        kv = L * (w["kv_lora"] + w["qk_rope"]) * ab * T_mean
    return dict(weights=weights, scales=scales, kv=kv, embed=d * ab, total=weights + scales + kv + d * ab)
