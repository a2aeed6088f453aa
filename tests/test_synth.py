"""Seeded input generator (CPU side): published SplitMix64 vectors, E4M3/bf16 encoders, block-FP8 recipe."""
import math
import os

import numpy as np
import pytest
import torch

import synth
from oracle.numerics import E4M3_TABLE
from synth import workloads

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _read_splitmix_vectors():
    cases, cur = [], None
    for line in open(os.path.join(GOLDEN, "splitmix64.txt")):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        if line.startswith("seed"):
            cur = (int(line.split()[1], 0), [])
            cases.append(cur)
        else:
            cur[1].append(int(line, 0))
    return cases


def test_splitmix64_published_vectors():
    L = synth.cpu_lib()
    for seed, outs in _read_splitmix_vectors():
        got = [L.synth_draw(seed, i) for i in range(len(outs))]
        assert got == outs


def test_e4m3_encoder_matches_torch_rne():
    L = synth.cpu_lib()
    rng = np.random.default_rng(0)
    xs = np.concatenate([rng.normal(0, 50, 20000), rng.normal(0, 0.01, 20000), rng.uniform(-448, 448, 20000),
                         (E4M3_TABLE[0:0x7E] + E4M3_TABLE[1:0x7F]) / 2]).astype(np.float32)  # exact ties
    xs = xs[np.abs(xs) <= 448]
    ours = np.array([L.synth_e4m3_rne(float(x)) for x in xs], dtype=np.uint8)
    ref = torch.from_numpy(xs).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(ours, ref)


def test_e4m3_encoder_saturates():
    L = synth.cpu_lib()
    assert L.synth_e4m3_rne(449.0) == 0x7E
    assert L.synth_e4m3_rne(1e30) == 0x7E
    assert L.synth_e4m3_rne(-1e30) == 0xFE


def test_bf16_encoder_matches_torch():
    L = synth.cpu_lib()
    rng = np.random.default_rng(1)
    xs = np.concatenate([rng.normal(0, 1, 5000), rng.normal(0, 1e-30, 500), rng.normal(0, 1e30, 500)])
    xs = xs.astype(np.float32)
    ours = np.array([L.synth_bf16_rne(float(x)) for x in xs], dtype=np.uint16)
    ref = torch.from_numpy(xs).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)


def test_irwin_hall_moments():
    v = synth.normal_f32(7, 123, 200000, 0.02)
    assert abs(v.mean()) < 0.02 * 0.01
    assert abs(v.std() / 0.02 - 1) < 0.01
    # bounded support of Irwin-Hall(4): |n| <= 131070
    assert np.max(np.abs(v)) <= 131070 * synth.scale_for_std(0.02) * (1 + 1e-6)


def test_streams_are_offsettable():
    a = synth.normal_f32(3, 99, 1000, 1.0)
    b = synth.normal_f32(3, 99, 400, 1.0, start=600)
    assert np.array_equal(a[600:], b)
    g = synth.normal_f32(3, 98, 1000, 0.1, offset=1.0)
    assert abs(g.mean() - 1) < 0.02


def test_fp8_block_recipe():
    rows, cols = 300, 200  # ragged in both directions
    q, s = synth.fp8_b128(5, 77, rows, cols, 0.02)
    v = synth.normal_f32(5, 77, rows * cols, 0.02).reshape(rows, cols)
    assert s.shape == (3, 2)
    for br in range(3):
        for bc in range(2):
            blk = v[br * 128:(br + 1) * 128, bc * 128:(bc + 1) * 128]
            amax = np.float32(np.max(np.abs(blk)))
            assert s[br, bc] == np.float32(amax / np.float32(448.0))
            deq = E4M3_TABLE[q[br * 128:(br + 1) * 128, bc * 128:(bc + 1) * 128]] * float(s[br, bc])
            # round to nearest within E4M3's relative half-ulp (2^-4) or the subnormal grid
            err = np.abs(deq - blk)
            bound = np.maximum(np.abs(blk) * 2.0 ** -4, 2.0 ** -10 * float(s[br, bc])) * (1 + 1e-6)
            assert np.all(err <= bound)
            assert np.max(np.abs(deq)) == pytest.approx(float(amax), rel=1e-6)


def test_tokens_in_range():
    t = synth.tokens(1, synth.TOKENS_CONTEXT, 5000, 1000)
    assert t.min() >= 0 and t.max() < 1000
    assert len(np.unique(t)) > 900


def test_workload_bytes_match_hand_count():
    # dense BF16 1k workload: 16 layers of (qkv 3072x2048 + o 2048^2 + 3 x 8192x2048) + LM head 32000x2048
    w = workloads.get("dense_gqa_bf16_1k")
    b = workloads.active_bytes_per_token(w, T_mean=1536)
    per_layer = 3072 * 2048 + 2048 * 2048 + 3 * 8192 * 2048
    assert b["weights"] == (16 * per_layer + 32000 * 2048) * 2
    assert b["kv"] == 16 * 2 * 8 * 64 * 2 * 1536
    specs = workloads.weight_specs(w)
    assert sum(1 for s in specs if s["name"] == "wq") == 16
    m = workloads.get("moe_mla_fp8_1k")
    bm = workloads.active_bytes_per_token(m, T_mean=1536)
    assert 7.9e9 < bm["total"] < 8.1e9
    assert math.isclose(bm["kv"], 12 * 576 * 2 * 1536)
