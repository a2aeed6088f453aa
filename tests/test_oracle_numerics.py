"""Pins of the oracle's number formats and operators against definitions, closed forms and libraries."""
import math
import os

import numpy as np
import pytest
import torch

from oracle import model as om
from oracle import numerics as nm

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def test_e4m3_table_against_spec_fixture():
    for line in open(os.path.join(GOLDEN, "e4m3.txt")):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        code, val = line.split()
        got = nm.E4M3_TABLE[int(code, 16)]
        if val == "nan":
            assert math.isnan(got)
        else:
            assert got == float(val) and math.copysign(1, got) == math.copysign(1, float(val))


def test_e4m3_table_against_torch_all_codes():
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    ours = nm.E4M3_TABLE
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan)
    assert np.array_equal(ours[~nan], ref[~nan])


def test_round_bf16_matches_torch():
    rng = np.random.default_rng(2)
    x = np.concatenate([rng.normal(0, 1, 20000), rng.normal(0, 1e-3, 5000), rng.normal(0, 1e3, 5000),
                        rng.normal(0, 1e-39, 100)])
    ref = torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16).to(torch.float64).numpy()
    # torch rounds the fp32 value; compare on inputs that are exact in fp32
    ours = nm.round_bf16(x.astype(np.float32).astype(np.float64))
    assert np.array_equal(ours, ref)


def test_round_bf16_ties_to_even():
    # 1 + 2^-8 lies halfway between 1 and 1 + 2^-7: ties go to the even significand (1.0)
    assert nm.round_bf16(np.array([1 + 2 ** -8]))[0] == 1.0
    assert nm.round_bf16(np.array([1 + 3 * 2 ** -8]))[0] == 1 + 2 ** -6


def _brute_gemv(Wv, x):
    return np.array([sum(float(Wv[n, k]) * float(x[k]) for k in range(Wv.shape[1])) for n in range(Wv.shape[0])])


def _gemv_case(dtype, rng, N, K):
    """A host weight of `dtype` and its float64 value."""
    if dtype == "f32":
        data = rng.normal(size=(N, K)).astype(np.float32)
        t = dict(dtype="f32", data=data, scales=None)
        Wv = data.astype(np.float64)
    elif dtype == "bf16":
        data = torch.from_numpy(rng.normal(size=(N, K)).astype(np.float32)).to(torch.bfloat16)
        t = dict(dtype="bf16", data=data.view(torch.int16).numpy().view(np.uint16), scales=None)
        Wv = data.to(torch.float64).numpy()
    else:
        q = rng.integers(0, 256, size=(N, K), dtype=np.uint8)
        q[(q & 0x7F) == 0x7F] = 0x10  # no NaN codes in weights
        s = rng.uniform(0.5, 2, size=(3, 3)).astype(np.float32)
        t = dict(dtype="fp8", data=q, scales=s)
        Wv = np.empty((N, K))
        for n in range(N):
            for k in range(K):
                Wv[n, k] = nm.e4m3_value(int(q[n, k])) * float(s[n // 128, k // 128])
    return t, Wv


@pytest.mark.parametrize("dtype", ["f32", "bf16", "fp8"])
def test_gemv_against_brute_force(dtype):
    rng = np.random.default_rng(3)
    N, K = 260, 300  # ragged against the 128-blocks
    x = rng.normal(size=K)
    t, Wv = _gemv_case(dtype, rng, N, K)
    y = om.gemv(t, x)
    ref = _brute_gemv(Wv, x)
    np.testing.assert_allclose(y, ref, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("dtype", ["f32", "bf16", "fp8"])
def test_gemv_acc32_twin_is_float32_summation(dtype):
    """The float32-accumulation twin (a tolerance calibration, not the definition) stays within the
    textbook bound of float32 recursive summation, |y - y_exact| <= gamma_{K+2} * sum|w x| with
    gamma_n = n u / (1 - n u), u = 2^-24, and really does round in float32 (not bit-equal to float64)."""
    rng = np.random.default_rng(5)
    N, K = 260, 300
    x = rng.normal(size=K).astype(np.float32).astype(np.float64)  # activations are float32-exact
    t, Wv = _gemv_case(dtype, rng, N, K)
    y = om.gemv_acc32(t, x)
    ref = _brute_gemv(Wv, x)
    u = 2.0 ** -24
    gamma = (K + 2) * u / (1 - (K + 2) * u)
    assert np.all(np.abs(y - ref) <= gamma * (np.abs(Wv) @ np.abs(x)))
    assert np.any(y != ref)
    assert np.all(y.astype(np.float32).astype(np.float64) == y)


def test_fp8_block_dequant_against_scalar_definition():
    """w[n, k] = E4M3(q[n, k]) * s[n // 128, k // 128] on a ragged 2 x 3 block grid, whose
    distinct per-block scales expose a transposed or shifted block index."""
    rng = np.random.default_rng(12)
    N, K = 200, 300
    q = rng.integers(0, 256, size=(N, K), dtype=np.uint8)
    q[(q & 0x7F) == 0x7F] = 0x22
    s = np.array([[1.0, 2.0, 4.0], [8.0, 16.0, 32.0]], dtype=np.float32)
    W = nm.dequant_fp8_b128(q, s)
    assert W.shape == (N, K)
    for n, k in [(0, 0), (127, 127), (128, 0), (0, 128), (199, 299), (150, 260), (5, 256)]:
        assert W[n, k] == nm.e4m3_value(int(q[n, k])) * float(s[n // 128, k // 128])
    ref = np.array([[nm.e4m3_value(int(q[n, k])) * float(s[n // 128, k // 128]) for k in range(K)]
                    for n in range(0, N, 7)])
    np.testing.assert_array_equal(W[::7], ref)


def test_softmax_brute_force_and_sum():
    x = np.array([0.3, -1.2, 5.0, 5.0, 2.2])
    e = [math.exp(v - 5.0) for v in x]
    ref = np.array(e) / sum(e)
    np.testing.assert_allclose(nm.softmax(x), ref, rtol=1e-15)
    assert nm.softmax(np.random.default_rng(4).normal(size=1000) * 30).sum() == pytest.approx(1.0, abs=1e-14)


def test_rmsnorm_closed_form():
    x = np.array([3.0, 4.0])
    g = np.array([2.0, 0.5])
    r = math.sqrt((9 + 16) / 2 + 1e-6)
    np.testing.assert_allclose(nm.rmsnorm(x, g, 1e-6), [6 / r, 2 / r], rtol=1e-15)
    y = nm.rmsnorm(np.random.default_rng(5).normal(size=512) * 7, np.ones(512), 0.0)
    assert np.mean(y * y) == pytest.approx(1.0, rel=1e-12)


def test_rope_closed_form_and_invariants():
    theta = 10000.0
    # D = 2: a plain rotation by p radians (inv_freq_0 = 1)
    v = nm.rope(np.array([1.0, 0.0]), 3, theta)
    np.testing.assert_allclose(v, [math.cos(3), math.sin(3)], rtol=1e-15)
    rng = np.random.default_rng(6)
    D = 64
    q, k = rng.normal(size=D), rng.normal(size=D)
    # position 0 is the identity
    np.testing.assert_array_equal(nm.rope(q, 0, theta), q)
    # pair norms preserved
    r = nm.rope(q, 17, theta)
    np.testing.assert_allclose(r[:32] ** 2 + r[32:] ** 2, q[:32] ** 2 + q[32:] ** 2, rtol=1e-12)
    # q_m . k_n depends on m - n only
    a = nm.rope(q, 105, theta) @ nm.rope(k, 100, theta)
    b = nm.rope(q, 5, theta) @ nm.rope(k, 0, theta)
    assert a == pytest.approx(b, rel=1e-10)
    # frequencies: theta^(-2j/D)
    f = nm.rope_inv_freq(D, theta)
    assert f[0] == 1.0 and f[1] == pytest.approx(theta ** (-2 / D), rel=1e-15)


def test_silu_closed_form():
    np.testing.assert_allclose(nm.silu(np.array([0.0, 1.0, -1.0, 40.0])),
                               [0.0, 1 / (1 + math.exp(-1)), -1 / (1 + math.exp(1)), 40.0], rtol=1e-15)


def test_argmax_first_matches_numpy():
    rng = np.random.default_rng(7)
    for _ in range(50):
        x = rng.integers(0, 5, size=40).astype(np.float64)  # many ties
        assert nm.argmax_first(x) == int(np.argmax(x))


def test_topk_matches_full_sort_with_ties():
    rng = np.random.default_rng(8)
    for _ in range(50):
        p = rng.integers(0, 6, size=32).astype(np.float64)
        idx = nm.topk_lowest_index(p, 8)
        ref = np.lexsort((np.arange(32), -p))[:8]  # primary: value desc, secondary: index asc
        assert np.array_equal(idx, ref)


def test_margin_topk_hand_example():
    x = np.array([3.0, 1.0, 2.0, 2.0])
    assert nm.margin_topk(x, 1) == 1.0          # 3 vs 2
    assert nm.margin_topk(x, 2) == 0.0          # the two 2s tie across the cut
    assert nm.margin_topk(x, 3) == 1.0          # 2 vs 1
    assert nm.margin_topk(x, 4) == float("inf")  # nothing outside the set


def test_route_weights_sum_to_one():
    rng = np.random.default_rng(9)
    for k in (1, 4, 8):
        idx, w = om.route_topk(rng.normal(size=256) * 2, k)
        assert w.sum() == pytest.approx(1.0, abs=1e-14)
        assert len(set(idx.tolist())) == k


def test_split_lse_combine_equals_single_softmax():
    rng = np.random.default_rng(10)
    T, D = 203, 64
    q, K, V = rng.normal(size=D) * 3, rng.normal(size=(T, D)), rng.normal(size=(T, D))
    ref = nm.softmax(K @ q / math.sqrt(D)) @ V
    for bounds in ([(0, T)], [(0, 50), (50, 51), (51, 203)], [(i, min(T, i + 16)) for i in range(0, T, 16)]):
        np.testing.assert_allclose(om.attention_split_lse(q, K, V, bounds), ref, rtol=1e-12, atol=1e-13)


def test_mla_absorbed_equals_unabsorbed():
    rng = np.random.default_rng(11)
    H, nope, rdim, v, kvl, T = 4, 16, 8, 12, 32, 9
    qn, qpe = rng.normal(size=(H, nope)), rng.normal(size=(H, rdim))
    C, PE = rng.normal(size=(T, kvl)), rng.normal(size=(T, rdim))
    W_UK, W_UV = rng.normal(size=(H, nope, kvl)) * 0.2, rng.normal(size=(H, v, kvl)) * 0.2
    a = om.mla_absorbed(qn, qpe, C, PE, W_UK, W_UV)
    b = om.mla_unabsorbed(qn, qpe, C, PE, W_UK, W_UV)
    np.testing.assert_allclose(a, b, rtol=1e-11, atol=1e-12)
