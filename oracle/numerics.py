"""Scalar formats and elementwise operators of the decode step, in float64.

TEST INFRASTRUCTURE ONLY (see the package docstring).

The pages name the operators of the model (RMSNorm, RoPE, SwiGLU, softmax
routing; TileRT 是什么 §五 5.2) without their formulas; each function states the
textbook definition it implements.
"""
from __future__ import annotations

import numpy as np

# ----------------------------------------------------------------- number formats


def e4m3_value(code: int) -> float:
    """Value of one OCP FP8 E4M3 ("fn") code: 1 sign, 4 exponent (bias 7), 3 mantissa bits.

    Exponent field 0 encodes subnormals m/8 * 2^-6; S.1111.111 is NaN; there
    are no infinities, so S.1111.110 = +-448 is the largest finite value.
    """
    s = -1.0 if code & 0x80 else 1.0
    e = (code >> 3) & 0xF
    m = code & 0x7
    if e == 0xF and m == 0x7:
        return float("nan")
    if e == 0:
        return s * (m / 8.0) * 2.0 ** -6
    return s * (1.0 + m / 8.0) * 2.0 ** (e - 7)


E4M3_TABLE = np.array([e4m3_value(c) for c in range(256)], dtype=np.float64)


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns -> values: bf16 is the upper half of an IEEE binary32."""
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def round_bf16(x: np.ndarray) -> np.ndarray:
    """Round float64 values to the nearest bf16 (8 significant bits, 8-bit exponent), ties to even.

    Written from the format: for a normal value with exponent e the bf16 grid
    spacing is 2^(e-7); below 2^-126 the spacing is the subnormal one, 2^-133.
    Values beyond the largest finite bf16 are not produced by the decoder.
    """
    x = np.asarray(x, dtype=np.float64)
    out = np.zeros_like(x)
    nz = x != 0
    ax = np.abs(x[nz])
    e = np.floor(np.log2(ax))
    # guard against log2 rounding at exact powers of two
    e = np.where(2.0 ** e > ax, e - 1, e)
    e = np.where(2.0 ** (e + 1) <= ax, e + 1, e)
    spacing = 2.0 ** (np.maximum(e, -126.0) - 7.0)
    out[nz] = np.sign(x[nz]) * np.round(ax / spacing) * spacing  # np.round: half to even
    return out


def round_f32(x: np.ndarray) -> np.ndarray:
    return np.asarray(x, dtype=np.float64).astype(np.float32).astype(np.float64)


def rounder(act_dtype: str):
    """The rounding applied at each activation contract point of the model definition."""
    return round_bf16 if act_dtype == "bf16" else round_f32


def identity(x):
    return np.asarray(x, dtype=np.float64)


def dequant_fp8_b128(q: np.ndarray, s: np.ndarray) -> np.ndarray:
    """Block-scaled FP8 weight: w[n, k] = E4M3(q[n, k]) * s[n // 128, k // 128] (exact in float64)."""
    n, k = q.shape
    srow = np.repeat(np.repeat(s.astype(np.float64), 128, axis=0), 128, axis=1)[:n, :k]
    return E4M3_TABLE[q] * srow


# ----------------------------------------------------------------------- operators


def rmsnorm(x: np.ndarray, g: np.ndarray, eps: float) -> np.ndarray:
    """RMSNorm (Zhang & Sennrich 2019): y = x / sqrt(mean(x^2) + eps) * g."""
    x = np.asarray(x, dtype=np.float64)
    return x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps) * np.asarray(g, dtype=np.float64)


def rope_inv_freq(dim: int, theta: float) -> np.ndarray:
    """RoPE frequencies (Su et al. 2021): inv_freq_j = theta^(-2j/dim), j < dim/2."""
    return theta ** (-2.0 * np.arange(dim // 2, dtype=np.float64) / dim)


def rope(x: np.ndarray, pos, theta: float) -> np.ndarray:
    """Rotary embedding of the last axis with half-split pairing (x_j, x_{j+D/2}).

    x'_j       = x_j cos(p w_j) - x_{j+D/2} sin(p w_j)
    x'_{j+D/2} = x_j sin(p w_j) + x_{j+D/2} cos(p w_j)
    `pos` is a scalar or an array broadcast against x's leading axes.
    """
    x = np.asarray(x, dtype=np.float64)
    D = x.shape[-1]
    ang = np.asarray(pos, dtype=np.float64)[..., None] * rope_inv_freq(D, theta)
    c, s = np.cos(ang), np.sin(ang)
    a, b = x[..., : D // 2], x[..., D // 2:]
    return np.concatenate([a * c - b * s, a * s + b * c], axis=-1)


def softmax(x: np.ndarray, axis: int = -1) -> np.ndarray:
    x = np.asarray(x, dtype=np.float64)
    m = np.max(x, axis=axis, keepdims=True)
    e = np.exp(x - m)
    return e / np.sum(e, axis=axis, keepdims=True)


def silu(x: np.ndarray) -> np.ndarray:
    """SiLU (Elfwing et al. 2018): x * sigmoid(x) = x / (1 + e^-x)."""
    x = np.asarray(x, dtype=np.float64)
    return x / (1.0 + np.exp(-x))


def argmax_first(x: np.ndarray) -> int:
    """Greedy decoding: the smallest index among the maxima."""
    x = np.asarray(x)
    m = np.max(x)
    return int(np.flatnonzero(x == m)[0])


def topk_lowest_index(p: np.ndarray, k: int) -> np.ndarray:
    """Indices of the k largest entries, ordered by value descending, ties to the lower index."""
    p = np.asarray(p)
    order = sorted(range(p.shape[0]), key=lambda i: (-p[i], i))
    return np.array(order[:k], dtype=np.int64)


def margin_topk(logits: np.ndarray, k: int) -> float:
    """Gap between the k-th and (k+1)-th largest entries; infinite when there is no (k+1)-th
    entry (the top-k set is then forced, so no decision is near a tie)."""
    s = np.sort(np.asarray(logits, dtype=np.float64))[::-1]
    return float(s[k - 1] - s[k]) if s.shape[0] > k else float("inf")
