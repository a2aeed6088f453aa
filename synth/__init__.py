"""Seeded synthetic inputs shared by the oracle side and the GPU side.

This package makes inputs only: weights, norm gains, token ids and the
prefilled caches that the prefill engine would hand over.  It holds none of the
decode arithmetic.  `synth.c` (CPU) and `synth_cuda.cu` (GPU) each implement
the same published counter-based generator (SplitMix64, Steele/Lea/Flood 2014);
tests check that they agree byte for byte.

Tensor streams are keyed by (seed, tensor id); `tensor_id()` builds the id from
the tensor's kind, layer and expert index.
"""
from __future__ import annotations

import ctypes
import math
import os

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
CPU_LIB = os.path.join(_HERE, "libsynth.so")
GPU_LIB = os.path.join(_HERE, "libsynth_cuda.so")

# Tensor kinds of the synthetic workloads (ids of the generator streams).
KIND = {
    "embed": 1, "final_norm": 2, "lm_head": 3,
    "attn_norm": 10, "wq": 11, "wk": 12, "wv": 13, "wo": 14, "ffn_norm": 15,
    "w_gate": 16, "w_up": 17, "w_down": 18,
    "q_a": 20, "q_a_norm": 21, "q_b": 22, "kv_a": 23, "kv_a_norm": 24, "kv_b": 25,
    "router": 30, "exp_gate": 31, "exp_up": 32, "exp_down": 33,
    "sh_gate": 34, "sh_up": 35, "sh_down": 36,
    "k_cache": 40, "v_cache": 41, "latent_cache": 42, "pe_cache": 43,
}
TOKENS_CONTEXT = 0xC0
TOKENS_FIRST = 0xC1

# Irwin-Hall(4) of 16-bit uniforms: variance of the centred sum.
_IH_STD = math.sqrt((65536.0 ** 2 - 1.0) / 3.0)


def tensor_id(kind: str, layer: int = -1, expert: int = -1) -> int:
    return ((layer + 1) << 24) | (KIND[kind] << 16) | (expert + 1)


def scale_for_std(std: float) -> float:
    """fp32 constant c such that fp32(n) * c has standard deviation `std`."""
    return float(np.float32(std / _IH_STD))


# --------------------------------------------------------------------------- CPU
_cpu = None


def cpu_lib():
    global _cpu
    if _cpu is None:
        if not os.path.exists(CPU_LIB):
            raise RuntimeError(f"{CPU_LIB} missing: run __graft_entry__.build()")
        lib = ctypes.CDLL(CPU_LIB)
        u64, i64, f32 = ctypes.c_uint64, ctypes.c_int64, ctypes.c_float
        vp = ctypes.c_void_p
        lib.synth_mix64.restype = u64
        lib.synth_mix64.argtypes = [u64]
        lib.synth_stream.restype = u64
        lib.synth_stream.argtypes = [u64, u64]
        lib.synth_draw.restype = u64
        lib.synth_draw.argtypes = [u64, u64]
        lib.synth_normal_f32.argtypes = [u64, u64, u64, u64, f32, f32, vp]
        lib.synth_normal_bf16.argtypes = [u64, u64, u64, u64, f32, f32, vp]
        lib.synth_fp8_b128.argtypes = [u64, u64, i64, i64, f32, vp, vp]
        lib.synth_tokens.argtypes = [u64, u64, u64, u64, ctypes.c_uint32, vp]
        lib.synth_e4m3_rne.restype = ctypes.c_uint8
        lib.synth_e4m3_rne.argtypes = [f32]
        lib.synth_bf16_rne.restype = ctypes.c_uint16
        lib.synth_bf16_rne.argtypes = [f32]
        _cpu = lib
    return _cpu


def normal_f32(seed, tid, n, std, offset=0.0, start=0) -> np.ndarray:
    out = np.empty(n, dtype=np.float32)
    cpu_lib().synth_normal_f32(seed, tid, start, n, scale_for_std(std), offset, out.ctypes.data)
    return out


def normal_bf16_bits(seed, tid, n, std, offset=0.0, start=0) -> np.ndarray:
    """bf16 bit patterns (uint16) of the fp32 values, rounded to nearest even."""
    out = np.empty(n, dtype=np.uint16)
    cpu_lib().synth_normal_bf16(seed, tid, start, n, scale_for_std(std), offset, out.ctypes.data)
    return out


def fp8_b128(seed, tid, rows, cols, std):
    """E4M3 codes [rows][cols] (uint8) and fp32 scales [ceil(rows/128)][ceil(cols/128)]."""
    q = np.empty((rows, cols), dtype=np.uint8)
    s = np.empty(((rows + 127) // 128, (cols + 127) // 128), dtype=np.float32)
    cpu_lib().synth_fp8_b128(seed, tid, rows, cols, scale_for_std(std), q.ctypes.data, s.ctypes.data)
    return q, s


def tokens(seed, tid, n, vocab, start=0) -> np.ndarray:
    out = np.empty(n, dtype=np.int32)
    cpu_lib().synth_tokens(seed, tid, start, n, vocab, out.ctypes.data)
    return out


# --------------------------------------------------------------------------- GPU
_gpu = None


def gpu_lib():
    global _gpu
    if _gpu is None:
        if not os.path.exists(GPU_LIB):
            raise RuntimeError(f"{GPU_LIB} missing: run __graft_entry__.build()")
        lib = ctypes.CDLL(GPU_LIB)
        u64, i64, f32, vp = ctypes.c_uint64, ctypes.c_int64, ctypes.c_float, ctypes.c_void_p
        lib.synthc_normal_f32.argtypes = [u64, u64, u64, u64, f32, f32, vp, vp]
        lib.synthc_normal_bf16.argtypes = [u64, u64, u64, u64, f32, f32, vp, vp]
        lib.synthc_fp8_b128.argtypes = [u64, u64, i64, i64, f32, vp, vp, vp]
        lib.synthc_tokens.argtypes = [u64, u64, u64, u64, ctypes.c_uint32, vp, vp]
        for f in ("synthc_normal_f32", "synthc_normal_bf16", "synthc_fp8_b128", "synthc_tokens"):
            getattr(lib, f).restype = ctypes.c_int
        _gpu = lib
    return _gpu


def _check(rc, what):
    if rc != 0:
        raise RuntimeError(f"{what} failed with CUDA error {rc}")


def _stream_ptr(stream):
    return 0 if stream is None else int(stream.cuda_stream)


def gpu_normal_f32(out, seed, tid, std, offset=0.0, start=0, stream=None):
    _check(gpu_lib().synthc_normal_f32(seed, tid, start, out.numel(), scale_for_std(std), offset,
                                       out.data_ptr(), _stream_ptr(stream)), "synthc_normal_f32")


def gpu_normal_bf16(out, seed, tid, std, offset=0.0, start=0, stream=None):
    _check(gpu_lib().synthc_normal_bf16(seed, tid, start, out.numel(), scale_for_std(std), offset,
                                        out.data_ptr(), _stream_ptr(stream)), "synthc_normal_bf16")


def gpu_fp8_b128(q, s, seed, tid, rows, cols, std, stream=None):
    _check(gpu_lib().synthc_fp8_b128(seed, tid, rows, cols, scale_for_std(std), q.data_ptr(), s.data_ptr(),
                                     _stream_ptr(stream)), "synthc_fp8_b128")


def gpu_tokens(out, seed, tid, vocab, start=0, stream=None):
    _check(gpu_lib().synthc_tokens(seed, tid, start, out.numel(), vocab, out.data_ptr(), _stream_ptr(stream)),
           "synthc_tokens")
