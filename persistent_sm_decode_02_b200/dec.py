"""ctypes binding of libdec.so with the C ABI's names (include/dec.h).

The module-level functions (dec_create, dec_load_weights, ...) mirror the C
entry points one to one; `Decoder` wraps a context for convenience.  Device
memory is handed over as integer addresses (e.g. torch.Tensor.data_ptr());
host memory as numpy arrays.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libdec.so")

# ---- constants (include/dec.h)
DEC_OK = 0
DEC_ERR_INVALID_ARG = -1
DEC_ERR_STATE = -2
DEC_ERR_CAPACITY = -3
DEC_ERR_OOM = -4
DEC_ERR_CUDA = -5
DEC_ERR_TIMEOUT = -6
DEC_ERR_UNSUPPORTED = -7
DEC_ERR_NUMERIC = -8

DEC_ARCH_DENSE = 0
DEC_ARCH_MLA_MOE = 1
DEC_F32 = 0
DEC_BF16 = 1
DEC_FP8_E4M3_B128 = 2
DEC_PERSISTENT = 0
DEC_PER_OP = 1
DEC_PER_OP_GRAPH = 2
DEC_FLAG_TRACE = 1
DEC_FLAG_TEST_STALL = 2

DEC_W = dict(embed=1, final_norm=2, lm_head=3, attn_norm=10, wq=11, wk=12, wv=13, wo=14, ffn_norm=15,
             w_gate=16, w_up=17, w_down=18, q_a=20, q_a_norm=21, q_b=22, kv_a=23, kv_a_norm=24, kv_b=25,
             router=30, exp_gate=31, exp_up=32, exp_down=33, sh_gate=34, sh_up=35, sh_down=36)

DEC_DUMP_KV = 1
DEC_DUMP_ROUTES = 2
DEC_DUMP_TRACE = 3
DEC_DUMP_PLAN = 4
DEC_DUMP_WEIGHTS = 5
DEC_DUMP_TRACE_PRODUCER = 6
DEC_DUMP_STATUS = 7
DEC_DUMP_OP = 100

EXPORTED = ["dec_create", "dec_load_weights", "dec_set_kv_cache", "dec_step", "dec_step_async", "dec_sync",
            "dec_reset", "dec_destroy", "dec_set_stream", "dec_set_exec_mode", "dec_position", "dec_debug_dump",
            "dec_last_error", "dec_attention_noalloc", "dec_generate_async", "dec_generate_poll",
            "dec_generate_stop", "dec_generate_wait", "dec_generate"]


class dec_config(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in ("arch", "n_layers", "d_model", "vocab", "max_seq", "n_heads",
                                               "n_kv_heads", "head_dim", "ffn_hidden", "q_lora", "kv_lora",
                                               "qk_nope", "qk_rope", "v_head", "n_dense_layers", "n_experts",
                                               "top_k", "n_shared", "expert_hidden")] + [
        ("rope_theta", ctypes.c_float), ("norm_eps", ctypes.c_float), ("weight_dtype", ctypes.c_int32),
        ("exec_mode", ctypes.c_int32), ("device", ctypes.c_int32), ("wait_timeout_us", ctypes.c_uint32),
        ("flags", ctypes.c_uint32), ("n_ctas", ctypes.c_int32)]


class dec_tensor(ctypes.Structure):
    _fields_ = [("kind", ctypes.c_int32), ("layer", ctypes.c_int32), ("expert", ctypes.c_int32),
                ("data", ctypes.c_void_p), ("scales", ctypes.c_void_p), ("bytes", ctypes.c_size_t)]


_lib = None


def load_library():
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with __graft_entry__.build(); "
                               "this package has no CPU fallback")
        L = ctypes.CDLL(LIB_PATH)
        P = ctypes.c_void_p
        sig = {
            "dec_create": [ctypes.POINTER(dec_config), ctypes.POINTER(P)],
            "dec_load_weights": [P, ctypes.POINTER(dec_tensor), ctypes.c_int],
            "dec_set_kv_cache": [P, P, P, ctypes.c_int32],
            "dec_step": [P, ctypes.c_int32, P, ctypes.POINTER(ctypes.c_int32)],
            "dec_step_async": [P, ctypes.c_int32],
            "dec_sync": [P, P, ctypes.POINTER(ctypes.c_int32)],
            "dec_reset": [P],
            "dec_destroy": [P],
            "dec_set_stream": [P, P],
            "dec_set_exec_mode": [P, ctypes.c_int32],
            "dec_position": [P, ctypes.POINTER(ctypes.c_int32)],
            "dec_debug_dump": [P, ctypes.c_int32, P, ctypes.c_size_t, ctypes.POINTER(ctypes.c_size_t)],
            "dec_attention_noalloc": [P, P, P, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                                      ctypes.c_int32, P, P],
            "dec_generate_async": [P, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32],
            "dec_generate_poll": [P, P, ctypes.c_int32, ctypes.POINTER(ctypes.c_int32), ctypes.POINTER(ctypes.c_int32)],
            "dec_generate_stop": [P],
            "dec_generate_wait": [P, P, ctypes.c_int32, ctypes.POINTER(ctypes.c_int32)],
            "dec_generate": [P, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, P, ctypes.POINTER(ctypes.c_int32)],
        }
        for name, args in sig.items():
            f = getattr(L, name)
            f.argtypes = args
            f.restype = ctypes.c_int
        L.dec_last_error.argtypes = [P]
        L.dec_last_error.restype = ctypes.c_char_p
        _lib = L
    return _lib


class DecError(RuntimeError):
    def __init__(self, code, msg):
        super().__init__(f"{msg} (code {code})")
        self.code = code


def _chk(ctx, rc):
    if rc != DEC_OK:
        msg = load_library().dec_last_error(ctx).decode() if ctx else "error"
        raise DecError(rc, msg)


# ---- one-to-one wrappers of the C entry points (return the C status code)
def dec_create(cfg: dec_config):
    out = ctypes.c_void_p()
    rc = load_library().dec_create(ctypes.byref(cfg), ctypes.byref(out))
    return rc, out


def dec_load_weights(ctx, tensors):
    arr = (dec_tensor * len(tensors))(*tensors)
    return load_library().dec_load_weights(ctx, arr, len(tensors))


def dec_set_kv_cache(ctx, k_or_latent, v_or_pe, n_tokens):
    return load_library().dec_set_kv_cache(ctx, k_or_latent, v_or_pe, n_tokens)


def dec_step(ctx, token_id, out_logits, out_next):
    return load_library().dec_step(ctx, token_id, out_logits, out_next)


def dec_step_async(ctx, token_id):
    return load_library().dec_step_async(ctx, token_id)


def dec_sync(ctx, out_logits, out_next):
    return load_library().dec_sync(ctx, out_logits, out_next)


def dec_reset(ctx):
    return load_library().dec_reset(ctx)


def dec_destroy(ctx):
    return load_library().dec_destroy(ctx)


def dec_set_stream(ctx, stream):
    return load_library().dec_set_stream(ctx, stream)


def dec_set_exec_mode(ctx, mode):
    return load_library().dec_set_exec_mode(ctx, mode)


def dec_position(ctx, out):
    return load_library().dec_position(ctx, out)


def dec_debug_dump(ctx, what, dst, nbytes, out_bytes):
    return load_library().dec_debug_dump(ctx, what, dst, nbytes, out_bytes)


def dec_last_error(ctx):
    return load_library().dec_last_error(ctx).decode()


def dec_attention_noalloc(q, k_cache, v_cache, n_heads, n_kv_heads, head_dim, n_pos, cache_stride, out, stream):
    """Allocation-free split-KV attention (device addresses in, status code out); see include/dec.h."""
    return load_library().dec_attention_noalloc(q, k_cache, v_cache, n_heads, n_kv_heads, head_dim, n_pos,
                                                cache_stride, out, stream)


def dec_generate_async(ctx, token_id, n_steps, stop_token):
    return load_library().dec_generate_async(ctx, token_id, n_steps, stop_token)


def dec_generate_poll(ctx, out_tokens, cap, out_count, out_done):
    return load_library().dec_generate_poll(ctx, out_tokens, cap, out_count, out_done)


def dec_generate_stop(ctx):
    return load_library().dec_generate_stop(ctx)


def dec_generate_wait(ctx, out_tokens, cap, out_count):
    return load_library().dec_generate_wait(ctx, out_tokens, cap, out_count)


def dec_generate(ctx, token_id, n_steps, stop_token, out_tokens, out_count):
    return load_library().dec_generate(ctx, token_id, n_steps, stop_token, out_tokens, out_count)


# ---- convenience
def config_from_workload(w: dict, exec_mode=DEC_PERSISTENT, device=0, timeout_us=0, flags=0, n_ctas=0):
    c = dec_config()
    c.arch = DEC_ARCH_DENSE if w["arch"] == "dense" else DEC_ARCH_MLA_MOE
    for k in ("n_layers", "d_model", "vocab", "max_seq", "n_heads", "n_kv_heads", "head_dim", "ffn_hidden",
              "q_lora", "kv_lora", "qk_nope", "qk_rope", "v_head", "n_dense_layers", "n_experts", "top_k",
              "n_shared", "expert_hidden"):
        setattr(c, k, int(w.get(k, 0) or 0))
    c.rope_theta = float(w["rope_theta"])
    c.norm_eps = float(w["norm_eps"])
    c.weight_dtype = {"f32": DEC_F32, "bf16": DEC_BF16, "fp8": DEC_FP8_E4M3_B128}[w["weight_dtype"]]
    c.exec_mode = exec_mode
    c.device = device
    c.wait_timeout_us = timeout_us
    c.flags = flags
    c.n_ctas = n_ctas
    return c


class Decoder:
    """Owns one dec_ctx."""

    def __init__(self, cfg: dec_config):
        self.lib = load_library()
        rc, ctx = dec_create(cfg)
        self.ctx = ctx
        if rc != DEC_OK:
            msg = self.lib.dec_last_error(ctx).decode() if ctx else "dec_create failed"
            if ctx:
                self.lib.dec_destroy(ctx)
            self.ctx = None
            raise DecError(rc, msg)
        self.cfg = cfg

    def close(self):
        if self.ctx:
            self.lib.dec_destroy(self.ctx)
            self.ctx = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def load(self, kind, layer, data_ptr, nbytes, scales_ptr=None, expert=-1):
        t = dec_tensor(DEC_W[kind] if isinstance(kind, str) else kind, layer, expert, data_ptr, scales_ptr, nbytes)
        _chk(self.ctx, dec_load_weights(self.ctx, [t]))

    def set_kv_cache(self, k_ptr, v_ptr, n_tokens):
        _chk(self.ctx, dec_set_kv_cache(self.ctx, k_ptr, v_ptr, n_tokens))

    def step(self, token_id: int, logits_ptr=None) -> int:
        nxt = ctypes.c_int32(-1)
        _chk(self.ctx, dec_step(self.ctx, token_id, logits_ptr, ctypes.byref(nxt)))
        return nxt.value

    def step_async(self, token_id: int = -1):
        _chk(self.ctx, dec_step_async(self.ctx, token_id))

    def sync(self, logits_ptr=None) -> int:
        nxt = ctypes.c_int32(-1)
        _chk(self.ctx, dec_sync(self.ctx, logits_ptr, ctypes.byref(nxt)))
        return nxt.value

    def reset(self):
        _chk(self.ctx, dec_reset(self.ctx))

    def generate(self, token_id: int, n_steps: int, stop_token: int = -1):
        """Tokens of a whole generation (one kernel launch in DEC_PERSISTENT mode)."""
        out = (ctypes.c_int32 * max(1, n_steps))()
        n = ctypes.c_int32(0)
        _chk(self.ctx, dec_generate(self.ctx, token_id, n_steps, stop_token, out, ctypes.byref(n)))
        return list(out[:n.value])

    def generate_async(self, token_id: int, n_steps: int, stop_token: int = -1):
        _chk(self.ctx, dec_generate_async(self.ctx, token_id, n_steps, stop_token))

    def generate_poll(self, cap: int = 0):
        """(tokens so far, done) of the running generation, without waiting."""
        out = (ctypes.c_int32 * max(1, cap))()
        n, done = ctypes.c_int32(0), ctypes.c_int32(0)
        _chk(self.ctx, dec_generate_poll(self.ctx, out, cap, ctypes.byref(n), ctypes.byref(done)))
        return list(out[:min(n.value, cap)]), bool(done.value)

    def generate_stop(self):
        _chk(self.ctx, dec_generate_stop(self.ctx))

    def generate_wait(self, cap: int):
        out = (ctypes.c_int32 * max(1, cap))()
        n = ctypes.c_int32(0)
        _chk(self.ctx, dec_generate_wait(self.ctx, out, cap, ctypes.byref(n)))
        return list(out[:min(n.value, cap)])

    def set_exec_mode(self, mode):
        _chk(self.ctx, dec_set_exec_mode(self.ctx, mode))

    def set_stream(self, stream_ptr):
        _chk(self.ctx, dec_set_stream(self.ctx, stream_ptr))

    def position(self) -> int:
        p = ctypes.c_int32(0)
        _chk(self.ctx, dec_position(self.ctx, ctypes.byref(p)))
        return p.value

    def dump(self, what) -> bytes:
        need = ctypes.c_size_t(0)
        _chk(self.ctx, dec_debug_dump(self.ctx, what, None, 0, ctypes.byref(need)))
        buf = ctypes.create_string_buffer(max(1, need.value))
        _chk(self.ctx, dec_debug_dump(self.ctx, what, buf, need.value, None))
        return buf.raw[:need.value]

    def plan_text(self) -> str:
        return self.dump(DEC_DUMP_PLAN).rstrip(b"\0").decode()
