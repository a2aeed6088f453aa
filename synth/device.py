"""Fill a decoder with a synthetic workload on the device.

Weights are drawn on the GPU by the seeded generator (synth_cuda.cu) into
temporary torch tensors and handed to the decoder through the C ABI
(dec_load_weights copies them into its own tile-ordered store), one tensor at
a time, so device memory holds the model once plus one tensor in flight.
Prefilled caches come from the oracle (small workloads, host arrays) or are
drawn on the device (large workloads).
"""
from __future__ import annotations

import numpy as np
import torch

from . import gpu_fp8_b128, gpu_normal_bf16, gpu_normal_f32
from . import workloads


def _dtype_bytes(dt):
    return {"f32": 4, "bf16": 2, "fp8": 1}[dt]


def gen_tensor(w, spec, device="cuda"):
    """(data, scales) torch tensors on the device for one weight spec."""
    seed = w["seed"]
    shape = spec["shape"]
    n = int(np.prod(shape))
    if spec["dtype"] == "f32":
        t = torch.empty(n, dtype=torch.float32, device=device)
        gpu_normal_f32(t, seed, spec["tid"], spec["std"], spec["offset"])
        return t, None
    if spec["dtype"] == "bf16":
        t = torch.empty(n, dtype=torch.int16, device=device)
        gpu_normal_bf16(t, seed, spec["tid"], spec["std"], spec["offset"])
        return t, None
    rows, cols = shape
    q = torch.empty(n, dtype=torch.uint8, device=device)
    s = torch.empty(((rows + 127) // 128) * ((cols + 127) // 128), dtype=torch.float32, device=device)
    gpu_fp8_b128(q, s, seed, spec["tid"], rows, cols, spec["std"])
    return q, s


def load_weights(dec, w, device="cuda"):
    """Generate and load every weight tensor of workload w into Decoder `dec`."""
    for spec in workloads.weight_specs(w):
        data, sc = gen_tensor(w, spec, device)
        nbytes = data.numel() * data.element_size()
        dec.load(spec["name"], spec["layer"], data.data_ptr(), nbytes,
                 sc.data_ptr() if sc is not None else None, spec["expert"])
        del data, sc
    torch.cuda.synchronize()


def synthetic_cache_device(w, device="cuda"):
    """Prefilled cache drawn on the device, in the layout dec_set_kv_cache takes:
    dense (k, v) [L][hkv][ctx][hd]; MLA (latent [L][ctx][kv_lora], pe [L][ctx][rope]); bf16 bits."""
    L = w["n_layers"]
    specs = workloads.cache_specs(w)
    parts = {}
    for s in specs:
        n = int(np.prod(s["shape"]))
        buf = parts.setdefault(s["name"], torch.empty((L, n), dtype=torch.int16, device=device))
        gpu_normal_bf16(buf[s["layer"]], w["seed"], s["tid"], s["std"])
    if w["arch"] == "dense":
        return parts["k_cache"], parts["v_cache"]
    return parts["latent_cache"], parts["pe_cache"]


def host_cache_arrays(w, parts: dict):
    """Oracle cache (float64 values already on the cache grid) -> contiguous host arrays in the cache dtype."""
    keys = ("k", "v") if w["arch"] == "dense" else ("latent", "pe")
    out = []
    for k in keys:
        a = np.ascontiguousarray(parts[k])
        if workloads.act_dtype(w) == "f32":
            out.append(a.astype(np.float32))
        else:
            t = torch.from_numpy(a.astype(np.float32)).to(torch.bfloat16)
            out.append(t.view(torch.int16).numpy().copy())
    return out


def context_ids(w, n=None):
    """The workload's context: n (default ctx) seeded uniform-random token ids."""
    from . import TOKENS_CONTEXT, tokens

    return tokens(w["seed"], TOKENS_CONTEXT, w["ctx"] if n is None else n, w["vocab"])


def prefill_by_decode(d, w, n=None, device="cuda"):
    """Fill decoder d's cache with a real context: from an empty cache, the GPU decodes the
    workload's first n context ids (default ctx), one step per id, each fed from the host.

    Returns the cache as device tensors in the layout dec_set_kv_cache takes (dense (k, v),
    MLA (latent, pe); the cache dtype's bits), so that it can be installed again later.
    The decoder is left at position n."""
    ids = context_ids(w, n)
    d.set_kv_cache(0, 0, 0)
    for t in ids:
        d.step_async(int(t))
    d.sync()
    raw = np.frombuffer(d.dump(_dump_kv()), np.uint8)
    if w["arch"] == "dense":
        first = raw.size // 2  # K then V, equal sizes
    else:  # latent [L][n][kv_lora] then pe [L][n][rope]
        first = raw.size * w["kv_lora"] // (w["kv_lora"] + w["qk_rope"])
    el = torch.float32 if workloads.act_dtype(w) == "f32" else torch.int16
    a = torch.from_numpy(raw[:first].copy()).view(el).to(device)
    b = torch.from_numpy(raw[first:].copy()).view(el).to(device)
    return a, b


def _dump_kv():
    from persistent_sm_decode_02_b200 import dec

    return dec.DEC_DUMP_KV
