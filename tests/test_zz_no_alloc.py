"""dec_attention_noalloc: split-KV decode attention that allocates no device memory.

Some callers cannot call cudaMalloc -- code running while a CUDA graph is being
captured, runtimes whose device memory belongs to an outside allocator that
forbids allocation on the serving path, embedders that must keep a fixed
footprint -- so this entry point keeps its per-chunk partials in a fixed
array inside the library.  The test checks it against the attention the decode
step itself computes: two decode steps of a small bf16 model run through
dec_step; after each, the step's own dumps give the attention inputs (the fused
q/k/v output and the KV cache after the new row was appended) and its output
(the split-KV partials, combined here); the allocation-free call on the same
inputs must agree within the bf16 tolerance of the other GPU tests.

A second set of cases checks the call against the oracle's float64 attention
(the split-KV definition taken as one chunk, softmax(q K^T / sqrt(head_dim)) V) on
seeded random q and bf16 K/V, over shapes the decode step never produces: head_dim
128 with 8 query heads per kv head, a cache row stride larger than the positions
used, one position, thousands of positions (many shared-memory tiles per chunk, so
the online softmax rescales across tiles), and 64 chunks on a single kv head.  The
host-side refusals (unsupported shapes, misaligned pointers, partials larger than
the fixed scratch) return before anything is launched.

Kept in its own file, collected last, so a run that stops at the first failure
has run every other test before it.
"""
import numpy as np
import pytest
import torch

from oracle import model as om
from synth import device as sdev
from synth import workloads

pytestmark = pytest.mark.gpu

TOL = 5e-3  # bf16 logits tolerance used by the parity tests


def _bf16_bits(x: np.ndarray) -> np.ndarray:
    return torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16).view(torch.int16).numpy()


def _from_bf16_bits(b: np.ndarray) -> np.ndarray:
    return (b.astype(np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def test_noalloc_attention_matches_decode_step():
    import persistent_sm_decode_02_b200 as pkg

    w = workloads.get("small_dense_bf16")
    hq, hkv, hd, L = w["n_heads"], w["n_kv_heads"], w["head_dim"], w["n_layers"]
    d = pkg.Decoder(pkg.config_from_workload(w))
    try:
        sdev.load_weights(d, w)
        k, v = sdev.synthetic_cache_device(w)
        d.set_kv_cache(k.data_ptr(), v.data_ptr(), w["ctx"])
        plan = [line.split() for line in d.plan_text().splitlines()[:-1]]
        assert plan[0][1] == "qkv" and plan[1][1] == "attn"
        S = int(dict(f.split("=") for f in plan[0][2:] if "=" in f)["S"])
        nch = int(dict(f.split("=") for f in plan[1][2:] if "=" in f)["nch"])
        tok = 5
        for call in range(2):
            pos = w["ctx"] + call
            tok = d.step(tok)
            # the step's attention inputs: q of layer 0 (RoPE at pos, rounded to bf16) ...
            qkv = np.frombuffer(d.dump(pkg.dec.DEC_DUMP_OP + 0), np.float32).astype(np.float64).reshape(S, -1).sum(0)
            qr = qkv[: hq * hd].reshape(hq, hd)
            half = hd // 2
            ang = pos * w["rope_theta"] ** (-2.0 * np.arange(half) / hd)
            c, s = np.cos(ang).astype(np.float32).astype(np.float64), np.sin(ang).astype(np.float32).astype(np.float64)
            q = np.concatenate([qr[:, :half] * c - qr[:, half:] * s, qr[:, :half] * s + qr[:, half:] * c], axis=1)
            q = _from_bf16_bits(_bf16_bits(q))
            # ... and the layer-0 cache after the append (positions 0..pos)
            n = pos + 1
            raw = np.frombuffer(d.dump(pkg.dec.DEC_DUMP_KV), np.int16)
            kv = raw.reshape(2, L, hkv, n, hd)
            k0 = torch.from_numpy(kv[0, 0].copy()).cuda()
            v0 = torch.from_numpy(kv[1, 0].copy()).cuda()
            qd = torch.from_numpy(q.astype(np.float32)).cuda()
            out = torch.empty(hq * hd, dtype=torch.float32, device="cuda")
            torch.cuda.synchronize()
            rc = pkg.dec.dec_attention_noalloc(qd.data_ptr(), k0.data_ptr(), v0.data_ptr(), hq, hkv, hd, n, n,
                                               out.data_ptr(), torch.cuda.current_stream().cuda_stream)
            assert rc == pkg.dec.DEC_OK
            torch.cuda.synchronize()
            # the step's own attention output: its split-KV partials, combined
            part = np.frombuffer(d.dump(pkg.dec.DEC_DUMP_OP + 1), np.float32).astype(np.float64)
            m = part[: hq * nch].reshape(hq, nch)
            l_ = part[hq * nch: 2 * hq * nch].reshape(hq, nch)
            o = part[2 * hq * nch:].reshape(hq, nch, hd)
            M = np.max(np.where(l_ > 0, m, -np.inf), axis=1, keepdims=True)
            wgt = np.where(l_ > 0, np.exp(m - M), 0.0)
            ref = (wgt[:, :, None] * o).sum(1) / (wgt * l_).sum(1, keepdims=True)
            got = out.cpu().numpy().astype(np.float64).reshape(hq, hd)
            err = np.max(np.abs(got - ref)) / np.max(np.abs(ref))
            assert err <= TOL, f"call {call}: max error {err:.3e}"
    finally:
        d.close()


ORACLE_TOL = 1e-4  # fp32 GPU arithmetic against float64 on the same bf16 / fp32 inputs

# (n_heads, n_kv_heads, head_dim, n_pos, cache_stride)
SHAPES = [(6, 2, 64, 79, 79), (16, 2, 128, 3000, 4096), (8, 8, 128, 1, 16), (32, 8, 64, 1025, 2048),
          (8, 1, 64, 5000, 5000)]


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "h%d_kv%d_d%d_n%d_s%d" % s)
def test_noalloc_attention_matches_oracle(shape):
    import persistent_sm_decode_02_b200 as pkg

    hq, hkv, hd, n, stride = shape
    rng = np.random.default_rng(1000 + hq * 7 + hd + n)
    kv = torch.from_numpy(rng.standard_normal((2, hkv, stride, hd)).astype(np.float32)).to(torch.bfloat16)
    kv_d = kv.view(torch.int16).cuda()
    kv64 = kv.float().numpy().astype(np.float64)
    out = torch.empty(hq * hd, dtype=torch.float32, device="cuda")
    gs = hq // hkv
    for call in range(2):  # two calls in a row share the fixed scratch
        q = rng.standard_normal((hq, hd)).astype(np.float32)
        qd = torch.from_numpy(q).cuda()
        torch.cuda.synchronize()
        rc = pkg.dec.dec_attention_noalloc(qd.data_ptr(), kv_d[0].data_ptr(), kv_d[1].data_ptr(), hq, hkv, hd, n,
                                           stride, out.data_ptr(), torch.cuda.current_stream().cuda_stream)
        assert rc == pkg.dec.DEC_OK
        torch.cuda.synchronize()
        got = out.cpu().numpy().astype(np.float64).reshape(hq, hd)
        ref = np.stack([om.attention_split_lse(q[h].astype(np.float64), kv64[0, h // gs, :n], kv64[1, h // gs, :n],
                                               [(0, n)]) for h in range(hq)])
        err = np.max(np.abs(got - ref)) / np.max(np.abs(ref))
        assert err <= ORACLE_TOL, f"call {call}: max error {err:.3e}"
        if n == 1:  # one position: the output is that position's V row
            assert np.max(np.abs(got - kv64[1, np.arange(hq) // gs, 0])) <= ORACLE_TOL * np.max(np.abs(ref))


def test_noalloc_attention_rejects_bad_shapes():
    import persistent_sm_decode_02_b200 as pkg

    x = torch.zeros(1024, device="cuda")
    p = x.data_ptr()
    # head_dim 96 is not supported; n_heads not a multiple of n_kv_heads; positions beyond the cache
    assert pkg.dec.dec_attention_noalloc(p, p, p, 4, 4, 96, 4, 4, p, None) == pkg.dec.DEC_ERR_INVALID_ARG
    assert pkg.dec.dec_attention_noalloc(p, p, p, 6, 4, 64, 4, 4, p, None) == pkg.dec.DEC_ERR_INVALID_ARG
    assert pkg.dec.dec_attention_noalloc(p, p, p, 4, 4, 64, 8, 4, p, None) == pkg.dec.DEC_ERR_INVALID_ARG
    # K / V not 16-byte aligned, q / out not 4-byte aligned (refused before any launch)
    assert pkg.dec.dec_attention_noalloc(p, p + 2, p, 4, 4, 64, 4, 4, p, None) == pkg.dec.DEC_ERR_INVALID_ARG
    assert pkg.dec.dec_attention_noalloc(p, p, p + 8, 4, 4, 64, 4, 4, p, None) == pkg.dec.DEC_ERR_INVALID_ARG
    assert pkg.dec.dec_attention_noalloc(p + 2, p, p, 4, 4, 64, 4, 4, p, None) == pkg.dec.DEC_ERR_INVALID_ARG
    assert pkg.dec.dec_attention_noalloc(p, p, p, 4, 4, 64, 4, 4, p + 1, None) == pkg.dec.DEC_ERR_INVALID_ARG
    # one chunk per head already needs 4096 * 130 floats, more than the fixed 2 MiB scratch
    assert pkg.dec.dec_attention_noalloc(p, p, p, 4096, 512, 128, 4, 4, p, None) == pkg.dec.DEC_ERR_CAPACITY
