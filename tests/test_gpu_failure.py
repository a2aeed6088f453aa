"""Failure detection and host-side error paths of the decoder (GPU).

The device path is tested without faulting the GPU: DEC_FLAG_TEST_STALL makes
the signaller never publish one task, so the tasks that depend on it wait on a
counter that nothing will raise; every wait is bounded, the kernel records the
timeout in its status word and all CTAs stop, and dec_step returns
DEC_ERR_TIMEOUT.  The GPU stays usable: a fresh decoder runs a step afterwards.
"""
import time

import numpy as np
import pytest
import torch

from synth import device as sdev
from synth import workloads

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def pkg():
    import persistent_sm_decode_02_b200 as p
    assert torch.cuda.is_available()
    return p


def _decoder(pkg, w, **kw):
    d = pkg.Decoder(pkg.config_from_workload(w, **kw))
    sdev.load_weights(d, w)
    return d


def test_device_wait_times_out_and_gpu_stays_usable(pkg):
    w = workloads.get("small_dense_bf16")
    d = _decoder(pkg, w, timeout_us=200_000, flags=pkg.dec.DEC_FLAG_TEST_STALL)
    try:
        k, v = sdev.synthetic_cache_device(w)
        d.set_kv_cache(k.data_ptr(), v.data_ptr(), w["ctx"])
        t0 = time.time()
        with pytest.raises(pkg.DecError) as e:
            d.step(3)
        assert e.value.code == pkg.dec.DEC_ERR_TIMEOUT
        assert time.time() - t0 < 10.0
        # the context is poisoned until reset
        with pytest.raises(pkg.DecError) as e:
            d.step(3)
        assert e.value.code == pkg.dec.DEC_ERR_STATE
        d.reset()
        assert d.position() == 0
    finally:
        d.close()
    # a healthy decoder on the same GPU still works
    d2 = _decoder(pkg, w)
    try:
        k, v = sdev.synthetic_cache_device(w)
        d2.set_kv_cache(k.data_ptr(), v.data_ptr(), w["ctx"])
        nxt = d2.step(3)
        assert 0 <= nxt < w["vocab"]
    finally:
        d2.close()


def test_state_and_capacity_errors(pkg):
    w = workloads.get("tiny_dense_f32", ctx=4, n_decode=2)
    d = pkg.Decoder(pkg.config_from_workload(w))
    try:
        with pytest.raises(pkg.DecError) as e:
            d.step(1)  # no weights yet
        assert e.value.code == pkg.dec.DEC_ERR_STATE
        sdev.load_weights(d, w)
        with pytest.raises(pkg.DecError) as e:
            d.step(1)  # no context yet
        assert e.value.code == pkg.dec.DEC_ERR_STATE
        kv = np.zeros((w["n_layers"], w["n_kv_heads"], w["max_seq"], w["head_dim"]), np.float32)
        with pytest.raises(pkg.DecError) as e:
            d.set_kv_cache(kv.ctypes.data, kv.ctypes.data, w["max_seq"])  # no room to decode
        assert e.value.code == pkg.dec.DEC_ERR_CAPACITY
        d.set_kv_cache(kv.ctypes.data, kv.ctypes.data, w["ctx"])
        with pytest.raises(pkg.DecError) as e:
            d.step(-1)  # nothing to feed back yet
        assert e.value.code == pkg.dec.DEC_ERR_STATE
        with pytest.raises(pkg.DecError) as e:
            d.step(w["vocab"])
        assert e.value.code == pkg.dec.DEC_ERR_INVALID_ARG
        d.step(1)
        d.step(-1)
        assert d.position() == w["max_seq"]
        with pytest.raises(pkg.DecError) as e:
            d.step(1)  # cache full
        assert e.value.code == pkg.dec.DEC_ERR_CAPACITY
        # empty context: decoding starts at position 0
        d.set_kv_cache(None, None, 0)
        assert 0 <= d.step(2) < w["vocab"]
    finally:
        d.close()


def test_wrong_weight_size_is_rejected(pkg):
    w = workloads.get("tiny_dense_f32")
    d = pkg.Decoder(pkg.config_from_workload(w))
    try:
        buf = torch.zeros(1000, dtype=torch.float32, device="cuda")
        with pytest.raises(pkg.DecError) as e:
            d.load("wq", 0, buf.data_ptr(), 1000 * 4)
        assert e.value.code == pkg.dec.DEC_ERR_INVALID_ARG
        with pytest.raises(pkg.DecError) as e:
            d.load("wq", 7, buf.data_ptr(), 1000 * 4)  # layer out of range
        assert e.value.code == pkg.dec.DEC_ERR_INVALID_ARG
        with pytest.raises(pkg.DecError) as e:
            d.load("router", 0, buf.data_ptr(), 1000 * 4)  # no MoE in a dense model
        assert e.value.code == pkg.dec.DEC_ERR_INVALID_ARG
    finally:
        d.close()


def test_a_stream_given_to_the_decoder_stays_the_callers(pkg):
    """dec_set_stream borrows the caller's stream: after dec_destroy the stream still works, and
    the step it ran gives the same token as a decoder on the library's own stream (bf16 model:
    the drawn cache is bf16, the layout dec_set_kv_cache takes for it)."""
    w = workloads.get("small_dense_bf16")
    k, v = sdev.synthetic_cache_device(w)
    s = torch.cuda.Stream()
    d = _decoder(pkg, w)
    try:
        d.set_stream(s.cuda_stream)
        d.set_kv_cache(k.data_ptr(), v.data_ptr(), w["ctx"])
        tok = d.step(3)
    finally:
        d.close()
    with torch.cuda.stream(s):
        y = (torch.arange(1024, device="cuda", dtype=torch.float32) * 2).sum()
    s.synchronize()
    assert float(y) == 1024.0 * 1023.0
    d2 = _decoder(pkg, w)
    try:
        d2.set_kv_cache(k.data_ptr(), v.data_ptr(), w["ctx"])
        assert d2.step(3) == tok
    finally:
        d2.close()


def test_nonfinite_lm_logits_are_reported(pkg):
    """A NaN final-norm gain (a corrupt weight, injected on the host) makes every logit NaN: the
    step returns DEC_ERR_NUMERIC instead of a greedy token, the context stays poisoned until
    dec_reset, and with the weight restored the decoder works again."""
    w = workloads.get("small_dense_bf16")
    d = _decoder(pkg, w)
    try:
        k, v = sdev.synthetic_cache_device(w)
        good, _ = sdev.gen_tensor(w, [s for s in workloads.weight_specs(w) if s["name"] == "final_norm"][0])
        bad = np.full(w["d_model"], np.nan, np.float32)
        d.load("final_norm", -1, bad.ctypes.data, bad.nbytes)
        d.set_kv_cache(k.data_ptr(), v.data_ptr(), w["ctx"])
        with pytest.raises(pkg.DecError) as e:
            d.step(3)
        assert e.value.code == pkg.dec.DEC_ERR_NUMERIC
        assert "final" in str(e.value)
        with pytest.raises(pkg.DecError) as e:
            d.step(3)
        assert e.value.code == pkg.dec.DEC_ERR_STATE
        d.load("final_norm", -1, good.data_ptr(), good.numel() * 4)
        d.set_kv_cache(k.data_ptr(), v.data_ptr(), w["ctx"])
        assert 0 <= d.step(3) < w["vocab"]
    finally:
        d.close()


def test_nonfinite_router_logits_are_reported(pkg):
    """One router row of E4M3 NaN codes (0x7F) in the first MoE layer gives that expert a NaN
    logit: the router's top-k reports it (DEC_ERR_NUMERIC, op 'router') instead of silently
    routing around it."""
    w = workloads.get("small_mla_moe_fp8")
    d = _decoder(pkg, w)
    try:
        k, v = sdev.synthetic_cache_device(w)
        layer = w["n_dense_layers"]
        spec = [s for s in workloads.weight_specs(w) if s["name"] == "router" and s["layer"] == layer][0]
        q, sc = sdev.gen_tensor(w, spec)
        q = q.view(spec["shape"]).clone()
        q[3] = 0x7F
        d.load("router", layer, q.data_ptr(), q.numel(), sc.data_ptr())
        d.set_kv_cache(k.data_ptr(), v.data_ptr(), w["ctx"])
        with pytest.raises(pkg.DecError) as e:
            d.step(3)
        assert e.value.code == pkg.dec.DEC_ERR_NUMERIC
        assert "router" in str(e.value)
        d.reset()
        q0, sc0 = sdev.gen_tensor(w, spec)
        d.load("router", layer, q0.data_ptr(), q0.numel(), sc0.data_ptr())
        d.set_kv_cache(k.data_ptr(), v.data_ptr(), w["ctx"])
        assert 0 <= d.step(3) < w["vocab"]
    finally:
        d.close()
