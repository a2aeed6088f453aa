"""Generation: a whole decode lifetime in one kernel launch (dec_generate*).

The pages' engine is launched once by the host and keeps the decode on the GPU
(InferenceX article, "what TileRT is").  dec_generate runs N steps that way in
DEC_PERSISTENT mode: each step's greedy token is fed back on the device and written
to a host-mapped ring.  These tests check that it computes exactly what N chained
single steps compute (same tokens, same final logits, same cache), in all three
execution modes; that a stop token and a host stop request end it early; that the
host can read tokens while it runs; and that a device wait that runs out ends the
launch with DEC_ERR_TIMEOUT (no GPU fault: a test-only flag withholds one task's
publication, every wait is bounded).
"""
import numpy as np
import pytest
import torch

from oracle import model as om
from synth import device as sdev
from synth import workloads

pytestmark = pytest.mark.gpu

CASES = ["small_dense_bf16", "small_mla_moe_fp8", "tiny_dense_f32"]


@pytest.fixture(scope="module")
def pkg():
    import persistent_sm_decode_02_b200 as p
    assert torch.cuda.is_available()
    return p


def _setup(pkg, name, n, **kw):
    w = workloads.get(name, n_decode=n + 2)
    oracle_dec, first, _ = om.build_context(w)
    cache = oracle_dec.export_cache()
    d = pkg.Decoder(pkg.config_from_workload(w, **kw))
    sdev.load_weights(d, w)
    return w, d, cache, first


def _install(d, w, cache):
    k, v = sdev.host_cache_arrays(w, cache)
    d.set_kv_cache(k.ctypes.data, v.ctypes.data, w["ctx"])


@pytest.mark.parametrize("name", CASES)
def test_generate_matches_chained_steps(pkg, name):
    n = 12
    w, d, cache, first = _setup(pkg, name, n)
    try:
        # reference: n chained single steps, each fed the previous greedy token on the device
        _install(d, w, cache)
        ref = [d.step(first)]
        for _ in range(n - 1):
            d.step_async(-1)
            ref.append(d.sync())
        ref_logits = np.empty(w["vocab"], np.float32)
        d.sync(ref_logits.ctypes.data)
        ref_kv = d.dump(pkg.dec.DEC_DUMP_KV)
        for mode in (pkg.dec.DEC_PERSISTENT, pkg.dec.DEC_PER_OP, pkg.dec.DEC_PER_OP_GRAPH):
            d.set_exec_mode(mode)
            _install(d, w, cache)
            toks = d.generate(first, n)
            assert toks == ref, f"mode {mode}: {toks} vs {ref}"
            assert d.position() == w["ctx"] + n
            logits = np.empty(w["vocab"], np.float32)
            assert d.sync(logits.ctypes.data) == ref[-1]
            assert np.array_equal(logits, ref_logits), f"mode {mode}: final logits differ"
            assert d.dump(pkg.dec.DEC_DUMP_KV) == ref_kv, f"mode {mode}: cache differs"
            # the generation can continue with single steps
            d.step(-1)
    finally:
        d.close()


def test_generate_stops_at_stop_token_and_on_request(pkg):
    n = 12
    w, d, cache, first = _setup(pkg, "small_dense_bf16", n)
    try:
        _install(d, w, cache)
        full = d.generate(first, n)
        stop = full[4]
        k = full.index(stop) + 1  # ends after the first step that yields the stop token
        _install(d, w, cache)
        toks = d.generate(first, n, stop_token=stop)
        assert toks == full[:k]
        assert d.position() == w["ctx"] + k
        # a host request: the launch ends after the step in progress, with the tokens so far
        _install(d, w, cache)
        d.generate_async(first, n)
        d.generate_stop()
        toks = d.generate_wait(n)
        assert 1 <= len(toks) <= n and toks == full[:len(toks)]
        assert d.position() == w["ctx"] + len(toks)
        # while a generation runs, calls that would queue work are refused; polling works
        _install(d, w, cache)
        d.generate_async(first, n)
        with pytest.raises(pkg.DecError) as e:
            d.step(1)
        assert e.value.code == pkg.dec.DEC_ERR_STATE
        seen, _ = d.generate_poll(n)
        assert seen == full[:len(seen)]
        assert d.generate_wait(n) == full
    finally:
        d.close()


def test_generate_capacity_and_state_errors(pkg):
    w, d, cache, first = _setup(pkg, "small_dense_bf16", 4)
    try:
        with pytest.raises(pkg.DecError) as e:
            d.generate(first, 2)  # no context
        assert e.value.code == pkg.dec.DEC_ERR_STATE
        _install(d, w, cache)
        with pytest.raises(pkg.DecError) as e:
            d.generate(first, w["n_decode"] + 1)  # beyond max_seq
        assert e.value.code == pkg.dec.DEC_ERR_CAPACITY
        with pytest.raises(pkg.DecError) as e:
            d.generate_wait(4)  # nothing running
        assert e.value.code == pkg.dec.DEC_ERR_STATE
    finally:
        d.close()


def test_generate_device_wait_timeout(pkg):
    """A task that is never published: the single launch's bounded waits run out, the status word
    records it and dec_generate_wait returns DEC_ERR_TIMEOUT; the GPU stays usable."""
    w, d, cache, first = _setup(pkg, "small_dense_bf16", 6, timeout_us=200_000,
                                flags=pkg.dec.DEC_FLAG_TEST_STALL)
    try:
        _install(d, w, cache)
        with pytest.raises(pkg.DecError) as e:
            d.generate(first, 6)
        assert e.value.code == pkg.dec.DEC_ERR_TIMEOUT
        d.reset()
    finally:
        d.close()
    w, d, cache, first = _setup(pkg, "small_dense_bf16", 6)
    try:
        _install(d, w, cache)
        assert len(d.generate(first, 3)) == 3
    finally:
        d.close()
