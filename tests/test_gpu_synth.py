"""The GPU side of the seeded generator reproduces the CPU side byte for byte."""
import numpy as np
import pytest
import torch

import synth

pytestmark = pytest.mark.gpu


def test_gpu_generator_matches_cpu():
    seed = 4242
    a = torch.empty(10007, dtype=torch.float32, device="cuda")
    synth.gpu_normal_f32(a, seed, 17, 0.1, 1.0, start=5)
    assert np.array_equal(a.cpu().numpy(), synth.normal_f32(seed, 17, 10007, 0.1, 1.0, start=5))
    b = torch.empty(9999, dtype=torch.int16, device="cuda")
    synth.gpu_normal_bf16(b, seed, 18, 0.02)
    assert np.array_equal(b.cpu().numpy().view(np.uint16), synth.normal_bf16_bits(seed, 18, 9999, 0.02))
    rows, cols = 300, 272
    q = torch.empty(rows * cols, dtype=torch.uint8, device="cuda")
    s = torch.empty(3 * 3, dtype=torch.float32, device="cuda")
    synth.gpu_fp8_b128(q, s, seed, 19, rows, cols, 0.02)
    qc, sc = synth.fp8_b128(seed, 19, rows, cols, 0.02)
    assert np.array_equal(q.cpu().numpy().reshape(rows, cols), qc)
    assert np.array_equal(s.cpu().numpy().reshape(3, 3), sc)
    t = torch.empty(1000, dtype=torch.int32, device="cuda")
    synth.gpu_tokens(t, seed, synth.TOKENS_CONTEXT, 32000)
    assert np.array_equal(t.cpu().numpy(), synth.tokens(seed, synth.TOKENS_CONTEXT, 1000, 32000))
