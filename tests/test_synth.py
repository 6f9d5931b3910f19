"""The seeded input generator: bfloat16 rounding and determinism."""
import numpy as np
import torch

from softmax_attention_ar_b200 import synth


def test_bf16_rounding_matches_torch():
    x = np.random.default_rng(0).standard_normal(100_000).astype(np.float32) * 10
    x[:4] = [1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -0.0, 65504.0]  # ties to even, signed zero
    ours = synth.bf16_bits(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(ours, ref)
    np.testing.assert_array_equal(synth.bf16_to_f64(ours), torch.from_numpy(x).to(torch.bfloat16).double().numpy())


def test_streams_are_seeded_and_distinct():
    a = synth.qkv(0, 1, 3, 2, 1, 16, 2, 8)
    b = synth.qkv(0, 1, 3, 2, 1, 16, 2, 8)
    c = synth.qkv(0, 1, 3, 1, 1, 16, 2, 8)
    for x, y in zip(a, b):
        np.testing.assert_array_equal(x, y)
    assert not np.array_equal(a[0], c[0])
    assert not np.array_equal(a[0], a[1])


def test_distributions():
    alpha, beta = synth.gates(0, 1, 0, 1, 12, 1560)
    assert alpha.dtype == np.float32 and alpha.shape == (1, 12, 1560)
    assert 0.85 < alpha.mean() < 0.90 and np.all((alpha > 0) & (alpha < 1))
    assert 0.45 < beta.mean() < 0.55
    Wq, _, _ = synth.feature_maps(0, 1, 12, 128)
    w = synth.bf16_to_f64(Wq)
    assert abs(w.std() * np.sqrt(128) - 1) < 0.02
