"""Host side of the input generator: determinism, distribution, bf16 rounding."""

import numpy as np
import torch

import synth


def test_deterministic_and_counter_based():
    a = synth.normal_values(7, 3, 1000, 0.5, "f32")
    b = synth.normal_values(7, 3, 1000, 0.5, "f32")
    np.testing.assert_array_equal(a, b)
    # element i does not depend on where the range starts or on chunking
    c = synth.normal_values(7, 3, 600, 0.5, "f32", start=400, chunk=77)
    np.testing.assert_array_equal(a[400:], c)
    # other seed / tensor id give other values
    assert not np.array_equal(a, synth.normal_values(8, 3, 1000, 0.5, "f32"))
    assert not np.array_equal(a, synth.normal_values(7, 4, 1000, 0.5, "f32"))


def test_distribution_moments():
    z = synth.normal_u16bits_f32(0, 1, 0, 1 << 20).astype(np.float64)
    assert abs(z.mean()) < 5e-3
    assert abs(z.var() - 1.0) < 5e-3
    assert np.abs(z).max() <= 6.0
    # Irwin-Hall(12) kurtosis is 3 - 1.2/12 = 2.9
    assert abs(np.mean(z ** 4) / z.var() ** 2 - 2.9) < 0.03


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(0)
    v = (rng.standard_normal(100000) * np.exp(rng.uniform(-20, 20, 100000))).astype(np.float32)
    ref = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(synth.bf16_round_bits(v), ref)
    # ties go to even
    ties = np.array([1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8], dtype=np.float32)
    assert synth.bf16_bits_to_f32(synth.bf16_round_bits(ties)).tolist() == [1.0, 1.0 + 2 ** -6]


def test_shapes_and_scales():
    s = synth.MoEShape("t", 8, 32, 48, 4, 2, "bf16")
    t = synth.host_inputs(s, seed=1)
    assert t["x"].shape == (8, 32) and t["Wg"].shape == (4, 32)
    assert t["W1"].shape == (4, 48, 32) and t["W3"].shape == (4, 48, 32) and t["W2"].shape == (4, 32, 48)
    w2 = synth.bf16_bits_to_f64(t["W2"])
    assert abs(w2.std() * np.sqrt(48) - 1) < 0.05
    assert synth.CONFIGS["prefill"].flops == 4096 * (2 * 4096 * 8 + 2 * 6 * 4096 * 14336)
