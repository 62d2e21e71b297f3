"""Pins of the oracle's LayerNorm / RMSNorm (the second producer with fused
Group Scaling maxima) against closed forms and invariants."""
import numpy as np

import oracle


def _bf16(v):
    return oracle.round_to_bf16(np.asarray(v, dtype=np.float64))


def test_hand_example_closed_forms():
    x = _bf16([[1.0, 2.0, 3.0, 4.0]])
    # mean 5/2, variance 5/4: (x_i - 5/2) / sqrt(5/4) = (2 i - 5) / sqrt(5)
    want_ln = (2.0 * np.arange(1, 5) - 5.0) / np.sqrt(5.0)
    assert np.allclose(oracle.norm_f64(x, rms=False, eps=0.0)[0], want_ln, rtol=0, atol=1e-15)
    # mean of squares 30/4: x_i / sqrt(15/2)
    want_rms = np.arange(1, 5) / np.sqrt(7.5)
    assert np.allclose(oracle.norm_f64(x, rms=True, eps=0.0)[0], want_rms, rtol=0, atol=1e-15)
    # per-column weight and bias act column by column: w = (1, 2, 3, 4),
    # b = (1/2, 0, 0, -1) give ((2 i - 5) / sqrt 5) i + b_i
    w = np.array([1.0, 2.0, 3.0, 4.0], np.float32)
    b = np.array([0.5, 0.0, 0.0, -1.0], np.float32)
    want_aff = want_ln * np.arange(1, 5) + np.array([0.5, 0.0, 0.0, -1.0])
    got_aff = oracle.norm_f64(x, rms=False, eps=0.0, weight=w, bias=b)[0]
    assert np.allclose(got_aff, want_aff, rtol=0, atol=1e-15)
    # with eps the variance term grows by exactly eps (binary32 value of eps)
    e = float(np.float32(1e-3))
    want_eps = (2.0 * np.arange(1, 5) - 5.0) / 2.0 / np.sqrt(1.25 + e)
    assert np.allclose(oracle.norm_f64(x, rms=False, eps=1e-3)[0], want_eps, rtol=0, atol=1e-15)


def test_layernorm_invariants():
    rng = np.random.default_rng(1)
    x = _bf16(rng.standard_normal((16, 256)) * 3.0 + 0.5)
    y = oracle.norm_f64(x, rms=False, eps=0.0)
    assert np.allclose(y.mean(axis=1), 0.0, atol=1e-13)
    assert np.allclose((y * y).mean(axis=1), 1.0, atol=1e-12)
    # shifting every element by 8 and scaling by 4 (both exact in BF16 for
    # these small integers) changes nothing
    xi = _bf16(rng.integers(-20, 20, (4, 64)).astype(np.float64))
    shifted = _bf16(oracle.bf16_bits_to_f64(xi) * 4.0 + 8.0)
    assert np.array_equal(oracle.norm_bf16(xi, rms=False, eps=0.0),
                          oracle.norm_bf16(shifted, rms=False, eps=0.0))
    # a constant row normalises to exactly zero
    c = _bf16(np.full((1, 32), 1.5))
    assert np.all(oracle.norm_f64(c, rms=False, eps=1e-5) == 0.0)


def test_rmsnorm_invariants_and_affine():
    rng = np.random.default_rng(2)
    x = _bf16(rng.standard_normal((8, 128)))
    y = oracle.norm_f64(x, rms=True, eps=0.0)
    assert np.allclose(np.sqrt((y * y).mean(axis=1)), 1.0, atol=1e-13)
    assert np.array_equal(oracle.norm_bf16(x, rms=True, eps=0.0),
                          oracle.norm_bf16(_bf16(oracle.bf16_bits_to_f64(x) * 0.25), rms=True,
                                           eps=0.0))
    w = np.full(128, 2.0, np.float32)
    b = np.full(128, -1.0, np.float32)
    base = oracle.norm_f64(x, rms=False, eps=1e-5)
    assert np.array_equal(oracle.norm_f64(x, rms=False, eps=1e-5, weight=w, bias=b),
                          base * 2.0 - 1.0)
