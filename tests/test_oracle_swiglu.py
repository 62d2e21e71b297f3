"""Pins of the oracle's SwiGLU producer and its BF16 rounding (no GPU)."""
import numpy as np
import torch

import oracle


def test_round_to_bf16_matches_torch_on_binary32_inputs():
    rng = np.random.default_rng(11)
    bits = rng.integers(0, 2**32, 200_000, dtype=np.uint64).astype(np.uint32)
    x = bits.view(np.float32)
    x = x[np.isfinite(x)]
    want = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = oracle.round_to_bf16(x.astype(np.float64))
    assert np.array_equal(got, want)


def test_round_to_bf16_ties_and_limits():
    one = 1.0
    assert oracle.round_to_bf16(one + 2.0**-8) == 0x3F80          # tie -> even (1.0)
    assert oracle.round_to_bf16(one + 3 * 2.0**-8) == 0x3F82      # tie -> even (1 + 2^-6)
    assert oracle.round_to_bf16(one + 2.0**-8 + 2.0**-30) == 0x3F81
    assert oracle.round_to_bf16(2.0**-133) == 0x0001              # smallest subnormal
    assert oracle.round_to_bf16(2.0**-134) == 0x0000              # tie -> even (zero)
    assert oracle.round_to_bf16(oracle.BF16_MAX) == 0x7F7F
    assert oracle.round_to_bf16(2.0**128) == 0x7F80               # overflow -> inf
    assert oracle.round_to_bf16(-0.0) == 0x8000


def test_silu_identity_and_library_value():
    rng = np.random.default_rng(12)
    g = oracle.round_to_bf16(rng.normal(0, 3, 50_000))
    one = np.full(g.size, 0x3F80, dtype=np.uint16)                 # up = 1
    h_pos = oracle.bf16_bits_to_f64(oracle.swiglu_bf16(g, one))
    # against torch's binary64 silu, rounded by the same routine
    gt = torch.from_numpy(oracle.bf16_bits_to_f64(g))
    want = oracle.round_to_bf16(torch.nn.functional.silu(gt).numpy())
    assert np.array_equal(oracle.swiglu_bf16(g, one), want)
    # silu(g) - silu(-g) = g, checked before rounding on exact inputs
    x = oracle.bf16_bits_to_f64(g)
    s = lambda v: v / (1.0 + np.exp(-v))  # noqa: E731
    assert np.allclose(s(x) - s(-x), x, rtol=1e-14, atol=1e-300)
    # silu(0) = 0, silu(large) = large, silu(very negative) = -0
    z = oracle.round_to_bf16(np.array([0.0, 200.0, -2000.0]))
    h = oracle.bf16_bits_to_f64(oracle.swiglu_bf16(z, np.full(3, 0x3F80, np.uint16)))
    assert h[0] == 0.0 and h[1] == 200.0 and h[2] == 0.0
    assert np.all(np.isfinite(h_pos))


def test_group_amax_of():
    x = oracle.round_to_bf16(np.array([1.0, -3.0, 2.0, 0.5, -0.25]))
    assert np.array_equal(oracle.group_amax_of(x, 2), np.array([3.0, 2.0, 0.25], np.float32))
