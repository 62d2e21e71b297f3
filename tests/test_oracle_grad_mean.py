"""Pins of the oracle's data-parallel gradient mean (grad_mean_bf16): the
mean of the ranks' BF16 gradients, binary32 sum in rank order, binary32
division, BF16 rounding (COAT summary, section "结果和边界": multi-GPU
training with every rank computing a full BF16 gradient)."""
import math
from fractions import Fraction

import numpy as np
import pytest

import oracle as orc


def _bf16(rng, n, scale):
    x = (rng.standard_normal(n) * scale).astype(np.float32)
    return orc.to_bf16_array(x)


def test_one_rank_is_the_gradient_itself():
    g = _bf16(np.random.default_rng(1), 1000, 1e-3)
    assert np.array_equal(orc.grad_mean_bf16([g]), g)


@pytest.mark.parametrize("world", [2, 3, 5, 7, 8])
def test_equal_gradients_average_to_themselves(world):
    """w copies of g sum to w g exactly (8 significant bits times w <= 8) and
    w g / w = g exactly."""
    g = _bf16(np.random.default_rng(world), 4096, 3e-2)
    assert np.array_equal(orc.grad_mean_bf16([g] * world), g)


def _ulp_bf16(x: float) -> float:
    """Spacing of BF16 values (8 significant bits) at x; subnormal spacing
    2^-133 below 2^-126."""
    _, e = math.frexp(abs(x))
    return 2.0 ** max(e - 8, -133)


@pytest.mark.parametrize("world", [2, 3, 4, 6, 8])
def test_within_half_a_bf16_step_of_the_exact_mean(world):
    """Against the exact rational mean: the result is the BF16 rounding of a
    value within the binary32 roundings (world - 1 sums and a division,
    each at most 2^-24 relative of its own result, bounded here by 2^-20 of
    the mean's magnitude plus the sum of |g| / world) of the exact mean."""
    rng = np.random.default_rng(10 + world)
    grads = [_bf16(rng, 400, s) for s in np.geomspace(1e-4, 1e-1, world)]
    got = orc.bf16_bits_to_f64(orc.grad_mean_bf16(grads))
    vals = [orc.bf16_bits_to_f64(g) for g in grads]
    for i in range(400):
        exact = sum(Fraction(float(v[i])) for v in vals) / world
        absum = sum(abs(float(v[i])) for v in vals) / world
        slack = 2.0 ** -20 * (abs(float(exact)) + absum)
        assert abs(Fraction(float(got[i])) - exact) <= Fraction(_ulp_bf16(float(got[i]))) / 2 \
            + Fraction(slack), i
