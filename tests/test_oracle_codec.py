"""Pins of the oracle's number-format layer (CPU only).

The oracle's FP8 / BF16 codecs are checked against what the pages print
(golden files) and against torch's independent float8/bfloat16 casts.
"""
import math

import numpy as np
import pytest
import torch

from conftest import read_golden

E4M3, E5M2 = 0, 1
TORCH_DT = {E4M3: torch.float8_e4m3fn, E5M2: torch.float8_e5m2}
FMT_NAME = {"e4m3": E4M3, "e5m2": E5M2}


def test_e2m2_subnormal_list_from_page(orc):
    """FP8/FP4 formats blog, section "FP格式": E2M2 with bias 2."""
    for e, m, num, den in read_golden("e2m2_bias2_values.txt"):
        assert orc.exmy_value(2, 2, 2, int(e), int(m)) == int(num) / int(den)


def test_e2m2_products_without_bias(orc):
    """Same page: the 16 E2 x M2 products; bias 0 and no subnormal row."""
    for e, m, val in read_golden("e2m2_no_subnormal_values.txt"):
        e, m = int(e), int(m)
        if e == 0:
            continue  # the subnormal rule rewrites this row (checked above)
        assert orc.exmy_value(2, 2, 0, e, m) == float(val)


def test_fp8_limits_from_pages(orc):
    rows = {(k, f): float(v) for k, f, v in read_golden("fp8_format_limits.txt")}
    for f in ("e4m3", "e5m2"):
        fmt = FMT_NAME[f]
        assert orc.fp8_max(fmt) == rows[("max", f)]
        assert orc.fp8_min_subnormal(fmt) == rows[("min_subnormal", f)]
        # spacing at 1: the code after 1.0
        one = orc.fp8_encode(1.0, fmt)
        assert orc.fp8_decode(one, fmt) == 1.0
        assert orc.fp8_decode(one + 1, fmt) - 1.0 == rows[("spacing_at_one", f)]
    assert orc.fp8_max(E4M3) / 2.0 ** 8 == rows[("max_normal_significand", "e4m3")]
    assert orc.fp8_decode(0x07, E4M3) / 2.0 ** -6 == rows[("max_subnormal_significand", "e4m3")]
    assert orc.fp8_range(E4M3) == rows[("range", "e4m3")]


@pytest.mark.parametrize("fmt", [E4M3, E5M2])
def test_decode_all_codes_match_torch(orc, fmt):
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(TORCH_DT[fmt]).to(torch.float64).numpy()
    for c in range(256):
        got = orc.fp8_decode(c, fmt)
        if math.isnan(ref[c]):
            assert math.isnan(got), c
        else:
            assert got == ref[c], (c, got, ref[c])


@pytest.mark.parametrize("fmt", [E4M3, E5M2])
def test_encode_roundtrip_all_finite_codes(orc, fmt):
    top = 0x7E if fmt == E4M3 else 0x7B
    for c in list(range(0, top + 1)) + list(range(0x80, 0x80 + top + 1)):
        assert orc.fp8_encode(orc.fp8_decode(c, fmt), fmt) == c


def _boundary_floats(orc, fmt):
    """Every code's value, every midpoint between neighbours, and a few
    binary32 neighbours of each (the values where rounding decides)."""
    top = 0x7E if fmt == E4M3 else 0x7B
    vals = np.array([orc.fp8_decode(c, fmt) for c in range(top + 1)], dtype=np.float64)
    mids = (vals[:-1] + vals[1:]) / 2.0
    pts = np.concatenate([vals, mids]).astype(np.float32)
    out = [pts]
    for k in (1, 2, 3):
        up = pts.copy()
        dn = pts.copy()
        for _ in range(k):
            up = np.nextafter(up, np.float32(np.inf))
            dn = np.nextafter(dn, np.float32(-np.inf))
        out += [up, dn]
    allp = np.concatenate(out)
    allp = allp[allp >= 0]
    return np.concatenate([allp, -allp]).astype(np.float32)


@pytest.mark.parametrize("fmt", [E4M3, E5M2])
def test_encode_matches_torch_cast_in_range(orc, fmt):
    """Below the saturation point the oracle's RNE encoder must equal
    torch's float32 -> float8 cast (nearest-even, no saturation there)."""
    rng = np.random.default_rng(7)
    sat = 464.0 if fmt == E4M3 else 61440.0   # half-way to the next step above max
    # random bit patterns over the whole float range, plus boundary values
    bits = rng.integers(0, 2 ** 32, 2_000_000, dtype=np.uint64).astype(np.uint32)
    y = np.concatenate([bits.view(np.float32), _boundary_floats(orc, fmt)])
    y = y[np.isfinite(y) & (np.abs(y) < sat)]
    got = orc.fp8_encode_array(y, fmt)
    ref = torch.from_numpy(y).to(TORCH_DT[fmt]).view(torch.uint8).numpy()
    bad = np.nonzero(got != ref)[0]
    assert bad.size == 0, (y[bad[:5]], got[bad[:5]], ref[bad[:5]])


@pytest.mark.parametrize("fmt", [E4M3, E5M2])
def test_encode_saturates_and_nan(orc, fmt):
    top = 0x7E if fmt == E4M3 else 0x7B
    for y in (1e6, 3.0e38, float("inf"), 464.0 if fmt == E4M3 else 61440.0, 1e5):
        if abs(y) < orc.fp8_max(fmt):
            continue
        assert orc.fp8_encode(y, fmt) == top
        assert orc.fp8_encode(-y, fmt) == 0x80 | top
    assert orc.fp8_encode(float("nan"), fmt) == 0x7F
    assert orc.fp8_encode(-0.0, fmt) == 0x80
    assert orc.fp8_encode(0.0, fmt) == 0x00


def test_encode_ties_to_even(orc):
    # 1.0625 is half-way between 1.0 (code 0x38, even) and 1.125 (0x39)
    assert orc.fp8_encode(1.0625, E4M3) == 0x38
    # 1.1875 half-way between 1.125 (0x39) and 1.25 (0x3A, even)
    assert orc.fp8_encode(1.1875, E4M3) == 0x3A
    # half of the smallest subnormal rounds to zero (even), a hair above to 0x01
    assert orc.fp8_encode(2.0 ** -10, E4M3) == 0x00
    assert orc.fp8_encode(float(np.nextafter(np.float32(2.0 ** -10), np.float32(1))),
                          E4M3) == 0x01


def test_bf16_decode_all_patterns(orc):
    pats = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = torch.from_numpy(pats.view(np.int16)).view(torch.bfloat16).to(torch.float32).numpy()
    for b in range(0, 65536, 1):
        got = orc.bf16_to_f32(b)
        r = ref[b]
        assert (math.isnan(got) and math.isnan(r)) or got == r


def test_bf16_encode_matches_torch(orc):
    rng = np.random.default_rng(11)
    bits = rng.integers(0, 2 ** 32, 500_000, dtype=np.uint64).astype(np.uint32)
    x = bits.view(np.float32)
    x = x[~np.isnan(x)]
    got = orc.to_bf16_array(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(got, ref)
