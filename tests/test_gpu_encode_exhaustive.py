"""The hardware FP8 cast (coat_fp8_encode: cvt.rn.satfinite on sm_100a)
against the oracle's encoder, exhaustively over every binary32 bit pattern
of the binades in which rounding to the format happens (both signs, every
mantissa), plus a random sample of all other patterns and the special
values.  The oracle runs in a pool of spawned processes."""
import multiprocessing as mp
import os

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu
E4M3, E5M2 = 0, 1
# unbiased binary32 exponents whose binades reach from below half the
# smallest subnormal (codes round to 0 there) to above the largest finite
# value (codes saturate there)
WINDOW = {E4M3: (-12, 9), E5M2: (-19, 16)}
NAN_CODES = {E4M3: {0x7F, 0xFF}, E5M2: {0x7D, 0x7E, 0x7F, 0xFD, 0xFE, 0xFF}}


def _binade(e: int, neg: bool) -> np.ndarray:
    m = np.arange(1 << 23, dtype=np.uint32)
    bits = m | np.uint32((e + 127) << 23)
    if neg:
        bits |= np.uint32(0x80000000)
    return bits.view(np.float32)


def _oracle_binade(args):
    import oracle
    fmt, e, neg = args
    return oracle.fp8_encode_array(_binade(e, neg), fmt)


@pytest.fixture(scope="module")
def lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from quantized_optimizer_states_b200 import build
    build.build()
    import quantized_optimizer_states_b200 as q
    q.load()
    return q


def _gpu(lib, y: np.ndarray, fmt: int) -> np.ndarray:
    d = torch.from_numpy(np.ascontiguousarray(y)).cuda()
    q = torch.empty(y.size, dtype=torch.uint8, device="cuda")
    lib.coat_fp8_encode(d, q, fmt=fmt)
    return q.cpu().numpy()


@pytest.mark.parametrize("fmt", [E4M3, E5M2])
def test_every_pattern_of_the_rounding_binades(lib, fmt):
    lo, hi = WINDOW[fmt]
    jobs = [(fmt, e, neg) for e in range(lo, hi + 1) for neg in (False, True)]
    workers = max(1, min(32, os.cpu_count() or 1))
    ctx = mp.get_context("spawn")
    with ctx.Pool(workers) as pool:
        for (f, e, neg), ref in zip(jobs, pool.imap(_oracle_binade, jobs)):
            got = _gpu(lib, _binade(e, neg), fmt)
            bad = np.nonzero(got != ref)[0]
            assert bad.size == 0, (
                f"exponent {e} sign {neg}: {bad.size} codes differ, first at mantissa "
                f"{bad[0]:#x}: gpu {got[bad[0]]:#x} oracle {ref[bad[0]]:#x}")


@pytest.mark.parametrize("fmt", [E4M3, E5M2])
def test_random_patterns_and_specials(lib, orc, fmt):
    rng = np.random.default_rng(99 + fmt)
    bits = rng.integers(0, 2**32, 1 << 22, dtype=np.uint64).astype(np.uint32)
    specials = np.array([0x00000000, 0x80000000, 0x7F800000, 0xFF800000, 0x7FC00000,
                         0xFFC00000, 0x7F800001, 0x7F7FFFFF, 0xFF7FFFFF, 0x00000001,
                         0x807FFFFF], dtype=np.uint32)
    y = np.concatenate([bits, specials]).view(np.float32)
    got = _gpu(lib, y, fmt)
    ref = orc.fp8_encode_array(y, fmt)
    nan = np.isnan(y)
    assert np.array_equal(got[~nan], ref[~nan])
    assert all(int(c) in NAN_CODES[fmt] for c in got[nan])
