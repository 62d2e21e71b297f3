"""GPU tests of the multi-tensor pack / unpack (coat_pack_bf16,
coat_unpack_bf16): every element against the oracle's binary32 -> BF16
rounding, ragged and empty tensors, unaligned source views, missing
gradients, more tensors than one launch takes, and the untouched padding
between slices."""
import numpy as np
import pytest

import parity

pytestmark = pytest.mark.gpu

SIZES = [0, 1, 7, 8, 2047, 2048, 2049, 4096 + 5, 100_003, 16, 3, 65_536]


@pytest.fixture(scope="module")
def lib():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from quantized_optimizer_states_b200 import build
    build.build()
    import quantized_optimizer_states_b200 as q
    q.load()
    return q


def _layout(sizes, unit=16):
    offs, off = [], 0
    for n in sizes:
        offs.append(off)
        off += -(-n // unit) * unit + unit   # a gap of padding after every slice
    return offs, off


def _values(rng, n):
    x = (rng.standard_normal(n) * 10.0 ** rng.uniform(-30, 30, n)).astype(np.float32)
    if n > 4:
        x[:4] = [np.inf, -np.inf, 0.0, -0.0]
    return x


@pytest.mark.parametrize("count", [len(SIZES), 300])
def test_pack_fp32_sources(lib, orc, count):
    import torch
    rng = np.random.default_rng(count)
    sizes = [SIZES[i % len(SIZES)] for i in range(count)]
    offs, n = _layout(sizes)
    host = [_values(rng, m) for m in sizes]
    srcs = []
    for i, x in enumerate(host):
        if i % 11 == 5:
            srcs.append(None)                                   # no gradient: zeros
        elif i % 7 == 3 and x.size > 0:
            buf = parity.to_dev(np.concatenate([[1.0], x]).astype(np.float32))
            srcs.append(buf[1:])                                # 4-byte-aligned view
        else:
            srcs.append(parity.to_dev(x))
    dst = torch.full((n,), 0x5A5A, dtype=torch.int16, device="cuda")
    table = lib.PackTable(sizes, offs)
    lib.coat_pack_bf16(srcs, table, dst)
    torch.cuda.synchronize()
    got = parity.to_host(dst).view(np.uint16)
    covered = np.zeros(n, dtype=bool)
    for i, (x, off) in enumerate(zip(host, offs)):
        want = np.zeros(x.size, np.uint16) if srcs[i] is None else orc.to_bf16_array(x)
        assert np.array_equal(got[off:off + x.size], want), i
        covered[off:off + x.size] = True
    assert np.all(got[~covered] == 0x5A5A)                      # padding untouched


def test_pack_bf16_sources_and_unpack(lib, orc):
    import torch
    rng = np.random.default_rng(7)
    sizes = SIZES * 12                                           # 144 tensors: two launches
    offs, n = _layout(sizes)
    bits = [orc.to_bf16_array(_values(rng, m)) for m in sizes]
    srcs = [parity.to_dev(b.view(np.int16)) for b in bits]
    dst = torch.zeros(n, dtype=torch.int16, device="cuda")
    table = lib.PackTable(sizes, offs)
    lib.coat_pack_bf16(srcs, table, dst)
    torch.cuda.synchronize()
    got = parity.to_host(dst).view(np.uint16)
    for b, off in zip(bits, offs):
        assert np.array_equal(got[off:off + b.size], b)

    flat = _values(rng, n)
    outs = [torch.full((m,), 0x1234, dtype=torch.int16, device="cuda") for m in sizes]
    lib.coat_unpack_bf16(parity.to_dev(flat), table, outs)
    torch.cuda.synchronize()
    for o, m, off in zip(outs, sizes, offs):
        assert np.array_equal(parity.to_host(o).view(np.uint16),
                              orc.to_bf16_array(flat[off:off + m]))
