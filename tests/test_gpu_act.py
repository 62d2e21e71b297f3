"""GPU parity of COAT's activation quantizers and FP8 dequantization against
the oracle, through the C ABI.  These paths are bit-exact."""
import numpy as np
import pytest

import parity
from quantized_optimizer_states_b200 import inputs

pytestmark = pytest.mark.gpu

E4M3, E5M2 = 0, 1


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


def _gpu_1xG(lib, x, G, fmt, ld=None):
    import torch
    rows, cols = x.shape
    if ld is None:
        xd = parity.to_dev(x.view(np.int16))
    else:
        padded = np.zeros((rows, ld), dtype=np.uint16)
        padded[:, :cols] = x
        xd = parity.to_dev(padded.view(np.int16))[:, :cols]
    q = torch.empty(rows, cols, dtype=torch.uint8, device="cuda")
    sc = torch.empty(rows, cols // G, dtype=torch.float32, device="cuda")
    lib.coat_group_quant_1xG(xd, q, sc, group_size=G, fmt=fmt)
    torch.cuda.synchronize()
    return parity.to_host(q), parity.to_host(sc)


def test_group_quant_full_activation_set(lib, orc):
    """The activation workload: BF16 [16384, 2048], G = 128, E4M3."""
    w = inputs.activations()
    x = inputs.host_activations(w)
    q, sc = _gpu_1xG(lib, x, 128, E4M3)
    q_ref, sc_ref = orc.group_quant_1xG(x, 128, E4M3)
    assert np.array_equal(sc, sc_ref)
    assert np.array_equal(q, q_ref)


@pytest.mark.parametrize("G", [16, 32, 64, 256, 512, 1024, 2048])
@pytest.mark.parametrize("fmt", [E4M3, E5M2])
def test_group_quant_group_sizes(lib, orc, G, fmt):
    w = inputs.activations(seed=G + fmt)
    x = inputs.host_activations(w, rows=37)
    q, sc = _gpu_1xG(lib, x, G, fmt)
    q_ref, sc_ref = orc.group_quant_1xG(x, G, fmt)
    assert np.array_equal(sc, sc_ref) and np.array_equal(q, q_ref)


def test_group_quant_strided_rows_and_special_values(lib, orc):
    rng = np.random.default_rng(3)
    x = inputs.host_activations(inputs.activations(seed=9), rows=11)[:, :512].copy()
    x[0, :] = 0                      # all-zero groups -> s = 1
    x[1, :128] = 0x8000              # negative zeros
    x[2, 5] = 0x7F80                 # +inf in one group
    x[3, 7] = 0x0001                 # a BF16 subnormal
    x[4, :] = (rng.integers(0, 2, 512) * 0x8000 + 0x0080).astype(np.uint16)  # tiny values
    q, sc = _gpu_1xG(lib, x, 128, E4M3, ld=520)
    q_ref, sc_ref = orc.group_quant_1xG(x, 128, E4M3)
    assert np.array_equal(sc, sc_ref)
    assert np.array_equal(q, q_ref)


def test_group_quant_contiguous_group_4096_and_partial_tiles(lib, orc):
    """Contiguous rows go through the flat kernel (each block two
    4096-element tiles): G = 4096 (a group filling a whole tile), and sizes
    that end on a whole block, in the second tile of a block, or a few
    groups into a tile."""
    for rows, cols, G in ((5, 8192, 4096), (3, 4096 + 2048, 2048), (7, 1152, 128)):
        x = inputs.host_activations(inputs.activations(seed=rows), rows=rows)
        x = np.tile(x, (1, -(-cols // x.shape[1])))[:, :cols].copy()
        q, sc = _gpu_1xG(lib, x, G, E4M3)
        q_ref, sc_ref = orc.group_quant_1xG(x, G, E4M3)
        assert np.array_equal(sc, sc_ref) and np.array_equal(q, q_ref), (rows, cols, G)


def _gpu_group_scaling(lib, x, G, fmt, group_amax=None):
    import torch
    n = x.size
    ws = torch.empty(lib.coat_group_scaling_workspace_bytes(n, G) // 4, dtype=torch.float32,
                     device="cuda")
    if group_amax is not None:
        ws[:group_amax.size].copy_(torch.from_numpy(group_amax))
    q = torch.empty(n, dtype=torch.uint8, device="cuda")
    sc = torch.empty(1, dtype=torch.float32, device="cuda")
    lib.coat_group_scaling_quant_pertensor(parity.to_dev(x.view(np.int16)), ws, q, sc,
                                           group_size=G, fmt=fmt,
                                           amax_precomputed=group_amax is not None)
    torch.cuda.synchronize()
    ng = -(-n // G)
    return parity.to_host(q), float(parity.to_host(sc)[0]), parity.to_host(ws)[:ng]


@pytest.mark.parametrize("fmt", [E4M3, E5M2])
def test_group_scaling_full_activation_set(lib, orc, fmt):
    w = inputs.activations()
    x = inputs.host_activations(w).reshape(-1)
    q, s, ga = _gpu_group_scaling(lib, x, 128, fmt)
    q_ref, s_ref, ga_ref = orc.group_scaling_pertensor(x, 128, fmt)
    assert np.array_equal(ga, ga_ref)
    assert s == s_ref
    assert np.array_equal(q, q_ref)


@pytest.mark.parametrize("G", [16, 128, 1024, 4096])
def test_group_scaling_ragged_and_precomputed(lib, orc, G):
    x = inputs.host_activations(inputs.activations(seed=G), rows=19).reshape(-1)
    x = x[:x.size - 37].copy()
    q, s, ga = _gpu_group_scaling(lib, x, G, E4M3)
    q_ref, s_ref, ga_ref = orc.group_scaling_pertensor(x, G, E4M3)
    assert np.array_equal(ga, ga_ref) and s == s_ref and np.array_equal(q, q_ref)
    # the producer-fused path: maxima supplied, step (i) skipped
    q2, s2, _ = _gpu_group_scaling(lib, x, G, E4M3, group_amax=ga_ref)
    assert s2 == s_ref and np.array_equal(q2, q_ref)


@pytest.mark.parametrize("fmt", [E4M3, E5M2])
def test_activation_dequant_bit_exact(lib, orc, fmt):
    import torch
    x = inputs.host_activations(inputs.activations(seed=5), rows=64)
    q, sc = orc.group_quant_1xG(x, 128, fmt)
    n = q.size
    ref = orc.dequant(q.reshape(-1), None, sc.reshape(-1), 128, fmt)
    out = torch.empty(n, dtype=torch.float32, device="cuda")
    lib.coat_dequant(parity.to_dev(q.reshape(-1)), None, parity.to_dev(sc.reshape(-1)), out,
                     group_size=128, fmt=fmt)
    outb = torch.empty(n, dtype=torch.bfloat16, device="cuda")
    lib.coat_dequant(parity.to_dev(q.reshape(-1)), None, parity.to_dev(sc.reshape(-1)), outb,
                     group_size=128, fmt=fmt)
    torch.cuda.synchronize()
    assert np.array_equal(parity.to_host(out), ref)
    assert np.array_equal(parity.to_host(outb).view(np.uint16), orc.to_bf16_array(ref))
    # per-tensor: one scale for the whole tensor (G >= n), ragged length
    s1 = np.array([0.37], dtype=np.float32)
    m = n - 9
    ref1 = orc.dequant(q.reshape(-1)[:m], None, s1, m, fmt)
    out1 = torch.empty(m, dtype=torch.float32, device="cuda")
    lib.coat_dequant(parity.to_dev(q.reshape(-1)[:m]), None, parity.to_dev(s1), out1,
                     group_size=m, fmt=fmt)
    torch.cuda.synchronize()
    assert np.array_equal(parity.to_host(out1), ref1)


@pytest.mark.parametrize("out_bf16", [False, True])
def test_activation_dequant_full_set(lib, orc, out_bf16):
    """The activation workload's codes dequantized per 1xG group, and a
    per-tensor length that is not a whole number of tiles."""
    import torch
    x = inputs.host_activations(inputs.activations())
    q, sc = orc.group_quant_1xG(x, 128, E4M3)
    ref = orc.dequant(q.reshape(-1), None, sc.reshape(-1), 128, E4M3)
    dt = torch.bfloat16 if out_bf16 else torch.float32
    out = torch.empty(q.size, dtype=dt, device="cuda")
    lib.coat_dequant(parity.to_dev(q.reshape(-1)), None, parity.to_dev(sc.reshape(-1)), out,
                     group_size=128, fmt=E4M3)
    m = q.size - 4096 * 3 - 48
    s1 = np.array([1.5e-3], dtype=np.float32)
    out1 = torch.empty(m, dtype=dt, device="cuda")
    lib.coat_dequant(parity.to_dev(q.reshape(-1)[:m]), None, parity.to_dev(s1), out1,
                     group_size=m, fmt=E4M3)
    torch.cuda.synchronize()
    ref1 = orc.dequant(q.reshape(-1)[:m], None, s1, m, E4M3)
    if out_bf16:
        assert np.array_equal(parity.to_host(out).view(np.uint16), orc.to_bf16_array(ref))
        assert np.array_equal(parity.to_host(out1).view(np.uint16), orc.to_bf16_array(ref1))
    else:
        assert np.array_equal(parity.to_host(out), ref)
        assert np.array_equal(parity.to_host(out1), ref1)


def test_hardware_cvt_matches_oracle_encoder(lib, orc):
    """The sm_100a cvt...satfinite path (through the 1xG quantizer with unit
    scale, i.e. a group whose amax is exactly 448) against the oracle's
    encoder, on every BF16 bit pattern."""
    pats = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    # one group per pattern: [pattern, 448.0, 0...] so inv = 1 and y = x
    G = 16
    x = np.zeros((65536, G), dtype=np.uint16)
    x[:, 0] = pats
    x[:, 1] = 0x43E0  # 448.0 in BF16
    finite = (pats & 0x7F80) != 0x7F80
    small = np.abs(orc_f32(pats)) <= 448.0
    rows = x[finite & small]
    q, sc = _gpu_1xG(lib, rows, G, E4M3)
    q_ref, sc_ref = orc.group_quant_1xG(rows, G, E4M3)
    assert np.all(sc == np.float32(1.0)) and np.array_equal(sc, sc_ref)
    assert np.array_equal(q, q_ref)


def orc_f32(bits):
    return (bits.astype(np.uint32) << 16).view(np.float32)
