"""GPU parity of the LayerNorm / RMSNorm producer with fused 1xG maxima
(coat_norm_group_amax) against the oracle: the BF16 output equals the
binary64 norm rounded once, except one BF16 step apart where the binary64
value lies within the binary32 evaluation's error (4e-6 relative) of a
rounding midpoint, for at most 1e-3 of the elements; the maxima are those
of the output; Group Scaling with the producer's maxima equals Group
Scaling on its own."""
import numpy as np
import pytest

import parity
from quantized_optimizer_states_b200 import inputs

pytestmark = pytest.mark.gpu
E4M3 = 0


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


WINDOW = 4e-6          # relative error of the binary32 evaluation, with margin
MAX_FLIPS = 1e-3       # fraction of elements allowed one BF16 step off


def _midpoint_ok(orc, y64, got_bits, want_bits, offset):
    """Every difference is the correct rounding of a value within the
    binary32 evaluation's error of the binary64 norm: |got - y| <= half a
    BF16 step of got + WINDOW x (|y| + offset), offset = (|x - mean| +
    |mean|) / std x |weight| of the element's row (x - mean carries the
    rounding of the mean; with a bias the product's rounding is relative
    to it, not to y).  Without a bias that is one BF16 step next to a
    rounding midpoint."""
    bad = np.nonzero(got_bits != want_bits)[0]
    assert bad.size <= MAX_FLIPS * got_bits.size, bad.size
    for i in bad:
        g = orc.bf16_bits_to_f64(np.array([got_bits[i], got_bits[i] + 1, got_bits[i] - 1],
                                          dtype=np.uint16))
        half = 0.5 * max(abs(g[1] - g[0]), abs(g[0] - g[2]))
        assert abs(g[0] - y64[i]) <= half + WINDOW * (abs(y64[i]) + offset[i]), i
    return bad.size


def _offset(orc, x, weight, rms):
    """(|x - mean| + |mean|) / std x |weight| per element (binary64)."""
    xf = orc.bf16_bits_to_f64(x)
    w = np.ones(x.shape[1]) if weight is None else np.abs(weight.astype(np.float64))
    if rms:
        sd = np.sqrt((xf ** 2).mean(axis=1, keepdims=True) + float(np.float32(1e-5)))
        return (np.abs(xf) / sd * w).reshape(-1)
    mu = xf.mean(axis=1, keepdims=True)
    sd = np.sqrt(((xf - mu) ** 2).mean(axis=1, keepdims=True) + float(np.float32(1e-5)))
    return ((np.abs(xf - mu) + np.abs(mu)) / sd * w).reshape(-1)


# widths that are multiples of 256 up to 2048 take the register-resident
# kernel (every chunk count 1..8 below, groups within one load column and
# across several, more rows than the persistent grid has warps); the others
# the shared-memory one
@pytest.mark.parametrize("rows,cols,G", [(64, 2048, 128), (24, 4096, 128), (8, 16384, 4096),
                                         (40, 768, 256), (16, 5120, 512), (33, 1536, 128),
                                         (3000, 256, 16), (20, 2048, 1024), (12, 2048, 2048),
                                         (9, 1024, 512), (10, 1280, 256), (16, 1792, 64),
                                         (7, 512, 32), (24, 1040, 16)])
@pytest.mark.parametrize("rms", [False, True])
def test_norm_matches_oracle(lib, orc, rows, cols, G, rms):
    import torch
    w = inputs.activations(seed=rows + cols)
    x = inputs.host_activations(w, rows=rows)
    x = np.tile(x, (1, -(-cols // x.shape[1])))[:, :cols].copy()
    x[0, :] = x[0, 0]                          # a constant row
    rng = np.random.default_rng(cols)
    weight = (1.0 + 0.1 * rng.standard_normal(cols)).astype(np.float32)
    bias = None if rms else (0.05 * rng.standard_normal(cols)).astype(np.float32)
    out = torch.empty(rows, cols, dtype=torch.int16, device="cuda")
    ga = torch.empty(rows * cols // G, dtype=torch.float32, device="cuda")
    lib.coat_norm_group_amax(parity.to_dev(x.view(np.int16)), out, ga, rms=rms, eps=1e-5,
                             weight=parity.to_dev(weight),
                             bias=None if bias is None else parity.to_dev(bias), group_size=G)
    torch.cuda.synchronize()
    got = parity.to_host(out).view(np.uint16).reshape(-1)
    y64 = orc.norm_f64(x, rms=rms, eps=1e-5, weight=weight, bias=bias).reshape(-1)
    want = orc.round_to_bf16(y64)
    _midpoint_ok(orc, y64, got, want, _offset(orc, x, weight, rms))
    assert np.array_equal(parity.to_host(ga), orc.group_amax_of(got, G))


@pytest.mark.parametrize("cols", [2048, 768, 1040])
def test_norm_affine_terms_at_any_4_byte_alignment(lib, orc, cols):
    """weight and bias 16-byte aligned (the register form loads 8 columns
    by two 16-byte loads) and at a 4-byte offset (one load a column): the
    same output and maxima bit for bit, and those of the oracle check."""
    import torch
    rows, G = 40, 16
    x = inputs.host_activations(inputs.activations(seed=cols), rows=rows)
    x = np.tile(x, (1, -(-cols // x.shape[1])))[:, :cols].copy()
    rng = np.random.default_rng(cols + 1)
    weight = (1.0 + 0.1 * rng.standard_normal(cols)).astype(np.float32)
    bias = (0.05 * rng.standard_normal(cols)).astype(np.float32)
    runs = []
    for off in (0, 1):
        wbuf = torch.zeros(cols + 4, dtype=torch.float32, device="cuda")
        bbuf = torch.zeros(cols + 4, dtype=torch.float32, device="cuda")
        wbuf[off:off + cols] = torch.from_numpy(weight)
        bbuf[off:off + cols] = torch.from_numpy(bias)
        out = torch.empty(rows, cols, dtype=torch.int16, device="cuda")
        ga = torch.empty(rows * cols // G, dtype=torch.float32, device="cuda")
        lib.coat_norm_group_amax(parity.to_dev(x.view(np.int16)), out, ga, eps=1e-5,
                                 weight=wbuf[off:off + cols], bias=bbuf[off:off + cols],
                                 group_size=G)
        torch.cuda.synchronize()
        runs.append((parity.to_host(out).view(np.uint16).reshape(-1), parity.to_host(ga)))
    assert np.array_equal(runs[0][0], runs[1][0]) and np.array_equal(runs[0][1], runs[1][1])
    y64 = orc.norm_f64(x, rms=False, eps=1e-5, weight=weight, bias=bias).reshape(-1)
    _midpoint_ok(orc, y64, runs[0][0], orc.round_to_bf16(y64), _offset(orc, x, weight, False))
    assert np.array_equal(runs[0][1], orc.group_amax_of(runs[0][0], G))


def test_norm_feeds_group_scaling(lib, orc):
    """The producer's maxima make Group Scaling skip its first step with
    the same codes and scale as the standalone quantizer."""
    import torch
    rows, cols, G = 128, 2048, 128
    x = inputs.host_activations(inputs.activations(seed=3), rows=rows)
    out = torch.empty(rows, cols, dtype=torch.int16, device="cuda")
    n = rows * cols
    ws = torch.empty(lib.coat_group_scaling_workspace_bytes(n, G) // 4, dtype=torch.float32,
                     device="cuda")
    lib.coat_norm_group_amax(parity.to_dev(x.view(np.int16)), out, ws[:n // G], group_size=G)
    q1 = torch.empty(n, dtype=torch.uint8, device="cuda")
    s1 = torch.empty(1, dtype=torch.float32, device="cuda")
    lib.coat_group_scaling_quant_pertensor(out.reshape(-1), ws, q1, s1, group_size=G,
                                           amax_precomputed=True)
    q2 = torch.empty_like(q1)
    s2 = torch.empty_like(s1)
    ws2 = torch.empty_like(ws)
    lib.coat_group_scaling_quant_pertensor(out.reshape(-1), ws2, q2, s2, group_size=G)
    torch.cuda.synchronize()
    assert torch.equal(q1, q2) and torch.equal(s1, s2)
    q_ref, s_ref, _ = orc.group_scaling_pertensor(parity.to_host(out).view(np.uint16), G, E4M3)
    assert np.array_equal(parity.to_host(q1), q_ref) and float(s1.item()) == s_ref


@pytest.mark.parametrize("cols", [4096, 2048])
@pytest.mark.parametrize("rms", [False, True])
def test_norm_tensor_max_feeds_the_cast_alone(lib, orc, rms, cols):
    """tensor_amax: the producer also writes the tensor maximum; Group
    Scaling with amax_precomputed=2 then only casts, with the oracle's codes
    and scale; amax_precomputed outside 0..2 is rejected."""
    import torch
    rows, G = 300, 128
    x = inputs.host_activations(inputs.activations(seed=8), rows=rows)
    x = np.tile(x, (1, 2))[:, :cols].copy()
    n = rows * cols
    out = torch.empty(rows, cols, dtype=torch.int16, device="cuda")
    ws = torch.full((lib.coat_group_scaling_workspace_bytes(n, G) // 4,), 3.0,
                    dtype=torch.float32, device="cuda")
    lib.coat_norm_group_amax(parity.to_dev(x.view(np.int16)), out, ws[:n // G], rms=rms,
                             group_size=G, tensor_amax=ws[n // G:])
    q = torch.empty(n, dtype=torch.uint8, device="cuda")
    s = torch.empty(1, dtype=torch.float32, device="cuda")
    lib.coat_group_scaling_quant_pertensor(out.reshape(-1), ws, q, s, group_size=G,
                                           amax_precomputed=2)
    torch.cuda.synchronize()
    h = parity.to_host(out).view(np.uint16)
    q_ref, s_ref, ga_ref = orc.group_scaling_pertensor(h, G, E4M3)
    assert float(ws[n // G].item()) == float(ga_ref.max())
    assert np.array_equal(parity.to_host(q), q_ref) and float(s.item()) == s_ref
    with pytest.raises(lib.CoatError) as e:
        lib.coat_group_scaling_quant_pertensor(out.reshape(-1), ws, q, s, group_size=G,
                                               amax_precomputed=3)
    assert e.value.status == 1


def test_norm_argument_errors(lib):
    import torch
    x = torch.zeros(4, 128, dtype=torch.int16, device="cuda")
    ga = torch.zeros(4, dtype=torch.float32, device="cuda")
    b = torch.zeros(128, dtype=torch.float32, device="cuda")
    with pytest.raises(lib.CoatError) as e:
        lib.coat_norm_group_amax(x, x.clone(), ga, rms=True, bias=b)   # bias with RMSNorm
    assert e.value.status == 1
    with pytest.raises(lib.CoatError) as e:
        lib.coat_norm_group_amax(x, x.clone(), ga, eps=-1.0)
    assert e.value.status == 1
    with pytest.raises(lib.CoatError) as e:
        lib.coat_norm_group_amax(x, x.clone(), ga, group_size=96)
    assert e.value.status == 3
