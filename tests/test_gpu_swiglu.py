"""The SwiGLU producer with Group Scaling's step (i) fused in
(coat_swiglu_group_amax), against the oracle, and the per-tensor quantizer
fed with its maxima."""
import numpy as np
import pytest
import torch

import oracle
from quantized_optimizer_states_b200 import inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from quantized_optimizer_states_b200 import build
    build.build()
    import quantized_optimizer_states_b200 as q
    q.load()
    return q


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda()


def _run(lib, gate, up, G):
    n = gate.size
    out = torch.empty(n, dtype=torch.int16, device="cuda")
    ga = torch.full((-(-n // G),), -1.0, dtype=torch.float32, device="cuda")
    lib.coat_swiglu_group_amax(_dev(gate.reshape(-1)), _dev(up.reshape(-1)), out, ga,
                               group_size=G)
    torch.cuda.synchronize()
    return out.cpu().numpy().view(np.uint16), ga.cpu().numpy()


def _near_midpoint(gate, up, idx):
    """Is the exact binary64 product within 2^-18 (relative) of a BF16
    rounding midpoint?  Only there may binary32 evaluation round the other way."""
    g = oracle.bf16_bits_to_f64(gate.reshape(-1)[idx])
    u = oracle.bf16_bits_to_f64(up.reshape(-1)[idx])
    h = g / (1.0 + np.exp(-g)) * u
    m, e = np.frexp(h)
    frac = np.abs(np.ldexp(h, 8 - np.maximum(e, -125)))
    dist = np.abs(frac - np.floor(frac) - 0.5)
    return dist <= 2.0**-18 * 256


def _check_out(got, ref, gate, up):
    """Equal, except at most 1e-3 of the elements that are one BF16 step
    apart next to a rounding midpoint."""
    diff = np.nonzero(got != ref)[0]
    assert diff.size <= max(1, 1e-3 * got.size), diff.size
    if diff.size:
        step = np.abs(got[diff].astype(np.int32) - ref[diff].astype(np.int32))
        assert np.all(step == 1)
        assert np.all(_near_midpoint(gate, up, diff))


@pytest.mark.parametrize("G", [32, 128, 1024])
def test_swiglu_matches_oracle_and_maxima_are_exact(lib, G):
    w = inputs.activations()
    gate, up = inputs.host_swiglu_inputs(w, rows=64)
    got, ga = _run(lib, gate, up, G)
    ref = oracle.swiglu_bf16(gate.reshape(-1), up.reshape(-1))
    _check_out(got, ref, gate, up)
    # the fused maxima are exactly the maxima of the BF16 output
    assert np.array_equal(ga, oracle.group_amax_of(got, G))


def test_ragged_length_and_special_values(lib):
    G = 128
    vals = np.array([0.0, -0.0, 1.0, -1.0, 100.0, -100.0, 3e38, -3e38, 1e-40], dtype=np.float32)
    rng = np.random.default_rng(3)
    n = 3 * G + 37
    gate = oracle.round_to_bf16(rng.choice(vals, n).astype(np.float64))
    up = oracle.round_to_bf16(rng.normal(0, 2, n))
    got, ga = _run(lib, gate, up, G)
    ref = oracle.swiglu_bf16(gate, up)
    fin = np.isfinite(oracle.bf16_bits_to_f64(ref))
    assert np.array_equal(np.isfinite(oracle.bf16_bits_to_f64(got)), fin)
    _check_out(got[fin], ref[fin], gate[fin], up[fin])
    assert np.array_equal(ga, oracle.group_amax_of(got, G))


def test_fused_maxima_feed_group_scaling(lib):
    """Producer maxima + the per-tensor quantizer (step (i) skipped) give the
    same codes and scale as the oracle's Group Scaling on the same BF16
    tensor -- bit-exact."""
    G = 128
    w = inputs.activations()
    gate, up = inputs.host_swiglu_inputs(w, rows=32)
    n = gate.size
    out = torch.empty(n, dtype=torch.int16, device="cuda")
    ws = torch.empty(lib.coat_group_scaling_workspace_bytes(n, G) // 4, dtype=torch.float32,
                     device="cuda")
    lib.coat_swiglu_group_amax(_dev(gate.reshape(-1)), _dev(up.reshape(-1)), out, ws,
                               group_size=G)
    q = torch.empty(n, dtype=torch.uint8, device="cuda")
    sc = torch.empty(1, dtype=torch.float32, device="cuda")
    lib.coat_group_scaling_quant_pertensor(out, ws, q, sc, group_size=G, amax_precomputed=True)
    torch.cuda.synchronize()
    h = out.cpu().numpy().view(np.uint16)
    q_ref, s_ref, _ = oracle.group_scaling_pertensor(h, G, 0)
    assert np.array_equal(q.cpu().numpy(), q_ref)
    assert float(sc.item()) == s_ref


@pytest.mark.parametrize("rows,G", [(32, 128), (17, 512)])
def test_tensor_max_from_the_producer(lib, rows, G):
    """With tensor_amax the producer also folds step (ii) in: Group Scaling
    with amax_precomputed=2 runs the cast alone and gives the oracle's codes
    and scale (ragged length: 17 rows minus 5 elements)."""
    w = inputs.activations(seed=rows)
    gate, up = inputs.host_swiglu_inputs(w, rows=rows)
    n = gate.size - 5
    gate, up = gate.reshape(-1)[:n].copy(), up.reshape(-1)[:n].copy()
    out = torch.empty(n, dtype=torch.int16, device="cuda")
    ws = torch.full((lib.coat_group_scaling_workspace_bytes(n, G) // 4,), 7.0,
                    dtype=torch.float32, device="cuda")
    ng = -(-n // G)
    lib.coat_swiglu_group_amax(_dev(gate), _dev(up), out, ws, group_size=G,
                               tensor_amax=ws[ng:])
    q = torch.empty(n, dtype=torch.uint8, device="cuda")
    sc = torch.empty(1, dtype=torch.float32, device="cuda")
    lib.coat_group_scaling_quant_pertensor(out, ws, q, sc, group_size=G, amax_precomputed=2)
    torch.cuda.synchronize()
    h = out.cpu().numpy().view(np.uint16)
    q_ref, s_ref, ga_ref = oracle.group_scaling_pertensor(h, G, 0)
    assert float(ws[ng].item()) == float(ga_ref.max())
    assert np.array_equal(q.cpu().numpy(), q_ref)
    assert float(sc.item()) == s_ref


def test_argument_errors(lib):
    from quantized_optimizer_states_b200._lib import CoatError
    x = torch.zeros(256, dtype=torch.int16, device="cuda")
    ga = torch.zeros(4, dtype=torch.float32, device="cuda")
    with pytest.raises(CoatError):
        lib.coat_swiglu_group_amax(x, x, x, ga, group_size=100)
    with pytest.raises(ValueError):
        lib.coat_swiglu_group_amax(x, x[:128], x, ga, group_size=128)


def test_producers_write_the_tensor_max_into_a_whole_workspace_by_default(lib):
    """Handed a whole Group Scaling workspace (ceil(n/G) + 1 floats), both
    producers write the tensor maximum into its last slot unless told not
    to (tensor_amax=None leaves the slot as it was); handed exactly the
    group maxima they write nothing past them."""
    G, rows, cols = 128, 24, 1024
    w = inputs.activations(seed=3)
    gate, up = inputs.host_swiglu_inputs(w, rows=rows)
    gate, up = gate[:, :cols].copy(), up[:, :cols].copy()
    n = gate.size
    ng = n // G
    for default in (True, False):
        out = torch.empty(n, dtype=torch.int16, device="cuda")
        ws = torch.full((ng + 1,), -5.0, dtype=torch.float32, device="cuda")
        kw = {} if default else {"tensor_amax": None}
        lib.coat_swiglu_group_amax(_dev(gate), _dev(up), out, ws, group_size=G, **kw)
        ln = torch.empty(rows, cols, dtype=torch.int16, device="cuda")
        ws2 = torch.full((ng + 1,), -5.0, dtype=torch.float32, device="cuda")
        lib.coat_norm_group_amax(out.view(rows, cols), ln, ws2, group_size=G, **kw)
        torch.cuda.synchronize()
        for buf in (ws, ws2):
            want = float(buf[:ng].max().item()) if default else -5.0
            assert float(buf[ng].item()) == want
    exact = torch.full((ng + 8,), -5.0, dtype=torch.float32, device="cuda")
    lib.coat_swiglu_group_amax(_dev(gate), _dev(up), out, exact[:ng], group_size=G)
    torch.cuda.synchronize()
    assert torch.all(exact[ng:] == -5.0)
