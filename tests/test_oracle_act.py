"""Pins of the oracle's activation quantizers (CPU only).

COAT summary page, section "混合粒度：线性层和非线性层分开处理": nonlinear-layer
inputs use 1xG groups along channels; linear-layer inputs use one scale per
tensor, found by Group Scaling (max per 1xG run, then max of those).
Pinned against torch's abs-max and float8 cast (library routines) and the
special case that Group Scaling with one group is a single 1xG group.
"""
import numpy as np
import pytest
import torch

from quantized_optimizer_states_b200 import inputs

E4M3, E5M2 = 0, 1
TORCH_DT = {E4M3: torch.float8_e4m3fn, E5M2: torch.float8_e5m2}
FMAX = {E4M3: 448.0, E5M2: 57344.0}


def _bf16_to_f32(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).float()


@pytest.mark.parametrize("fmt", [E4M3, E5M2])
@pytest.mark.parametrize("G", [32, 128, 512])
def test_group_quant_1xG_matches_torch_cast(orc, fmt, G):
    w = inputs.activations()
    x = inputs.host_activations(w, rows=64)
    q, sc = orc.group_quant_1xG(x, G, fmt)
    xf = _bf16_to_f32(x).reshape(64, -1, G)
    amax = xf.abs().amax(dim=-1)
    fmax = torch.tensor(FMAX[fmt], dtype=torch.float32)
    assert torch.equal(torch.from_numpy(sc), amax / fmax)
    inv = fmax / amax
    ref = (xf * inv[..., None]).to(TORCH_DT[fmt]).view(torch.uint8).reshape(64, -1).numpy()
    assert np.array_equal(q, ref)


def test_group_quant_zero_group_and_negative_zero(orc):
    x = np.zeros((2, 64), dtype=np.uint16)
    x[1, :] = 0x8000             # -0.0 in BF16
    x[1, 3] = 0x3F80             # 1.0
    q, sc = orc.group_quant_1xG(x, 32, E4M3)
    assert sc[0, 0] == 1.0 and sc[0, 1] == 1.0 and np.all(q[0] == 0)
    assert sc[1, 0] == np.float32(1.0) / np.float32(448.0)
    assert q[1, 3] == 0x7E and q[1, 0] == 0x80
    assert sc[1, 1] == 1.0 and np.all(q[1, 32:] == 0x80)


@pytest.mark.parametrize("fmt", [E4M3, E5M2])
def test_group_scaling_matches_torch_and_single_group(orc, fmt):
    w = inputs.activations()
    x = inputs.host_activations(w, rows=48).reshape(-1)
    n = x.size - 123              # ragged tail group
    x = x[:n].copy()
    q, s, ga = orc.group_scaling_pertensor(x, 128, fmt)
    xf = _bf16_to_f32(x)
    amax = xf.abs().max()
    assert ga.max() == amax.item()
    assert s == (amax / torch.tensor(FMAX[fmt])).item()
    ref = (xf * (torch.tensor(FMAX[fmt]) / amax)).to(TORCH_DT[fmt]).view(torch.uint8).numpy()
    assert np.array_equal(q, ref)
    # one 1xG group spanning the whole tensor is the same quantizer
    q1, sc1 = orc.group_quant_1xG(x.reshape(1, n), n, fmt)
    assert np.array_equal(q1.reshape(-1), q) and sc1[0, 0] == np.float32(s)
    # producer-supplied per-group maxima give the same result
    q2, s2, _ = orc.group_scaling_pertensor(x, 128, fmt, group_amax=ga)
    assert np.array_equal(q2, q) and s2 == s


@pytest.mark.parametrize("fmt", [E4M3, E5M2])
def test_group_quant_1xG_row_stride(orc, fmt):
    """Rows taken from a wider buffer (row stride ld > cols) are quantized as
    the same rows stored contiguously, and the columns past cols -- here
    large values that would change every scale -- are never read."""
    G, rows, cols, ld = 64, 12, 256, 256 + 96
    x = inputs.host_activations(inputs.activations(seed=3), rows=rows)[:, :cols].copy()
    wide = np.full((rows, ld), 0x4780, dtype=np.uint16)          # BF16 65536
    wide[:, :cols] = x
    q, sc = orc.group_quant_1xG(wide, G, fmt, cols=cols)
    xf = _bf16_to_f32(x).reshape(rows, -1, G)
    amax = xf.abs().amax(dim=-1)
    fmax = torch.tensor(FMAX[fmt], dtype=torch.float32)
    assert torch.equal(torch.from_numpy(sc), amax / fmax)
    ref = (xf * (fmax / amax)[..., None]).to(TORCH_DT[fmt]).view(torch.uint8).reshape(rows, -1)
    assert np.array_equal(q, ref.numpy())


@pytest.mark.parametrize("fmt", [E4M3, E5M2])
def test_group_scaling_max_in_the_last_partial_group(orc, fmt):
    """The tensor maximum in the shorter last group still sets the scale:
    s = amax / fmt_max, the largest element encodes to the top code."""
    n, G = 1000, 128                                 # 7 full groups and one of 104
    x = np.full(n, 0x3F80, dtype=np.uint16)          # 1.0
    x[n - 1] = 0x447A                                # BF16 1000.0
    q, s, ga = orc.group_scaling_pertensor(x, G, fmt)
    assert ga[-1] == 1000.0 and np.all(ga[:-1] == 1.0)
    assert s == np.float32(1000.0) / np.float32(FMAX[fmt])
    top = 0x7E if fmt == E4M3 else 0x7B
    assert q[n - 1] == top
    ref = (_bf16_to_f32(x) * (torch.tensor(FMAX[fmt]) / 1000.0)).to(TORCH_DT[fmt])
    assert np.array_equal(q, ref.view(torch.uint8).numpy())


def test_group_scaling_takes_the_producers_maxima(orc):
    """With maxima supplied (a producer filled the intermediate), step (i) is
    skipped: the scale comes from the given values even where they differ
    from the tensor's own maxima (here one entry doubled)."""
    G = 128
    x = inputs.host_activations(inputs.activations(seed=4), rows=4).reshape(-1)
    _, s0, ga = orc.group_scaling_pertensor(x, G, E4M3)
    given = ga.copy()
    i = int(np.argmax(given))
    given[i] = 2.0 * given[i]
    q, s, ga_out = orc.group_scaling_pertensor(x, G, E4M3, group_amax=given)
    assert np.array_equal(ga_out, given)
    amax = torch.tensor(float(given[i]), dtype=torch.float32)
    assert s == (amax / torch.tensor(448.0)).item() and s == 2.0 * s0
    ref = (_bf16_to_f32(x) * (torch.tensor(448.0) / amax)).to(torch.float8_e4m3fn)
    assert np.array_equal(q, ref.view(torch.uint8).numpy())


@pytest.mark.parametrize("fmt", [E4M3, E5M2])
def test_activation_dequant(orc, fmt):
    w = inputs.activations()
    x = inputs.host_activations(w, rows=8)
    q, sc = orc.group_quant_1xG(x, 128, fmt)
    out = orc.dequant(q.reshape(-1), None, sc.reshape(-1), 128, fmt)
    ref = (torch.from_numpy(q.reshape(-1)).view(TORCH_DT[fmt]).float().reshape(-1, 128)
           * torch.from_numpy(sc.reshape(-1))[:, None]).reshape(-1).numpy()
    assert np.array_equal(out, ref)
    # and it reconstructs the input within half an FP8 step of each group's scale
    xf = _bf16_to_f32(x).reshape(-1).numpy()
    assert np.max(np.abs(out - xf) / np.maximum(np.abs(xf), 1e-3)) < 0.13
