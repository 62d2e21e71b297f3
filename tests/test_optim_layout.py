"""Host logic of the CoatAdamW wrapper: the padded flat layout (no GPU)."""
import pytest
import torch

from quantized_optimizer_states_b200.optim import CoatAdamW, padded_layout


def test_padded_layout_offsets_are_group_aligned():
    offs, n = padded_layout([5, 128, 129, 0, 300], 128)
    assert offs == [0, 128, 256, 512, 512]
    assert n == 512 + 384
    for o in offs:
        assert o % 128 == 0


def test_padded_layout_small_groups_keep_16_byte_alignment():
    # G = 16 pads to 16 elements: 16 codes / 32 B of BF16 / 64 B of FP32
    offs, n = padded_layout([1, 17, 16], 16)
    assert offs == [0, 16, 48] and n == 64


def test_padded_layout_rejects_bad_input():
    with pytest.raises(ValueError):
        padded_layout([4], 0)
    with pytest.raises(ValueError):
        padded_layout([-1], 128)


def test_cpu_parameters_are_rejected():
    with pytest.raises(ValueError):
        CoatAdamW([torch.nn.Parameter(torch.zeros(4))])


def test_bad_hyperparameters_are_rejected():
    p = [torch.nn.Parameter(torch.zeros(4))]
    with pytest.raises(ValueError):
        CoatAdamW(p, betas=(1.0, 0.9))
    with pytest.raises(ValueError):
        CoatAdamW(p, v_fmt="e3m4")


@pytest.mark.parametrize("kw", [dict(group_size=96), dict(group_size=8), dict(group_size=8192),
                                dict(group_size=128.0), dict(k_range=2),
                                dict(k_max=-1.0), dict(k_max=float("nan"))])
def test_unsupported_group_size_and_expansion_settings_are_rejected(kw):
    # rejected when the optimizer is made, not at its first step (the check
    # runs before the parameters' device is looked at, so CPU tensors do)
    with pytest.raises(ValueError, match="group_size|k_range|k_max"):
        CoatAdamW([torch.nn.Parameter(torch.zeros(4))], **kw)
