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


def test_groups_added_later_get_their_flat_buffers(monkeypatch):
    """A parameter group added after construction is built at once (step()
    walks one flat group per parameter group); its COAT settings are
    checked and normalised first, and a group that cannot be built (or has
    bad settings) is not added.  _build is replaced so that CPU tensors do."""
    built = []

    def fake_build(self, group):
        if group["params"][0].numel() == 3:
            raise ValueError("cannot build")
        built.append(dict(group))
        return object()

    monkeypatch.setattr(CoatAdamW, "_build", fake_build)
    p1, p2 = torch.nn.Parameter(torch.zeros(4)), torch.nn.Parameter(torch.zeros(8))
    opt = CoatAdamW([p1], lr=1e-3)
    assert len(opt._flat) == 1 and len(built) == 1
    opt.add_param_group({"params": [p2], "lr": 1e-4, "v_fmt": "e5m2", "group_size": 64})
    assert len(opt._flat) == len(opt.param_groups) == 2
    assert built[-1]["lr"] == 1e-4 and built[-1]["v_fmt"] == 1 and built[-1]["group_size"] == 64
    assert built[-1]["betas"] == (0.9, 0.999)                  # defaults filled in
    for bad in ({"v_fmt": "e3m4"}, {"group_size": 100}, {"k_range": 3}, {"k_max": -2.0}):
        with pytest.raises(ValueError):
            opt.add_param_group({"params": [torch.nn.Parameter(torch.zeros(2))], **bad})
    with pytest.raises(ValueError, match="cannot build"):
        opt.add_param_group({"params": [torch.nn.Parameter(torch.zeros(3))]})
    assert len(opt._flat) == len(opt.param_groups) == 2
