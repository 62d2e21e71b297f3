"""Host-side control flow of CoatAdamW (CPU only): which library calls a
step makes, in which order and with which arguments -- packed BF16
gradients, flat FP32 gradients, BF16 parameters with write-back, the
non-finite skip, parameter groups added later, and a checkpoint round trip.
The module is loaded from its source with the CUDA-device check removed and
the library calls replaced by recorders (a visible update stands in for the
kernel), so plain CPU tensors can drive it; the kernels themselves are the
GPU tests' business."""
import contextlib
import os
import sys
import types

import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _load_cpu_optim(monkeypatch):
    from quantized_optimizer_states_b200 import _lib
    with open(os.path.join(ROOT, "quantized_optimizer_states_b200", "optim.py")) as f:
        src = f.read()
    assert src.count('if dev.type != "cuda":') == 1
    src = src.replace('if dev.type != "cuda":', "if False:")
    src = src.replace("from . import _lib", "from quantized_optimizer_states_b200 import _lib")
    mod = types.ModuleType("optim_on_cpu")
    monkeypatch.setitem(sys.modules, "optim_on_cpu", mod)
    exec(compile(src, "optim_on_cpu", "exec"), mod.__dict__)
    calls = []

    class Tab:
        def __init__(self, numel, off):
            self.numel, self.off = numel, off

    def pack(grads, table, dst, **k):
        calls.append(("pack", len(grads)))
        for g, off in zip(grads, table.off):
            if g is not None:
                dst[off:off + g.numel()] = g.reshape(-1).to(dst.dtype)

    def unpack(src, table, dsts, **k):
        calls.append(("unpack", len(dsts)))
        for d, off in zip(dsts, table.off):
            d.copy_(src[off:off + d.numel()].view_as(d).to(d.dtype))

    def step(master, grad, *a, **k):
        calls.append(("step", grad.dtype, k["step"], k["v_fmt"], k["group_size"]))
        master -= 1.0

    def count(g, c, **k):
        calls.append(("count",))
        c += int((~torch.isfinite(g.float())).sum())

    monkeypatch.setattr(torch.cuda, "device", lambda d: contextlib.nullcontext())
    monkeypatch.setattr(_lib, "PackTable", Tab)
    monkeypatch.setattr(_lib, "coat_pack_bf16", pack)
    monkeypatch.setattr(_lib, "coat_unpack_bf16", unpack)
    monkeypatch.setattr(_lib, "coat_adamw_fp8_step", step)
    monkeypatch.setattr(_lib, "coat_count_nonfinite_bf16", count)
    return mod.CoatAdamW, calls


def test_step_control_flow(monkeypatch):
    A, calls = _load_cpu_optim(monkeypatch)

    # FP32 params, packed gradients
    p = torch.nn.Parameter(torch.zeros(300))
    opt = A([p], lr=1e-3, group_size=128)
    p.grad = torch.ones(300)
    opt.step()
    assert calls == [("pack", 1), ("step", torch.bfloat16, 1, 0, 128)], calls
    assert torch.all(p.detach() == -1.0)
    # flat grads: no pack, float32 gradients straight to the step
    calls.clear()
    q = torch.nn.Parameter(torch.zeros(100))
    opt2 = A([q], flat_grads=True, v_fmt="e5m2", group_size=64)
    q.grad.add_(0.5)
    opt2.step()
    opt2.step()
    assert calls == [("step", torch.float32, 1, 1, 64), ("step", torch.float32, 2, 1, 64)], calls
    opt2.zero_grad()
    assert q.grad is not None and float(q.grad.abs().sum()) == 0.0
    # BF16 params: pack, step, write back
    calls.clear()
    b = torch.nn.Parameter(torch.zeros(40, dtype=torch.bfloat16))
    opt3 = A([b])
    b.grad = torch.ones(40, dtype=torch.bfloat16)
    opt3.step()
    assert calls == [("pack", 1), ("step", torch.bfloat16, 1, 0, 128), ("unpack", 1)], calls
    assert torch.all(b.detach().float() == -1.0)
    # skip_nonfinite: a NaN skips the step and the counter does not advance
    calls.clear()
    r = torch.nn.Parameter(torch.zeros(20))
    opt4 = A([r], skip_nonfinite=True)
    g = torch.zeros(20); g[3] = float("nan"); r.grad = g
    opt4.step()
    assert calls == [("pack", 1), ("count",)] and opt4.skipped_steps == 1 and opt4._flat[0].step == 0
    r.grad = torch.zeros(20)
    opt4.step()
    assert calls[-1][0] == "step" and calls[-1][2] == 1
    # a group added later is stepped too
    calls.clear()
    s1, s2 = torch.nn.Parameter(torch.zeros(16)), torch.nn.Parameter(torch.zeros(32))
    opt5 = A([s1])
    opt5.add_param_group({"params": [s2], "lr": 1e-4, "v_fmt": "e5m2"})
    s1.grad, s2.grad = torch.ones(16), torch.ones(32)
    opt5.step()
    assert [c[0] for c in calls] == ["pack", "step", "pack", "step"] and calls[-1][3] == 1, calls
    assert torch.all(s2.detach() == -1.0)
    # checkpoint round trip keeps the per-group step and the flat state
    calls.clear()
    c1 = torch.nn.Parameter(torch.zeros(64, dtype=torch.bfloat16))
    o1 = A([c1], group_size=64)
    c1.grad = torch.ones(64, dtype=torch.bfloat16)
    o1.step(); o1.step()
    sd = o1.state_dict()
    c2 = torch.nn.Parameter(torch.zeros(64, dtype=torch.bfloat16))
    o2 = A([c2], group_size=64)
    o2.load_state_dict(sd)
    assert o2._flat[0].step == 2 and torch.equal(o2._flat[0].master, o1._flat[0].master)
    assert torch.all(c2.detach().float() == -2.0)          # written back from the master
    c2.grad = torch.ones(64, dtype=torch.bfloat16)
    o2.step()
    assert [c for c in calls if c[0] == "step"][-1][2] == 3      # the counter continues
    assert calls[-1] == ("unpack", 1)
