"""Non-finite gradients: coat_count_nonfinite_bf16, the guarded step (a
no-op decided on the device) and CoatAdamW(skip_nonfinite=True)."""
import numpy as np
import pytest
import torch

import parity
from quantized_optimizer_states_b200 import inputs

pytestmark = pytest.mark.gpu
H = inputs.HYPER
G = 128


@pytest.fixture(scope="module")
def lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from quantized_optimizer_states_b200 import build
    build.build()
    import quantized_optimizer_states_b200 as q
    q.load()
    return q


def test_count_matches_numpy(lib, orc):
    rng = np.random.default_rng(5)
    n = 3 * 8192 + 37
    g = orc.to_bf16_array(rng.normal(0, 1e-3, n).astype(np.float32))
    idx = rng.choice(n, 41, replace=False)
    g[idx[:20]] = 0x7F80            # +inf
    g[idx[20:30]] = 0xFF80          # -inf
    g[idx[30:]] = 0x7FC1            # NaN
    count = torch.zeros(1, dtype=torch.int32, device="cuda")
    lib.coat_count_nonfinite_bf16(parity.to_dev(g, torch.int16), count)
    lib.coat_count_nonfinite_bf16(parity.to_dev(g[:100], torch.int16), count)  # accumulates
    want = 41 + int(np.sum((g[:100] & 0x7F80) == 0x7F80))
    assert int(count.item()) == want


def _states(orc, n, seed):
    x = inputs.host_step_inputs(inputs.tiny(seed), n)
    mc, mk, ms = orc.quantize_state(x["m0"], G, 0)
    vc, vk, vs = orc.quantize_state(x["v0"], G, 0)
    d = [parity.to_dev(a) for a in (x["theta"], mc, mk, ms, vc, vk, vs)]
    return x, d


def test_guarded_step_runs_or_skips(lib, orc):
    n = 2 * 4096 + 300
    x, d = _states(orc, n, 71)
    g = parity.to_dev(x["grad"], torch.int16)
    e = [t.clone() for t in d]
    word = torch.zeros(1, dtype=torch.int32, device="cuda")
    lib.coat_adamw_fp8_step(*d[:1], g, *d[1:], step=10, group_size=G, **H)
    lib.coat_adamw_fp8_step(*e[:1], g, *e[1:], step=10, group_size=G, skip_if_nonzero=word, **H)
    torch.cuda.synchronize()
    for a, b in zip(d, e):
        assert torch.equal(a, b)        # word == 0: the plain step
    before = [t.clone() for t in e]
    word.fill_(3)
    lib.coat_adamw_fp8_step(*e[:1], g, *e[1:], step=11, group_size=G, skip_if_nonzero=word, **H)
    torch.cuda.synchronize()
    for a, b in zip(before, e):
        assert torch.equal(a, b)        # word != 0: nothing written


def test_optimizer_skips_nonfinite_steps(lib):
    from quantized_optimizer_states_b200.optim import CoatAdamW
    gen = torch.Generator().manual_seed(8)
    p = torch.nn.Parameter((torch.randn(3000, generator=gen) * 0.02).cuda())
    opt = CoatAdamW([p], lr=H["lr"], betas=(H["beta1"], H["beta2"]), eps=H["eps"],
                    weight_decay=H["weight_decay"], skip_nonfinite=True)
    p.grad = (torch.randn(3000, generator=gen) * 1e-3).cuda()
    opt.step()
    snap = p.detach().clone()
    p.grad[17] = float("nan")
    opt.step()
    assert torch.equal(p.detach(), snap) and opt.skipped_steps == 1 and opt._flat[0].step == 1
    p.grad[17] = 1e-3
    opt.step()
    assert not torch.equal(p.detach(), snap) and opt._flat[0].step == 2


def _guarded_raw(lib, x, g, c, m, skip_ptr):
    import ctypes
    from quantized_optimizer_states_b200._lib import CoatAdamwCfg, _check, load
    cfg = CoatAdamwCfg(0.9, 0.999, 1e-4, 1e-8, 0.1, 1, G, 0, 0, 0, 64.0, 0)
    P = ctypes.c_void_p
    st = load().coat_adamw_fp8_step_guarded(
        P(x.data_ptr()), P(g.data_ptr()), P(c.data_ptr()), P(m.data_ptr()), P(m.data_ptr()),
        P(c.data_ptr()), P(m.data_ptr()), P(m.data_ptr()), x.numel(), ctypes.byref(cfg),
        skip_ptr, None)
    _check("coat_adamw_fp8_step_guarded", st)


def test_guarded_argument_errors(lib):
    import ctypes
    from quantized_optimizer_states_b200._lib import CoatError
    x = torch.zeros(128, device="cuda")
    g = torch.zeros(128, dtype=torch.int16, device="cuda")
    c = torch.zeros(128, dtype=torch.uint8, device="cuda")
    m = torch.ones(1, device="cuda")
    word = torch.zeros(2, dtype=torch.int32, device="cuda")
    with pytest.raises(CoatError) as e:          # not 4-byte aligned
        _guarded_raw(lib, x, g, c, m, ctypes.c_void_p(word.data_ptr() + 2))
    assert e.value.status == 2
    with pytest.raises(CoatError) as e:          # null
        _guarded_raw(lib, x, g, c, m, None)
    assert e.value.status == 1
