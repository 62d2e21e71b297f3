"""GPU parity at the full workload sizes, in the launch configuration the
bench times: the OLMo-7B set (6,888,095,744 parameters) and the OLMo-1B set
(1,176,764,416, second moment in E5M2), built on the device exactly as
bench.py builds them and stepped by one coat_adamw_fp8_step call over the
whole flat buffer.

The oracle cannot take billions of parameters, but the 1xG groups of the
step are independent: the test copies a seeded sample of groups (the first
and last ones, those at tensor boundaries and a few thousand at random)
before the step, runs the oracle on them, and compares the GPU's outputs for
exactly those groups under the usual tolerances.  Over every group it also
checks properties that hold at any size: the group maximum of each state
encodes to the format's largest code (or the group is all zero with scale
0), no code is an inf/NaN code, and k, s and theta are finite."""
import numpy as np
import pytest

import parity
from quantized_optimizer_states_b200 import inputs

pytestmark = pytest.mark.gpu

E4M3, E5M2 = 0, 1
MAX_CODE = {E4M3: 0x7E, E5M2: 0x7B}
RANDOM_GROUPS = 4096


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


def _device_state(lib, w, v_fmt, dev):
    """theta, grad and quantized states on the device (the bench's recipe)."""
    import torch
    n, G = w.n, w.group_size
    ng = -(-n // G)
    theta, grad, chunks = inputs.device_step_inputs(w, dev)
    st = {"theta": theta, "grad": grad,
          "mc": torch.empty(n, dtype=torch.uint8, device=dev),
          "vc": torch.empty(n, dtype=torch.uint8, device=dev)}
    for k in ("mk", "ms", "vk", "vs"):
        st[k] = torch.empty(ng, dtype=torch.float32, device=dev)
    for off, m0, v0 in chunks():
        c = m0.numel()
        g0, g1 = off // G, -(-(off + c) // G)
        lib.coat_quantize_state(m0, st["mc"][off:off + c], st["mk"][g0:g1], st["ms"][g0:g1],
                                group_size=G, fmt=E4M3)
        lib.coat_quantize_state(v0, st["vc"][off:off + c], st["vk"][g0:g1], st["vs"][g0:g1],
                                group_size=G, fmt=v_fmt)
    torch.cuda.synchronize()
    return st


def _sample_groups(w):
    G = w.group_size
    ng = -(-w.n // G)
    rng = np.random.default_rng(w.seed + 31)
    picks = [0, 1, 2, ng - 3, ng - 2, ng - 1]
    off = 0
    for sz in (w.sizes or [w.n]):   # groups on both sides of every tensor boundary
        if 0 < off < w.n:
            picks += [off // G - 1, off // G]
        off += sz
    picks += list(rng.integers(0, ng, RANDOM_GROUPS))
    return np.unique(np.array(picks, dtype=np.int64))


def _gather(st, groups, G):
    import torch
    dev = st["theta"].device
    g = torch.from_numpy(groups).to(dev)
    idx = (g[:, None] * G + torch.arange(G, device=dev)[None, :]).reshape(-1)
    out = {k: st[k][idx].cpu().numpy() for k in ("theta", "mc", "vc")}
    out["grad"] = st["grad"][idx].view(torch.int16).cpu().numpy().view(np.uint16)
    for k in ("mk", "ms", "vk", "vs"):
        out[k] = st[k][g].cpu().numpy()
    return out


def _check_every_group(st, G, v_fmt, chunk_groups=1 << 21):
    """Properties of the step's outputs that hold for every group."""
    import torch
    ng = st["mk"].numel()
    for code, k, s, fmt in (("mc", "mk", "ms", E4M3), ("vc", "vk", "vs", v_fmt)):
        kk, ss = st[k], st[s]
        assert bool(torch.isfinite(kk).all()) and bool(torch.isfinite(ss).all()), k
        assert bool((ss >= 0).all()), s
        for g0 in range(0, ng, chunk_groups):
            g1 = min(ng, g0 + chunk_groups)
            c = st[code][g0 * G:g1 * G].view(g1 - g0, G)
            mag = c & 0x7F
            gmax = mag.max(dim=1).values
            zero = ss[g0:g1] == 0
            # every nonzero group reaches the format's largest finite code ...
            assert bool(((gmax == MAX_CODE[fmt]) | zero).all()), (code, g0)
            # ... an all-zero group is all code 0, and no code is inf/NaN
            assert bool((gmax[zero] == 0).all()), (code, g0)
            assert bool((mag <= MAX_CODE[fmt]).all()), (code, g0)
    n = st["theta"].numel()
    for off in range(0, n, chunk_groups * G):
        assert bool(torch.isfinite(st["theta"][off:off + chunk_groups * G]).all())


@pytest.mark.parametrize("name,v_fmt,f32_grads", [("olmo-1b", E5M2, False), ("olmo-7b", E4M3, False),
                                                  ("olmo-7b", E5M2, False),
                                                  ("olmo-7b", E4M3, True)])
def test_full_size_sampled_groups(lib, orc, name, v_fmt, f32_grads):
    """f32_grads: the same BF16 gradients widened to float32 (exactly) and
    stepped through the float32-gradient form, which rounds them back."""
    import torch
    if name == "olmo-7b":
        w = inputs.olmo_7b(v_fmt="e4m3" if v_fmt == E4M3 else "e5m2")
    else:
        w = inputs.olmo_1b()
    need = int(w.n * (8 + 32 / w.group_size + (4 if f32_grads else 0))) + (4 << 30)
    free, _ = torch.cuda.mem_get_info()
    if free < need:
        pytest.skip(f"needs {need / 2**30:.0f} GiB of free device memory")
    dev = torch.device("cuda", torch.cuda.current_device())
    G = w.group_size
    st = _device_state(lib, w, v_fmt, dev)
    groups = _sample_groups(w)
    before = _gather(st, groups, G)
    grad = st["grad"]
    if f32_grads:
        grad = torch.empty(w.n, dtype=torch.float32, device=dev)
        for off in range(0, w.n, 1 << 28):
            grad[off:off + (1 << 28)].copy_(st["grad"][off:off + (1 << 28)])
    lib.coat_adamw_fp8_step(st["theta"], grad, st["mc"], st["mk"], st["ms"], st["vc"],
                            st["vk"], st["vs"], step=w.step, group_size=G, v_fmt=v_fmt,
                            **w.hyper)
    del grad
    torch.cuda.synchronize()
    after = _gather(st, groups, G)
    _check_every_group(st, G, v_fmt)
    del st
    torch.cuda.empty_cache()

    ref = orc.adamw_fp8_step(before["theta"], before["grad"], before["mc"], before["mk"],
                             before["ms"], before["vc"], before["vk"], before["vs"],
                             step=w.step, group_size=G, v_fmt=v_fmt, return_moments=True,
                             **w.hyper)
    got = tuple(after[k] for k in ("theta", "mc", "mk", "ms", "vc", "vk", "vs"))
    stats = parity.assert_step_parity(got, ref, w.hyper["lr"], G, v_fmt,
                                      moments=(ref[7], ref[8]))
    print(f"{name} v_fmt={v_fmt} f32_grads={f32_grads}: {groups.size} groups sampled, {stats}")
