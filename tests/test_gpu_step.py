"""GPU parity of the fused COAT AdamW step and the state quantizer against
the oracle, through the C ABI (libcoat.so)."""
import numpy as np
import pytest

import parity
from quantized_optimizer_states_b200 import inputs

pytestmark = pytest.mark.gpu

E4M3, E5M2 = 0, 1
H = inputs.HYPER


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


def _init_states(orc, x, G, v_fmt, k_range=0, k_max=64.0):
    mc, mk, ms = orc.quantize_state(x["m0"], G, E4M3, k_range=k_range, k_max=k_max)
    vc, vk, vs = orc.quantize_state(x["v0"], G, v_fmt, k_range=k_range, k_max=k_max)
    return mc, mk, ms, vc, vk, vs


def _one_step(lib, orc, x, st, *, t, G, v_fmt, k_range=0, k_max=64.0, force_k1=False):
    th = x["theta"]
    cfg = dict(step=t, group_size=G, v_fmt=v_fmt, k_range=k_range, k_max=k_max, **H)
    ref = orc.adamw_fp8_step(th, x["grad"], *st, force_k1=force_k1, return_moments=True, **cfg)
    got = parity.gpu_step(lib, th, x["grad"], *st, flags=lib.COAT_FORCE_K1 if force_k1 else 0,
                          **cfg)
    stats = parity.assert_step_parity(got, ref, H["lr"], G, v_fmt, moments=(ref[7], ref[8]))
    return ref, stats


def test_tiny_three_steps(lib, orc):
    """Tiny workload: 2^20 parameters, G = 128, E4M3 + E4M3, t = 10, 11, 12.
    Each step starts both sides from the oracle's state."""
    w = inputs.tiny()
    x = inputs.host_step_inputs(w)
    st = _init_states(orc, x, 128, E4M3)
    rng = np.random.default_rng(5)
    for t in (10, 11, 12):
        ref, stats = _one_step(lib, orc, x, st, t=t, G=128, v_fmt=E4M3)
        print(f"t={t}", stats)
        x = dict(x, theta=ref[0])
        st = ref[1:7]
        # next step's gradient
        g = (rng.normal(0, 1e-3, w.n)).astype(np.float32)
        x["grad"] = orc.to_bf16_array(g)


@pytest.mark.parametrize("G", [16, 32, 64, 128, 256, 512, 1024, 2048, 4096])
@pytest.mark.parametrize("v_fmt", [E4M3, E5M2])
def test_group_sizes_ragged(lib, orc, G, v_fmt):
    """All group sizes on a size that is neither a multiple of G nor of 16."""
    n = 40 * 4096 + 2 * G + 7
    x = inputs.host_step_inputs(inputs.olmo_1b(), n)
    st = _init_states(orc, x, G, v_fmt)
    _one_step(lib, orc, x, st, t=10, G=G, v_fmt=v_fmt)


@pytest.mark.parametrize("regime", ["early", "late", "typical"])
@pytest.mark.parametrize("v_fmt", [E4M3, E5M2])
def test_regimes(lib, orc, regime, v_fmt):
    w = inputs.sweep(128, "e4m3", regime)
    x = inputs.host_step_inputs(w, 1 << 18)
    st = _init_states(orc, x, 128, v_fmt)
    _one_step(lib, orc, x, st, t=10, G=128, v_fmt=v_fmt)


@pytest.mark.parametrize("variant", ["k_range1", "force_k1", "no_clamp", "t1"])
def test_variants(lib, orc, variant):
    x = inputs.host_step_inputs(inputs.tiny(31), 1 << 17)
    kw = dict(G=128, v_fmt=E5M2, t=10)
    if variant == "k_range1":
        kw.update(k_range=1)
    elif variant == "force_k1":
        kw.update(force_k1=True)
    elif variant == "no_clamp":
        kw.update(k_max=0.0)
    elif variant == "t1":
        kw.update(t=1)
    st = _init_states(orc, x, 128, E5M2, k_range=kw.get("k_range", 0),
                      k_max=kw.get("k_max", 64.0))
    _one_step(lib, orc, x, st, **kw)


@pytest.mark.parametrize("v_fmt", [E4M3, E5M2])
def test_fp32_gradients_round_to_bf16(lib, orc, v_fmt):
    """coat_adamw_fp8_step_fp32grad: float32 gradients rounded to BF16 on
    load give the oracle's step on the rounded gradients (and the BF16
    entry point's bits), ragged size included."""
    import torch
    G, n = 128, 3 * 4096 + 1000 + 37
    x = inputs.host_step_inputs(inputs.olmo_1b(), n)
    rng = np.random.default_rng(11)
    g32 = (rng.standard_normal(n) * 1e-3).astype(np.float32)
    g32[:3] = [0.0, -0.0, 3.0e-39]                      # zeros and a subnormal
    gb = orc.to_bf16_array(g32)
    st = _init_states(orc, x, G, v_fmt)
    cfg = dict(step=10, group_size=G, v_fmt=v_fmt, **H)
    ref = orc.adamw_fp8_step(x["theta"], gb, *st, return_moments=True, **cfg)
    d = [parity.to_dev(x["theta"]), parity.to_dev(g32)] + [parity.to_dev(a) for a in st]
    lib.coat_adamw_fp8_step(*d, **cfg)
    torch.cuda.synchronize()
    got = tuple(parity.to_host(t) for t in (d[0], d[2], d[3], d[4], d[5], d[6], d[7]))
    parity.assert_step_parity(got, ref, H["lr"], G, v_fmt, moments=(ref[7], ref[8]))
    same = parity.gpu_step(lib, x["theta"], gb, *st, **cfg)
    for a, b in zip(got, same):
        assert np.array_equal(a, b)


def test_degenerate_groups(lib, orc):
    """All-zero, all-equal, single-nonzero, zero-gradient groups and a tail
    group of one element."""
    G = 64
    n = 10 * G + 1
    x = inputs.host_step_inputs(inputs.tiny(41), n)
    # group 0: zero state and zero gradient -> stays an all-zero group
    x["m0"][:G] = 0
    x["v0"][:G] = 0
    x["grad"][:G] = 0
    # group 1: all-equal magnitudes in m and v, zero grad keeps them equal-ish
    x["m0"][G:2 * G] = np.where(np.arange(G) % 2, 1e-4, -1e-4).astype(np.float32)
    x["v0"][G:2 * G] = 3e-8
    x["grad"][G:2 * G] = 0
    # group 2: a single nonzero element
    x["m0"][2 * G:3 * G] = 0
    x["m0"][2 * G + 5] = 2e-4
    x["v0"][2 * G:3 * G] = 0
    x["v0"][2 * G + 5] = 4e-8
    x["grad"][2 * G:3 * G] = 0
    st = _init_states(orc, x, G, E4M3)
    ref, _ = _one_step(lib, orc, x, st, t=10, G=G, v_fmt=E4M3)
    assert ref[2][0] == 1.0 and ref[3][0] == 0.0          # all-zero group: k = 1, s = 0
    assert ref[2][1] == 1.0                                # all-equal group: k = 1


def test_tiny_sizes(lib, orc):
    for n in (1, 5, 15, 16, 17, 127, 129):
        x = inputs.host_step_inputs(inputs.tiny(n), n)
        st = _init_states(orc, x, 16, E4M3)
        _one_step(lib, orc, x, st, t=10, G=16, v_fmt=E4M3)


def test_quantize_state_parity(lib, orc):
    import torch
    for G, fmt, dist in ((128, E4M3, "m"), (128, E5M2, "v"), (32, E4M3, "v"), (1024, E5M2, "m")):
        x = inputs.host_step_inputs(inputs.tiny(51), 300_001)["m0" if dist == "m" else "v0"]
        ref = orc.quantize_state(x, G, fmt)
        xd = parity.to_dev(x)
        n = x.size
        code = torch.empty(n, dtype=torch.uint8, device="cuda")
        k = torch.empty(orc.n_groups(n, G), dtype=torch.float32, device="cuda")
        s = torch.empty_like(k)
        lib.coat_quantize_state(xd, code, k, s, group_size=G, fmt=fmt)
        torch.cuda.synchronize()
        parity.compare_rel("k", parity.to_host(k), ref[1], parity.KS_RTOL)
        parity.compare_rel("s", parity.to_host(s), ref[2], parity.KS_RTOL)
        parity.compare_codes("code", parity.to_host(code), ref[0],
                             parity.tie_checker(x, ref[1], G, fmt))


def test_state_dequant_parity(lib, orc):
    import torch
    G = 128
    x = inputs.host_step_inputs(inputs.tiny(61), 200_003)
    for fmt, xs in ((E4M3, x["m0"]), (E5M2, x["v0"])):
        c, k, s = orc.quantize_state(xs, G, fmt)
        ref = orc.dequant(c, k, s, G, fmt)
        out = torch.empty(xs.size, dtype=torch.float32, device="cuda")
        lib.coat_dequant(parity.to_dev(c), parity.to_dev(k), parity.to_dev(s), out,
                         group_size=G, fmt=fmt)
        torch.cuda.synchronize()
        got = parity.to_host(out)
        # correctly rounded powers: identical except in vanishingly rare
        # double-rounding cases, which may differ by one unit in the last place
        parity.compare_rel("dequant", got, ref, 2.0 ** -23)
        assert np.count_nonzero(got != ref) <= 1e-5 * got.size


def test_deterministic_and_guarded(lib, orc):
    """Two runs give identical bytes; nothing is written past the buffers."""
    import torch
    G, n = 128, 100_003
    x = inputs.host_step_inputs(inputs.tiny(71), n)
    st = _init_states(orc, x, G, E4M3)
    outs = []
    for _ in range(2):
        pad = 4096
        bufs = []
        for a in (x["theta"], x["grad"], *st):
            a = np.ascontiguousarray(a)
            raw = torch.full((a.nbytes + 2 * pad,), 0xA5, dtype=torch.uint8, device="cuda")
            raw[pad:pad + a.nbytes].copy_(torch.from_numpy(a.view(np.uint8)).cuda())
            bufs.append((raw, a))
        views = [raw[pad:pad + a.nbytes].view(
            {np.float32: torch.float32, np.uint16: torch.int16, np.uint8: torch.uint8}[a.dtype.type])
            for raw, a in bufs]
        lib.coat_adamw_fp8_step(*views, step=10, group_size=G, **H)
        torch.cuda.synchronize()
        for raw, a in bufs:
            assert torch.all(raw[:pad] == 0xA5) and torch.all(raw[pad + a.nbytes:] == 0xA5)
        outs.append([parity.to_host(v).tobytes() for v in views])
    assert outs[0] == outs[1]


def test_argument_errors(lib):
    import torch
    n = 1024
    th = torch.zeros(n + 4, dtype=torch.float32, device="cuda")
    g = torch.zeros(n, dtype=torch.int16, device="cuda")
    mc = torch.zeros(n, dtype=torch.uint8, device="cuda")
    meta = [torch.ones(8, dtype=torch.float32, device="cuda") for _ in range(4)]
    vc = torch.zeros(n, dtype=torch.uint8, device="cuda")
    base = dict(step=10, **H)
    with pytest.raises(lib.CoatError) as e:
        lib.coat_adamw_fp8_step(th[1:n + 1], g, mc, meta[0], meta[1], vc, meta[2], meta[3],
                                group_size=128, **base)
    assert e.value.status == 2
    with pytest.raises(lib.CoatError) as e:
        lib.coat_adamw_fp8_step(th[:n], g, mc, meta[0], meta[1], vc, meta[2], meta[3],
                                group_size=96, **base)
    assert e.value.status == 3
    with pytest.raises(lib.CoatError) as e:
        lib.coat_adamw_fp8_step(th[:n], g, mc, meta[0], meta[1], vc, meta[2], meta[3],
                                group_size=128, v_fmt=7, **base)
    assert e.value.status == 3
    bad = dict(base, step=0)
    with pytest.raises(lib.CoatError) as e:
        lib.coat_adamw_fp8_step(th[:n], g, mc, meta[0], meta[1], vc, meta[2], meta[3],
                                group_size=128, **bad)
    assert e.value.status == 1
    # an empty step is valid and launches nothing
    e0 = torch.empty(0, dtype=torch.float32, device="cuda")
    lib.coat_adamw_fp8_step(e0, g[:0], mc[:0], meta[0], meta[1], vc[:0], meta[2], meta[3],
                            group_size=128, **base)


def _step_cfg(orc, lib, x, st, *, G, t, v_fmt, hyper):
    cfg = dict(step=t, group_size=G, v_fmt=v_fmt, k_range=0, k_max=64.0, **hyper)
    ref = orc.adamw_fp8_step(x["theta"], x["grad"], *st, return_moments=True, **cfg)
    got = parity.gpu_step(lib, x["theta"], x["grad"], *st, flags=0, **cfg)
    return parity.assert_step_parity(got, ref, hyper["lr"], G, v_fmt,
                                     moments=(ref[7], ref[8]))


def test_exact_path_when_the_estimates_are_disabled(lib, orc):
    """eps = 0 leaves the estimate-based quotient's range: every warp takes
    the fully IEEE path."""
    x = inputs.host_step_inputs(inputs.tiny(61), 3 * 4096 + 100)
    st = _init_states(orc, x, 128, E4M3)
    _step_cfg(orc, lib, x, st, G=128, t=10, v_fmt=E4M3, hyper=dict(H, eps=0.0))


def test_exact_path_for_out_of_range_moments(lib, orc):
    """A group whose second moment is tiny (v_t < 2^-120 with a zero
    gradient) and one whose gradients are huge (v_t far above the estimates'
    range) make their warps rewrite theta with the IEEE operations; the
    other warps keep the estimate-based result.  All against the oracle."""
    G = 128
    n = 8 * 4096
    x = inputs.host_step_inputs(inputs.tiny(62), n)
    x["v0"][3 * G:4 * G] = 1e-38
    x["grad"][3 * G:4 * G] = 0
    big = orc.to_bf16_array(np.full(G, 1e19, dtype=np.float32))
    x["grad"][9 * G:10 * G] = big
    x["grad"][9 * G + 1:10 * G:2] ^= 0x8000          # alternate signs
    st = _init_states(orc, x, G, E4M3)
    _step_cfg(orc, lib, x, st, G=G, t=10, v_fmt=E4M3, hyper=H)


@pytest.mark.parametrize("G", [128, 1024])
def test_group_parameters_special_cases(lib, orc, G):
    """Branch-free k and s on all-equal groups (k = 1, s = M / fmax), a
    group whose range would exceed k_max (clamped) and ordinary groups,
    with v in E5M2."""
    n = 6 * G
    x = inputs.host_step_inputs(inputs.tiny(63), n)
    x["m0"][:G] = 3e-4
    x["v0"][:G] = 5e-8
    x["grad"][:G] = 0
    x["m0"][G:2 * G] = np.where(np.arange(G) % 2, 1e-4, 1.0001e-4).astype(np.float32)
    x["v0"][G:2 * G] = np.where(np.arange(G) % 2, 2e-8, 2.00001e-8).astype(np.float32)
    x["grad"][G:2 * G] = 0
    st = _init_states(orc, x, G, E5M2)
    _step_cfg(orc, lib, x, st, G=G, t=10, v_fmt=E5M2, hyper=H)
