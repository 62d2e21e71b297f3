"""GPU: coat_state_stats against the oracle's definitions, on the hand-built
state of the oracle pin, on states quantized by the library (both formats,
ragged length), and through CoatAdamW.state_stats after real steps."""
import numpy as np
import pytest

import parity

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


def _same(got, want):
    for key, w in want.items():
        if key == "k_sum":
            assert abs(got[key] - w) <= 1e-12 * max(abs(w), 1.0), key
        else:
            assert got[key] == w, (key, got[key], w)


def test_hand_built_state(lib, orc):
    code = np.array([0, 0, 0, 0, 0x7E, 0x01, 0x80, 0xFE, 0x7F, 0x7E, 0x00, 0x33, 0x7E, 0x10],
                    dtype=np.uint8)
    buf = np.zeros(16, np.uint8)
    buf[:14] = code
    k = np.array([1.0, 2.0, 1.0, 3.5], dtype=np.float32)
    s = np.array([0.0, 0.25, 0.5, 1.0], dtype=np.float32)
    dc = parity.to_dev(buf)[:14]
    for fmt in (E4M3, E5M2):
        got = lib.coat_state_stats(dc, parity.to_dev(k), parity.to_dev(s), group_size=16,
                                   fmt=fmt)
        _same(got, orc.state_stats(code, k, s, 16, fmt))


@pytest.mark.parametrize("fmt", [E4M3, E5M2])
@pytest.mark.parametrize("G", [32, 128, 1024])
def test_quantized_states(lib, orc, fmt, G):
    import torch
    rng = np.random.default_rng(G + fmt)
    n = 300_000 + 77
    x = (rng.standard_normal(n) * 1e-4).astype(np.float32)
    x[: 5 * G] = 0.0                                  # a few all-zero groups
    x[5 * G: 6 * G] = 3e-5                            # an all-equal group (k = 1)
    xd = parity.to_dev(x)
    ng = -(-n // G)
    code = torch.empty(n, dtype=torch.uint8, device="cuda")
    k = torch.empty(ng, device="cuda")
    s = torch.empty(ng, device="cuda")
    lib.coat_quantize_state(xd, code, k, s, group_size=G, fmt=fmt)
    got = lib.coat_state_stats(code, k, s, group_size=G, fmt=fmt)
    want = orc.state_stats(parity.to_host(code), parity.to_host(k), parity.to_host(s), G, fmt)
    _same(got, want)
    assert got["zero_groups"] == 5 and got["k1_groups"] >= 1
    assert got["max_codes"] >= got["groups"] - got["zero_groups"]
    assert got["nonfinite_codes"] == 0


def test_optimizer_state_stats(lib):
    import torch
    from quantized_optimizer_states_b200.optim import CoatAdamW
    g = torch.Generator().manual_seed(3)
    params = [torch.nn.Parameter((torch.randn(s, generator=g) * 0.02).cuda())
              for s in [(256, 96), (1000,)]]
    opt = CoatAdamW(params, lr=1e-3, group_size=128)
    for t in range(3):
        for p in params:
            p.grad = (torch.randn(p.shape, generator=g) * 1e-3).cuda()
        opt.step()
    st = opt.state_stats()
    for key in ("m", "v"):
        assert st[key]["groups"] == opt._flat[0].n // 128
        assert st[key]["nonfinite_codes"] == 0
        assert st[key]["k_min"] > 0 and st[key]["k_max"] <= 64.0
    # COAT's expansion: v's groups are narrower, so its k runs larger than m's
    mean = {key: st[key]["k_sum"] / (st[key]["groups"] - st[key]["zero_groups"])
            for key in ("m", "v")}
    assert mean["v"] > mean["m"]
