"""CoatAdamW (torch.optim wrapper over coat_adamw_fp8_step) on the GPU:
the same result as the oracle on the flat layout, bit-identical
checkpoint/resume, the BF16-parameter path, and agreement in direction with
torch.optim.AdamW."""
import io

import numpy as np
import pytest
import torch

from quantized_optimizer_states_b200 import inputs

pytestmark = pytest.mark.gpu
H = inputs.HYPER


@pytest.fixture(scope="module")
def optim():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from quantized_optimizer_states_b200 import build
    build.build()
    from quantized_optimizer_states_b200 import optim as o
    return o


def _model(seed=0, dtype=torch.float32):
    g = torch.Generator().manual_seed(seed)
    shapes = [(64, 48), (48,), (130, 7), (1000,)]
    return [torch.nn.Parameter((torch.randn(s, generator=g) * 0.02).to("cuda", dtype))
            for s in shapes]


def _grads(params, step, seed=1):
    g = torch.Generator().manual_seed(seed * 1000 + step)
    for p in params:
        p.grad = (torch.randn(p.shape, generator=g) * 1e-3).to("cuda", p.dtype)


def _opt(o, params, **kw):
    return o.CoatAdamW(params, lr=H["lr"], betas=(H["beta1"], H["beta2"]), eps=H["eps"],
                       weight_decay=H["weight_decay"], group_size=128, **kw)


def test_matches_oracle_on_flat_layout(optim, orc):
    """Each step: the oracle starts from the optimizer's own flat state and
    gradients; its result must match the optimizer's under the parity
    tolerances."""
    params = _model()
    opt = _opt(optim, params)
    fg = opt._flat[0]
    for t in (1, 2, 3):
        _grads(params, t)
        theta = fg.master.cpu().numpy().copy()
        st = tuple(x.cpu().numpy().copy() for x in (fg.m_code, fg.m_k, fg.m_s, fg.v_code,
                                                   fg.v_k, fg.v_s))
        opt.step()
        g = fg.grad.view(torch.int16).cpu().numpy().view(np.uint16)
        ref = orc.adamw_fp8_step(theta, g, *st, step=t, group_size=128, **H)
        got = fg.master.cpu().numpy()
        err = np.max(np.abs(got - ref[0]) / np.maximum(np.abs(ref[0]), H["lr"]))
        assert err <= 1e-6, f"step {t}: theta error {err}"
        assert np.mean(fg.m_code.cpu().numpy() != ref[1]) <= 1e-4
        assert np.mean(fg.v_code.cpu().numpy() != ref[4]) <= 1e-4
        for name, i in (("m_k", 2), ("m_s", 3), ("v_k", 5), ("v_s", 6)):
            a = getattr(fg, name).cpu().numpy().astype(np.float64)
            rel = np.abs(a - ref[i]) / np.maximum(np.abs(ref[i]), 1e-38)
            assert rel.max() <= 1e-5, name
        # the optimizer writes the parameters themselves (views of the master)
        for p, off in zip(params, fg.offsets):
            assert p.data_ptr() == fg.master[off:].data_ptr()


def test_checkpoint_resume_is_bit_identical(optim):
    a = _model(seed=3)
    opt_a = _opt(optim, a)
    for t in range(1, 5):
        _grads(a, t)
        opt_a.step()

    b = _model(seed=3)
    opt_b = _opt(optim, b)
    for t in range(1, 3):
        _grads(b, t)
        opt_b.step()
    buf = io.BytesIO()
    torch.save({"model": [p.detach().cpu() for p in b], "opt": opt_b.state_dict()}, buf)
    del opt_b, b
    buf.seek(0)
    ck = torch.load(buf, weights_only=False)
    c = [torch.nn.Parameter(t.to("cuda")) for t in ck["model"]]
    opt_c = _opt(optim, c)
    opt_c.load_state_dict(ck["opt"])
    for t in range(3, 5):
        _grads(c, t)
        opt_c.step()
    fa, fc = opt_a._flat[0], opt_c._flat[0]
    for k in ("master", "m_code", "v_code", "m_k", "m_s", "v_k", "v_s"):
        assert torch.equal(getattr(fa, k), getattr(fc, k)), k
    for pa, pc in zip(a, c):
        assert torch.equal(pa, pc)


def test_bf16_parameters(optim):
    p32 = _model(seed=5)
    p16 = [torch.nn.Parameter(p.detach().to(torch.bfloat16)) for p in p32]
    opt = _opt(optim, p16)
    fg = opt._flat[0]
    for t in (1, 2):
        _grads(p16, t)
        opt.step()
    for p, off in zip(p16, fg.offsets):
        want = fg.master[off:off + p.numel()].to(torch.bfloat16).view_as(p)
        assert torch.equal(p.detach(), want)


def test_direction_matches_torch_adamw(optim):
    """Against unquantized torch.optim.AdamW: the FP8 moments change the
    update only slightly (cosine similarity of the parameter change)."""
    pa = _model(seed=7)
    pb = [torch.nn.Parameter(p.detach().clone()) for p in pa]
    opt_a = _opt(optim, pa)
    opt_b = torch.optim.AdamW(pb, lr=H["lr"], betas=(H["beta1"], H["beta2"]), eps=H["eps"],
                              weight_decay=H["weight_decay"])
    start = [p.detach().clone() for p in pb]
    for t in range(1, 6):
        _grads(pa, t)
        _grads(pb, t)
        opt_a.step()
        opt_b.step()
    da = torch.cat([(p.detach() - s).reshape(-1) for p, s in zip(pa, start)])
    db = torch.cat([(p.detach() - s).reshape(-1) for p, s in zip(pb, start)])
    cos = torch.nn.functional.cosine_similarity(da, db, dim=0).item()
    assert cos > 0.99, cos


def test_dequantized_moments_shape(optim):
    params = _model(seed=9)
    opt = _opt(optim, params, v_fmt="e5m2")
    _grads(params, 1)
    opt.step()
    m, v = opt.dequantized_moments()
    assert m.shape == v.shape == opt.flat_master().shape
    assert torch.all(v >= 0)
    assert torch.isfinite(m).all() and torch.isfinite(v).all()


def test_zero1_shard_single_rank_is_the_plain_step(optim):
    """Without a process group the ZeRO-1 shard is the whole (padded) buffer:
    its step equals a direct coat_adamw_fp8_step."""
    import quantized_optimizer_states_b200 as q
    from quantized_optimizer_states_b200 import zero
    n = 3 * 128 + 50
    g = torch.Generator().manual_seed(4)
    theta = (torch.randn(n, generator=g) * 0.02).cuda()
    sh = zero.Zero1Shard(theta, group_size=128)
    L = sh.L
    th = torch.zeros(L, device="cuda")
    th[:n] = theta
    mc = torch.zeros(L, dtype=torch.uint8, device="cuda")
    vc = torch.zeros_like(mc)
    ng = L // 128
    mk, vk = torch.ones(ng, device="cuda"), torch.ones(ng, device="cuda")
    ms, vs = torch.zeros(ng, device="cuda"), torch.zeros(ng, device="cuda")
    for t in (1, 2):
        grad = (torch.randn(n, generator=g) * 1e-3).to(torch.bfloat16).cuda()
        full = sh.step(grad, t, H)
        gp = torch.zeros(L, dtype=torch.bfloat16, device="cuda")
        gp[:n] = grad
        q.coat_adamw_fp8_step(th, gp, mc, mk, ms, vc, vk, vs, step=t, group_size=128, **H)
        assert torch.equal(full, th[:n])
        assert torch.equal(sh.m_code, mc) and torch.equal(sh.v_code, vc)


def test_flat_fp32_gradients_match_the_packed_path(optim):
    """flat_grads=True: .grad are views of one FP32 buffer, the step reads it
    directly (rounding to BF16 on load); the parameters and states must be
    bit-identical to the packed path on the same gradients, also when a
    .grad is replaced by a tensor of its own (that group is packed)."""
    pa, pb = _model(3), _model(3)
    oa = _opt(optim, pa, flat_grads=True)
    ob = _opt(optim, pb)
    fa, fb = oa._flat[0], ob._flat[0]
    for t in (1, 2, 3, 4):
        g = torch.Generator().manual_seed(77 + t)
        grads = [(torch.randn(p.shape, generator=g) * 1e-3).cuda() for p in pa]
        for p, q, x in zip(pa, pb, grads):
            if t == 3 and p is pa[1]:
                p.grad = x.clone()          # replaced: this step takes the packed path
            else:
                p.grad.copy_(x)             # in place into the flat buffer
            q.grad = x.clone()
        assert oa._grads_are_views(fa) == (t != 3)
        oa.step()
        ob.step()
        oa.zero_grad()
        assert oa._grads_are_views(fa)
        for k in ("master", "m_code", "m_k", "m_s", "v_code", "v_k", "v_s"):
            assert torch.equal(getattr(fa, k), getattr(fb, k)), (t, k)


def test_flat_fp32_gradients_through_backward(optim):
    """backward accumulates into the flat buffer in place (the .grad stay
    views), and the result equals the packed path."""
    torch.manual_seed(5)
    lin_a = torch.nn.Linear(96, 80).cuda()
    lin_b = torch.nn.Linear(96, 80).cuda()
    lin_b.load_state_dict(lin_a.state_dict())
    oa = _opt(optim, list(lin_a.parameters()), flat_grads=True)
    ob = _opt(optim, list(lin_b.parameters()))
    x = torch.randn(32, 96, device="cuda")
    for _ in range(3):
        for lin, opt in ((lin_a, oa), (lin_b, ob)):
            opt.zero_grad()
            lin(x).square().mean().backward()
        assert oa._grads_are_views(oa._flat[0])
        oa.step()
        ob.step()
    for pa, pb in zip(lin_a.parameters(), lin_b.parameters()):
        assert torch.equal(pa, pb)


@pytest.mark.parametrize("path", ["peers", "nccl"])
def test_bench_zero1_path_on_one_rank(path):
    """bench.py's ZeRO-1 timing paths run end to end as a one-rank process
    group on the 2^28-parameter sweep set (a subprocess, so its process group
    and environment stay out of this one): the one-kernel step over peer
    memory with its barrier and kernel phases, and the NCCL path (BF16
    reduce-scatter, the step on the shard, BF16 all-gather) with its three."""
    import json
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = {k: v for k, v in os.environ.items()
           if k not in ("WORLD_SIZE", "RANK", "LOCAL_RANK", "MASTER_ADDR", "MASTER_PORT")}
    out = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--zero1",
                          "--zero1-path", path, "--workload", "sweep", "--steps", "2",
                          "--warmup", "1", "--e2e-steps", "1"], capture_output=True, text=True,
                         timeout=600, env=env)
    assert out.returncode == 0, out.stderr[-3000:]
    line = json.loads([l for l in out.stdout.splitlines() if l.startswith("{")][-1])
    assert line["n_gpus"] == 1 and line["scaling"] == "strong" and line["value"] > 0
    if path == "peers":
        ph = line["phases"]
        assert ph["kernel_ms"] > 0 and ph["barrier_ms"] >= 0
        assert line["roofline"]["bound"] == "hbm" and 0 < line["roofline"]["frac"] < 1.5
    else:
        c = line["collectives"]
        assert c["reduce_scatter_ms"] > 0 and c["step_ms"] > 0 and c["all_gather_ms"] > 0
    assert line["e2e"]["value"] > 0 and line["gpu_launches"] == 2
