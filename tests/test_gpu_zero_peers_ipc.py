"""The one-kernel ZeRO-1 step across processes: two ranks (processes) on one
GPU, gloo for the barriers and the exchange of CUDA IPC handles, each rank's
kernel reading the other's gradient buffer and writing the other's parameter
buffer through the IPC mapping (on a multi-GPU node the same mapping is a
peer GPU's memory).  Checked against the oracle's step on the oracle's
gradient mean.  No kernel waits for another: the ranks meet on the host."""
import datetime
import os
import socket

import numpy as np
import pytest

import parity
from quantized_optimizer_states_b200 import inputs

pytestmark = pytest.mark.gpu

E4M3 = 0
H = inputs.HYPER
G = 128


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _problem(n, world):
    import oracle as orc
    x = inputs.host_step_inputs(inputs.olmo_1b(), n)
    mc, mk, ms = orc.quantize_state(x["m0"], G, E4M3)
    vc, vk, vs = orc.quantize_state(x["v0"], G, E4M3)
    grads = []
    for r in range(world):
        rng = np.random.default_rng(1000 + r)
        grads.append(orc.to_bf16_array((rng.standard_normal(n) * 1e-3).astype(np.float32)))
    return x["theta"], (mc, mk, ms, vc, vk, vs), grads


def _worker(rank, world, port, n, q):
    import torch
    import torch.distributed as dist
    import quantized_optimizer_states_b200 as coat
    from quantized_optimizer_states_b200 import zero
    try:
        torch.cuda.set_device(0)
        dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                                world_size=world, timeout=datetime.timedelta(seconds=120))
        coat.load()
        th, st, grads = _problem(n, world)
        shard = zero.Zero1Shard(torch.from_numpy(th).cuda(), group_size=G)
        lo, L = rank * shard.L, shard.L
        hi = min(n, lo + L)
        for name, a, per in zip(("m_code", "m_k", "m_s", "v_code", "v_k", "v_s"), st,
                                (1, G, G, 1, G, G)):
            dst = getattr(shard, name)
            src = torch.from_numpy(np.ascontiguousarray(a[lo // per:-(-hi // per)]))
            dst[:src.numel()].copy_(src)
        bufs = zero.PeerBuffers(shard, torch.bfloat16)
        bufs.grad[:n].copy_(torch.from_numpy(grads[rank].view(np.int16)).view(torch.bfloat16))
        out = shard.step_peers(bufs, 10, dict(H))
        torch.cuda.synchronize()
        res = {name: getattr(shard, name).cpu().numpy() for name in
               ("master", "m_code", "m_k", "m_s", "v_code", "v_k", "v_s")}
        res["param"] = out.view(torch.int16).cpu().numpy()
        q.put((rank, res))
        del bufs, out                    # unmap the other rank's buffers before either exits
        torch.cuda.synchronize()
        dist.barrier()
        dist.destroy_process_group()
    except Exception as e:  # reported to the parent, which fails the test
        q.put((rank, repr(e)))


def test_two_processes_on_one_gpu(orc):
    import torch
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import torch.multiprocessing as mp
    from quantized_optimizer_states_b200 import build, zero
    build.build()
    world, n = 2, 7 * 4096 + 3 * G + 5
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, n, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = {}
    for _ in range(world):
        rank, res = q.get(timeout=300)
        assert not isinstance(res, str), f"rank {rank}: {res}"
        got[rank] = res
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0

    th, st, grads = _problem(n, world)
    cfg = dict(step=10, group_size=G, v_fmt=E4M3, **H)
    g_mean = orc.grad_mean_bf16(grads)
    ref = orc.adamw_fp8_step(th, g_mean, *st, return_moments=True, **cfg)
    L = zero.shard_length(n, G, world)
    theta_new = np.concatenate([got[r]["master"] for r in range(world)])[:n]
    gpu = (theta_new,) + tuple(
        np.concatenate([got[r][k] for r in range(world)])[:m]
        for k, m in (("m_code", n), ("m_k", -(-n // G)), ("m_s", -(-n // G)),
                     ("v_code", n), ("v_k", -(-n // G)), ("v_s", -(-n // G))))
    parity.assert_step_parity(gpu, ref, H["lr"], G, E4M3, moments=(ref[7], ref[8]))
    want = orc.to_bf16_array(theta_new).view(np.int16)
    for r in range(world):               # every rank holds every rank's updated shard
        assert np.array_equal(got[r]["param"], want), r
    assert L * world >= n
