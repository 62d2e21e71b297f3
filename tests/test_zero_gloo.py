"""ZeRO-1 sharded COAT step (quantized_optimizer_states_b200.zero) with two
gloo ranks on CPU.  The CUDA step is replaced by the oracle on each shard;
the sharded result must equal one oracle step over the whole buffer on the
rank-mean gradient, bit for bit (groups never straddle shards)."""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

from quantized_optimizer_states_b200 import inputs, zero

H = inputs.HYPER
G = 128


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_shard_length():
    assert zero.shard_length(1000, 128, 2) == 512
    assert zero.shard_length(1024, 128, 2) == 512
    assert zero.shard_length(1025, 128, 2) == 640
    assert zero.shard_length(7, 16, 3) == 16
    assert zero.shard_length(0, 128, 4) == 0
    with pytest.raises(ValueError):
        zero.shard_length(10, 0, 2)


def _inputs(n, world, steps):
    rng = np.random.default_rng(42)
    theta = rng.normal(0, 0.02, n).astype(np.float32)
    grads = rng.normal(0, 1e-3, (steps, world, n)).astype(np.float32)
    return theta, grads


def _oracle_step_fn():
    import oracle
    import torch

    def step_fn(shard, g_shard, t, hyper):
        gb = g_shard.view(torch.int16).numpy().view(np.uint16)
        st = tuple(x.numpy() for x in (shard.m_code, shard.m_k, shard.m_s, shard.v_code,
                                       shard.v_k, shard.v_s))
        out = oracle.adamw_fp8_step(shard.master.numpy(), gb, *st, step=t, group_size=G,
                                    **hyper)
        for dst, src in zip((shard.master, shard.m_code, shard.m_k, shard.m_s, shard.v_code,
                             shard.v_k, shard.v_s), out[:7]):
            dst.copy_(torch.from_numpy(np.ascontiguousarray(src)))
    return step_fn


def _worker(rank, world, port, n, steps, q):
    import torch
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        theta, grads = _inputs(n, world, steps)
        sh = zero.Zero1Shard(torch.from_numpy(theta), group_size=G)
        step_fn = _oracle_step_fn()
        full = None
        for t in range(steps):
            g = torch.from_numpy(grads[t, rank]).to(torch.bfloat16)
            full = sh.step(g, 10 + t, H, step_fn=step_fn)
        q.put((rank, full.numpy().copy(), sh.L))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_match_the_single_rank_step():
    import oracle
    import torch
    world, n, steps = 2, 5 * 128 + 77, 3
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, n, steps, q))
             for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=180) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0

    # reference: one rank, whole buffer, gradient = BF16(mean over ranks)
    theta, grads = _inputs(n, world, steps)
    L = zero.shard_length(n, G, world)
    npad = world * L
    th = np.zeros(npad, np.float32)
    th[:n] = theta
    z = np.zeros(npad, np.uint8)
    ng = npad // G
    st = (z, np.ones(ng, np.float32), np.zeros(ng, np.float32), z.copy(),
          np.ones(ng, np.float32), np.zeros(ng, np.float32))
    for t in range(steps):
        gsum = torch.zeros(npad, dtype=torch.float32)
        for r in range(world):
            gsum[:n] += torch.from_numpy(grads[t, r]).to(torch.bfloat16).float()
        gmean = (gsum / world).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
        out = oracle.adamw_fp8_step(th, gmean, *st, step=10 + t, group_size=G, **H)
        th, st = out[0], out[1:7]
    for rank, full, Lr in res:
        assert Lr == L
        assert np.array_equal(full, th[:n]), f"rank {rank}"


def _resume_worker(rank, world, port, n, steps, cut, q):
    import io

    import torch
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        theta, grads = _inputs(n, world, steps)
        step_fn = _oracle_step_fn()
        g = [torch.from_numpy(grads[t, rank]).to(torch.bfloat16) for t in range(steps)]
        # straight through
        a = zero.Zero1Shard(torch.from_numpy(theta), group_size=G)
        for t in range(steps):
            full_a = a.step(g[t], 10 + t, H, step_fn=step_fn)
        # stopped after `cut` steps, saved, restored into a fresh shard
        b = zero.Zero1Shard(torch.from_numpy(theta), group_size=G)
        for t in range(cut):
            b.step(g[t], 10 + t, H, step_fn=step_fn)
        buf = io.BytesIO()
        torch.save(b.state_dict(), buf)
        buf.seek(0)
        c = zero.Zero1Shard(torch.from_numpy(np.zeros(n, np.float32)), group_size=G)
        c.load_state_dict(torch.load(buf))
        for t in range(cut, steps):
            full_c = c.step(g[t], 10 + t, H, step_fn=step_fn)
        wrong = zero.Zero1Shard(torch.from_numpy(theta), group_size=2 * G)
        try:
            wrong.load_state_dict(b.state_dict())
            rejected = False
        except ValueError:
            rejected = True
        # the BF16 all-gather: each rank's shard rounded to BF16, gathered as bits
        bf = c.gather_params(torch.bfloat16)
        same_bf16 = (bf.dtype == torch.bfloat16 and
                     torch.equal(bf.view(torch.int16), full_c.to(torch.bfloat16).view(torch.int16)))
        q.put((rank, np.array_equal(full_a.numpy(), full_c.numpy()) and same_bf16, rejected))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_resume_from_a_checkpoint_bit_for_bit():
    """Each rank saves its shard after 2 of 4 steps; fresh shards that load
    the checkpoints and take steps 3-4 end with the same parameters, bit for
    bit, as the shards that never stopped; a shard of another group size
    refuses the checkpoint."""
    world, n, steps, cut = 2, 5 * 128 + 77, 4, 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_resume_worker, args=(r, world, port, n, steps, cut, q))
             for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=180) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, same, rejected in res:
        assert same, f"rank {rank}: resumed run (or its BF16 gather) differs"
        assert rejected, f"rank {rank}: mismatched layout accepted"


def _reduce_worker(rank, world, port, n, q):
    import torch
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        grads = _exact_grads(n, world)
        g = torch.from_numpy(grads[rank]).to(torch.bfloat16)
        f32 = zero.Zero1Shard(torch.zeros(n), group_size=G, reduce_dtype=torch.float32)
        f32.F32_CHUNK = 100          # several chunks, the last one ragged
        a = f32.reduce_gradient_f32(g)
        padded = torch.zeros(f32.padded_numel, dtype=torch.bfloat16)
        padded[:n] = g
        b = f32.reduce_gradient_f32(padded)
        bf = zero.Zero1Shard(torch.zeros(n), group_size=G)
        c = bf.reduce_gradient(g)
        q.put((rank, a.numpy().copy(), b.numpy().copy(),
               c.float().numpy().copy(), c.dtype == torch.bfloat16, f32.L))
    finally:
        dist.destroy_process_group()


def _exact_grads(n, world):
    """BF16 gradients whose binary32 sums over ranks are exact (multiples of
    2^-16 below 1 in magnitude), so the binary32 mean is order-independent."""
    rng = np.random.default_rng(7)
    k = rng.integers(-60000, 60000, (world, n))
    return (k * 2.0 ** -16).astype(np.float32)


def test_reduce_scatter_bf16_and_chunked_binary32_three_gloo_ranks():
    """Three gloo ranks: the binary32 reduce-scatter, done in chunks of 100
    elements of the shard, gives each rank its shard of the binary32 mean of
    the BF16 gradients exactly, whether the gradient is passed with n
    elements or padded to world x L; the BF16 reduce-scatter gives BF16
    values within 2 BF16 steps of that mean (its partial sums are rounded
    to BF16)."""
    import torch
    world, n = 3, 5 * 128 + 77
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_reduce_worker, args=(r, world, port, n, q))
             for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=180) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    grads = _exact_grads(n, world)
    gb = torch.from_numpy(grads).to(torch.bfloat16).float().numpy().astype(np.float64)
    L = res[0][5]
    mean = np.zeros(world * L)
    mean[:n] = gb.sum(axis=0) / world
    mean32 = mean.astype(np.float32)
    # BF16 keeps 8 significant bits (unit roundoff 2^-8): each rounding of a
    # partial sum errs by at most 2^-8 of sum |g_i|, the division's by 2^-8 of
    # the result
    absum = np.zeros(world * L)
    absum[:n] = np.abs(gb).sum(axis=0)
    for rank, a, b, c, is_bf16, Lr in res:
        assert Lr == L == zero.shard_length(n, G, world)
        want = mean32[rank * L:(rank + 1) * L]
        assert np.array_equal(a, want) and np.array_equal(b, want), f"rank {rank}"
        assert is_bf16
        bound = (world - 1) * 2.0 ** -8 * absum[rank * L:(rank + 1) * L] / world \
            + 2.0 ** -8 * np.abs(want)
        assert np.all(np.abs(c - want) <= bound), f"rank {rank}: BF16 mean too far"


def _share_fail_worker(rank, world, port, fail_rank, q):
    import torch
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        sh = zero.Zero1Shard(torch.zeros(4 * G), group_size=G)

        def share(t):
            if rank == fail_rank:
                raise OSError("no shareable memory here")
            return ("handle", rank)

        zero._share = share
        zero._open = lambda shared: (_ for _ in ()).throw(AssertionError("not reached"))
        try:
            zero.PeerBuffers(sh)
            q.put((rank, "no error"))
        except Exception as e:  # noqa: BLE001 -- what the test checks
            q.put((rank, f"{type(e).__name__}: {e}"))
        dist.barrier()          # every rank is still in step with the others
    finally:
        dist.destroy_process_group()


def test_peer_buffer_exchange_fails_on_every_rank_when_one_rank_cannot_share():
    """A rank whose buffers cannot be shared (the failure made on the host,
    in one rank) still takes part in the exchange, so no rank is left
    waiting: every rank raises, the failing one with its own error, the
    others naming another rank, and all of them meet at a barrier after."""
    world = 3
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_share_fail_worker, args=(r, world, port, 1, q))
             for r in range(world)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=180) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert res[1] == "OSError: no shareable memory here"
    assert res[0].startswith("RuntimeError: another rank") and res[2] == res[0]
