"""Multi-rank host logic on CPU: group-aligned sharding and max-over-ranks
timing, with two gloo ranks."""
import os
import socket

import pytest
import torch.multiprocessing as mp

from quantized_optimizer_states_b200 import shard


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_shard_ranges_partition_single_process():
    for n in (0, 1, 127, 128, 129, 1000, 6_888_095_744):
        for G in (16, 128, 1024):
            for world in (1, 2, 3, 8):
                spans = [shard.shard_range(n, G, r, world) for r in range(world)]
                assert spans[0][0] == 0 and spans[-1][1] == n
                for (a0, a1), (b0, b1) in zip(spans, spans[1:]):
                    assert a1 == b0
                for a0, a1 in spans:
                    assert (a0 % G == 0 or a0 == n) and a0 <= a1
                sizes = [-(-(a1 - a0) // G) for a0, a1 in spans]
                assert max(sizes) - min(sizes) <= 1
    with pytest.raises(ValueError):
        shard.shard_range(10, 0, 0, 1)


def _worker(rank, world, port, n, G, q):
    import torch
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        start, end = shard.shard_range(n, G, rank, world)
        t = torch.tensor([start, end], dtype=torch.int64)
        out = [torch.zeros(2, dtype=torch.int64) for _ in range(world)]
        dist.all_gather(out, t)
        tmax = shard.max_over_ranks(1.5 + rank)
        q.put((rank, [tuple(o.tolist()) for o in out], tmax))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_agree_on_shards_and_max():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    world, n, G = 2, 1_000_003, 128
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, n, G, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, spans, tmax in res:
        assert spans == [shard.shard_range(n, G, r, world) for r in range(world)]
        assert tmax == 2.5
