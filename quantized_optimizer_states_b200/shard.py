"""Group-aligned sharding of a flat parameter buffer across data-parallel ranks.

The COAT step works on independent 1xG groups, so a parameter set can be
split across ranks at group boundaries with no exchange inside the step:
each rank owns a contiguous, whole-group slice of the flat parameter, grad,
code and metadata buffers.  Timing across ranks is reported as the maximum
over ranks.
"""
from __future__ import annotations


def shard_range(n: int, group_size: int, rank: int, world: int) -> tuple[int, int]:
    """[start, end) element range owned by `rank`: contiguous, starting on a
    group boundary, with the ceil(n / G) groups spread as evenly as possible
    (the first ngroups % world ranks get one extra group)."""
    if n < 0 or group_size < 1 or world < 1 or not 0 <= rank < world:
        raise ValueError("bad shard arguments")
    ngroups = -(-n // group_size)
    base, extra = divmod(ngroups, world)
    g0 = rank * base + min(rank, extra)
    g1 = g0 + base + (1 if rank < extra else 0)
    return min(n, g0 * group_size), min(n, g1 * group_size)


def group_range(n: int, group_size: int, rank: int, world: int) -> tuple[int, int]:
    """[first, last) group indices owned by `rank` (metadata slice)."""
    start, end = shard_range(n, group_size, rank, world)
    return start // group_size, -(-end // group_size)


def max_over_ranks(value: float, device=None) -> float:
    """Maximum of a per-rank float over the default process group (identity
    when torch.distributed is not initialised)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())
