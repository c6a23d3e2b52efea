"""Multi-GPU plumbing of the VSA attention call (host logic only).

Every (batch, head) slice is independent from pooling to the output (the
adaptive statistics are per head as well), so a call shards over heads, or
runs as independent replicas, with no collective on the data path. One
process per GPU; torch.distributed carries only the timing reductions.
"""

from __future__ import annotations


def head_range(rank: int, world: int, H: int) -> tuple[int, int]:
    """Contiguous heads [h0, h1) of `rank` when H heads are split over `world`
    ranks; the first H % world ranks take one head more."""
    if world < 1 or not 0 <= rank < world or H < 0:
        raise ValueError("bad rank/world/H")
    base, extra = divmod(H, world)
    h0 = rank * base + min(rank, extra)
    return h0, h0 + base + (1 if rank < extra else 0)


def head_slice(x, h0: int, h1: int):
    """The heads [h0, h1) of a [B, S, H, ...] tensor as a view (same strides):
    the library takes element strides, so a head slice needs no copy."""
    return x[:, :, h0:h1]


def replica_seed(base: int, rank: int) -> int:
    """Seed of a replica's synthetic inputs: every rank draws its own problem."""
    return base + rank


def _reduce(values, dist, op_name: str, device=None):
    import torch
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    if dist is not None and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=getattr(dist.ReduceOp, op_name))
    return t.tolist()


def max_over_ranks(values, dist=None, device=None):
    """Element-wise maximum over ranks (times: the slowest rank sets the job time)."""
    return _reduce(values, dist, "MAX", device)


def sum_over_ranks(values, dist=None, device=None):
    """Element-wise sum over ranks (work: the units every rank processed)."""
    return _reduce(values, dist, "SUM", device)
