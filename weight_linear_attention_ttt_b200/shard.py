"""Data-parallel placement of independent streams over ranks (one process per GPU).

Every (batch, head) stream of the dual form and of the associative mode is independent of the
others ("Learning to (Learn at Test Time)" reading, long-context section: states of different
batch items are kept apart), and the columns of the In-Place W_down are independent of each
other. Work therefore shards over ranks with no collective on the data path: each rank runs the
library on its own slice. The only collectives are host-side bookkeeping: a barrier and the
max-over-ranks reduction of timings.
"""
from __future__ import annotations

from typing import Tuple


def split_range(n: int, rank: int, world: int) -> Tuple[int, int]:
    """Contiguous, balanced [start, stop) share of n items for `rank` of `world` (the first
    n % world ranks get one extra item)."""
    if world <= 0 or not 0 <= rank < world:
        raise ValueError("rank must lie in [0, world)")
    base, extra = divmod(n, world)
    start = rank * base + min(rank, extra)
    return start, start + base + (1 if rank < extra else 0)


def shard_streams(x: dict, rank: int, world: int) -> dict:
    """Rank's slice, along the batch dimension, of dual/associative inputs
    ({Q, K, V: [B,H,T,d], eta: [B,H,T] or None, W0: [B,H,d,d] or None, ...})."""
    B = x["Q"].shape[0]
    b0, b1 = split_range(B, rank, world)
    out = {}
    for k, v in x.items():
        out[k] = v[b0:b1].contiguous() if hasattr(v, "shape") and getattr(v, "dim", lambda: 0)() >= 3 \
            else v
    return out


def shard_columns(x: dict, rank: int, world: int) -> dict:
    """Rank's slice of In-Place inputs by output column: Z is shared, Vhat[:, cols] and
    W0[:, cols] are the rank's own (each output column of O and W depends only on them)."""
    D = x["Vhat"].shape[1]
    c0, c1 = split_range(D, rank, world)
    out = dict(x)
    out["Vhat"] = x["Vhat"][:, c0:c1].contiguous()
    out["W0"] = x["W0"][:, c0:c1].contiguous()
    return out


def max_over_ranks(value: float, device=None) -> float:
    """The maximum of `value` over all ranks (identity without an initialised process group)."""
    import torch
    import torch.distributed as dist

    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64,
                     device=device if device is not None else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())
