"""Independent replicas across ranks for the mixer's data-parallel path.

Sequences (and decode streams) are independent, so N GPUs run N replicas,
each on its own sequences, with no collective on the data path.  The only
cross-rank steps are the timing barrier and the aggregation below:
whole-job throughput = all ranks' tokens / the slowest rank's time.
"""
from __future__ import annotations

import torch
import torch.distributed as dist


def rank_slice(total: int, rank: int, world: int) -> tuple[int, int]:
    """[start, stop) of the items rank `rank` owns when `total` items are
    split as evenly as possible over `world` ranks (earlier ranks get the
    remainder)."""
    if world <= 0 or not 0 <= rank < world or total < 0:
        raise ValueError("bad rank/world/total")
    base, extra = divmod(total, world)
    start = rank * base + min(rank, extra)
    return start, start + base + (1 if rank < extra else 0)


def aggregate(tokens: float, ms: float, device=None) -> tuple[float, float, float]:
    """Combine per-rank (tokens processed, elapsed ms) into
    (total tokens, max ms over ranks, tokens/s).  Single process: identity."""
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        t = torch.tensor([float(tokens)], dtype=torch.float64, device=device)
        m = torch.tensor([float(ms)], dtype=torch.float64, device=device)
        dist.all_reduce(t, op=dist.ReduceOp.SUM)
        dist.all_reduce(m, op=dist.ReduceOp.MAX)
        tokens, ms = float(t.item()), float(m.item())
    return tokens, ms, tokens / (ms / 1e3) if ms > 0 else 0.0
