"""Sequence parallelism for the bidirectional mixer core: one sequence split
into contiguous shards, one per rank of a torch.distributed group.

The scan carries a state along the sequence in both directions.  A shard's
effect on the state crossing it is affine, h -> 2^dec h + S, so each rank
first reduces its shard to (S, dec) for both directions (the library's
state-only kernel), the ranks all-gather them, and each rank then computes
its outputs entering its shard with the states the shards before it
(forward) or after it (reverse) hand on; the chaining runs in the scan
kernel's prologue.  The conv reads 3 tokens across each shard boundary, so
the ranks also exchange their first and last 4 raw tokens.  The only
collectives are these all-gathers (NCCL between GPUs; gloo in the CPU tests).
"""
import torch
import torch.distributed as dist

from . import _lib


def _all_gather(t, group):
    out = [torch.empty_like(t) for _ in range(dist.get_world_size(group))]
    dist.all_gather(out, t.contiguous(), group=group)
    return out


def exchange_halos(xbc, group=None):
    """(tail, head): the 4 raw tokens before this rank's shard (the previous
    rank's last 4; zeros on rank 0) and the 4 after it (the next rank's
    first 4; zeros on the last rank).  Every shard needs at least 4 tokens."""
    rank, world = dist.get_rank(group), dist.get_world_size(group)
    if xbc.shape[1] < 4:
        raise ValueError("sequence shards need at least 4 tokens each")
    firsts = _all_gather(xbc[:, :4], group)
    lasts = _all_gather(xbc[:, -4:], group)
    zeros = torch.zeros_like(firsts[0])
    tail = lasts[rank - 1] if rank > 0 else zeros
    head = firsts[rank + 1] if rank + 1 < world else zeros
    return tail, head


def bimamba_sequence_parallel(xbc, dt, A, D, conv_w, conv_b, init_state, y, workspace, *, heads,
                              headdim, d_state, group=None, final_state=None, kernels=None):
    """This rank's outputs y (batch, shard_len, H*P) of the bidirectional
    mixer over the whole sharded sequence; final_state (optional) receives
    the forward state after this shard (the sequence's on the last rank).
    `kernels` replaces the library's two shard calls (tests only)."""
    k = kernels or _lib
    rank, world = dist.get_rank(group), dist.get_world_size(group)
    bsz = xbc.shape[0]
    tail, head = exchange_halos(xbc, group)
    states = torch.empty((2, bsz, heads, headdim, d_state), dtype=torch.float32, device=xbc.device)
    decays = torch.empty((2, bsz, heads), dtype=torch.float32, device=xbc.device)
    k.bimamba_shard_states(xbc, dt, A, conv_w, conv_b, tail, head, states, decays, workspace,
                           heads=heads, headdim=headdim, d_state=d_state)
    all_states = torch.stack(_all_gather(states, group))
    all_decays = torch.stack(_all_gather(decays, group))
    k.bimamba_ssd_fwd_rev_shard(xbc, dt, A, D, conv_w, conv_b, tail, head, init_state, all_states,
                                all_decays, rank, world, final_state, y, workspace, heads=heads,
                                headdim=headdim, d_state=d_state)
    return y
