"""Multi-rank host logic of the replica path, on CPU with gloo (world size 2)."""
import os
import socket

import pytest
import torch.multiprocessing as mp

from bidirectional_mamba_ssm_b200.replicas import aggregate, rank_slice


def test_rank_slice_covers_everything_once():
    for total in (0, 1, 7, 8, 32, 33):
        for world in (1, 2, 3, 8):
            parts = [rank_slice(total, r, world) for r in range(world)]
            assert parts[0][0] == 0 and parts[-1][1] == total
            for (a0, a1), (b0, b1) in zip(parts, parts[1:]):
                assert a1 == b0
            sizes = [b - a for a, b in parts]
            assert max(sizes) - min(sizes) <= 1
    with pytest.raises(ValueError):
        rank_slice(4, 2, 2)


def _worker(rank, world, port, q):
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        tokens = 1000.0 * (rank + 1)       # ranks process different amounts
        ms = 10.0 + 5.0 * rank             # rank 1 is the slowest
        q.put((rank, aggregate(tokens, ms)))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def test_aggregate_two_ranks_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    world = 2
    procs = [ctx.Process(target=_worker, args=(r, world, PORT, q))
             for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    got = dict(q.get(timeout=10) for _ in range(world))
    for r in range(world):
        tokens, ms, tps = got[r]
        assert tokens == 3000.0 and ms == 15.0
        assert abs(tps - 3000.0 / 0.015) < 1e-6


PORT = _free_port()


def test_aggregate_single_process_is_identity():
    assert aggregate(500.0, 2.0) == (500.0, 2.0, 250000.0)
