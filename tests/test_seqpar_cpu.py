"""Host logic of the sequence-parallel path on CPU with gloo (world sizes 2
and 3): the halo exchange hands each rank its neighbours' boundary tokens,
and the gathered shard states arrive in rank order.  The two kernel calls are
replaced by recorders; their arithmetic is tested on the GPU with simulated
ranks (tests/test_parity_gpu.py)."""
import os
import socket

import pytest
import torch
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


class _Recorder:
    """Stands in for the library's shard calls: writes rank-tagged states and
    records what the orchestration hands to the output call."""

    def __init__(self):
        self.got = {}

    def bimamba_shard_states(self, xbc, dt, A, conv_w, conv_b, tail, head, states, decays, ws,
                             **kw):
        import torch.distributed as dist
        r = dist.get_rank()
        states.copy_(torch.arange(states.numel(), dtype=torch.float32).reshape(states.shape) + 1000 * r)
        decays.fill_(-1.0 - r)
        self.got["tail"], self.got["head"] = tail.clone(), head.clone()

    def bimamba_ssd_fwd_rev_shard(self, xbc, dt, A, D, conv_w, conv_b, tail, head, init, all_states,
                                  all_decays, rank, nranks, final, y, ws, **kw):
        self.got.update(all_states=all_states.clone(), all_decays=all_decays.clone(), rank=rank,
                        nranks=nranks, tail2=tail.clone(), head2=head.clone())
        y.fill_(float(rank))


def _worker(rank, world, port, lens, q):
    import torch.distributed as dist
    from bidirectional_mamba_ssm_b200 import seqpar
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        bsz, ch, H, P, N = 2, 24, 2, 4, 8
        total = sum(lens)
        full = torch.arange(bsz * total * ch, dtype=torch.float32).reshape(bsz, total, ch)
        s0 = sum(lens[:rank])
        shard = full[:, s0:s0 + lens[rank]].contiguous()
        dt = torch.ones(bsz, lens[rank], H)
        y = torch.empty(bsz, lens[rank], H * P)
        rec = _Recorder()
        seqpar.bimamba_sequence_parallel(shard, dt, torch.ones(H), torch.ones(H), None, None, None,
                                         y, None, heads=H, headdim=P, d_state=N, kernels=rec)
        g = rec.got
        # halos: the previous shard's last 4 tokens and the next shard's first 4 (zeros at the ends)
        want_tail = full[:, s0 - 4:s0] if rank > 0 else torch.zeros(bsz, 4, ch)
        e = s0 + lens[rank]
        want_head = full[:, e:e + 4] if rank + 1 < world else torch.zeros(bsz, 4, ch)
        ok = torch.equal(g["tail"], want_tail) and torch.equal(g["head"], want_head)
        ok &= torch.equal(g["tail2"], want_tail) and torch.equal(g["head2"], want_head)
        # gathered states in rank order, with each rank's own values
        base = torch.arange(2 * bsz * H * P * N, dtype=torch.float32).reshape(2, bsz, H, P, N)
        for r in range(world):
            ok &= torch.equal(g["all_states"][r], base + 1000 * r)
            ok &= bool((g["all_decays"][r] == -1.0 - r).all())
        ok &= g["rank"] == rank and g["nranks"] == world and bool((y == rank).all())
        q.put((rank, bool(ok)))
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("lens", [(9, 7), (5, 12, 4)])
def test_sequence_parallel_exchange_gloo(lens):
    from bidirectional_mamba_ssm_b200 import build
    build.build()   # the orchestration module imports the library (it only loads here)
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    world = len(lens)
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, lens, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=180)
        assert p.exitcode == 0
    got = dict(q.get(timeout=10) for _ in range(world))
    assert all(got[r] for r in range(world)), got


def test_shards_shorter_than_the_halo_are_refused():
    import torch.distributed as dist
    from bidirectional_mamba_ssm_b200 import build
    build.build()
    from bidirectional_mamba_ssm_b200 import seqpar
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(_free_port())
    dist.init_process_group("gloo", rank=0, world_size=1)
    try:
        with pytest.raises(ValueError):
            seqpar.exchange_halos(torch.zeros(1, 3, 8))
    finally:
        dist.destroy_process_group()


def test_orchestration_calls_match_the_binding_signatures():
    """The recorders above accept anything; this binds the orchestration's
    actual calls against the real binding functions' signatures, so that an
    argument added, dropped or reordered in either place fails on CPU."""
    import inspect
    import torch.distributed as dist
    from bidirectional_mamba_ssm_b200 import build
    build.build()
    from bidirectional_mamba_ssm_b200 import _lib, seqpar

    class Binder:
        def __init__(self):
            self.bound = []

        def __getattr__(self, name):
            real = getattr(_lib, name)

            def call(*a, **kw):
                inspect.signature(real).bind(*a, **kw)   # raises TypeError on a mismatch
                self.bound.append(name)
            return call

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(_free_port())
    dist.init_process_group("gloo", rank=0, world_size=1)
    try:
        b = Binder()
        x = torch.zeros(1, 8, 24)
        seqpar.bimamba_sequence_parallel(x, torch.zeros(1, 8, 2), torch.zeros(2), torch.zeros(2),
                                         None, None, None, torch.zeros(1, 8, 8), None, heads=2,
                                         headdim=4, d_state=8, kernels=b)
        assert b.bound == ["bimamba_shard_states", "bimamba_ssd_fwd_rev_shard"]
    finally:
        dist.destroy_process_group()
