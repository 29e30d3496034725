"""Host-side pieces of bench.py that need no GPU: the algorithmic byte and
flop counts behind the roofline, and the code hash that ties a committed
DRAM-traffic capture to the kernel source it was taken on."""
import os

import bench
from bidirectional_mamba_ssm_b200 import inputs as I

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_algorithmic_counts_of_the_benchmarked_layer():
    w = I.LAYER_1P3B
    nbytes, flops = bench.algorithmic(w, 8, 4096)
    # per token: xBC in (64*64 + 2*128) + dt (64) + y out (64*64), bf16
    assert nbytes == 2 * (4096 + 256 + 64 + 4096) * 8 * 4096 == 557_842_432
    # 2*(2*Q*N + H*(Q*P + 4*P*N)) per token with Q = 64
    assert flops == 2 * (2 * 64 * 128 + 64 * (64 * 64 + 4 * 64 * 128)) * 8 * 4096
    ub, uf = bench.algorithmic(w, 8, 4096, untied=True)
    assert ub == 2 * nbytes and uf == flops
    db, _ = bench.algorithmic(w, 32, 64, decode=True)
    state = 64 * 64 * 128 * 4
    tail = 4 * (4096 + 256) * 2
    assert db == 2 * (4096 + 256 + 64 + 4096) * 32 * 64 + 32 * (state + tail)


def test_code_hash_ignores_comments_and_whitespace_only():
    a = "int f(int x) {\n    return x + 1;   // one\n}\n/* block\n comment */\n"
    b = "int f(int x) { return x + 1; }\n// another comment\n"
    c = "int f(int x) { return x + 2; }\n"
    assert bench.code_sha(a) == bench.code_sha(b)
    assert bench.code_sha(a) != bench.code_sha(c)


def test_traffic_record_applies_only_to_the_code_it_was_taken_on():
    """The bench reports the committed DRAM traffic of a workload only while
    the kernel's code (comments aside) is the one the capture was taken on;
    otherwise traffic is null."""
    lines = [l for l in open(os.path.join(ROOT, "profiles", "traffic.txt")) if l.strip()]
    assert lines
    for line in lines:
        parts = dict(kv.split("=", 1) for kv in line.split() if "=" in kv)
        src = open(os.path.join(ROOT, "bidirectional_mamba_ssm_b200", "csrc", parts["file"])).read()
        want = float(parts["dram_bytes_per_launch"]) if parts["code_sha"] == bench.code_sha(src) else None
        assert bench.kernel_traffic(parts["file"], parts["workload"]) == want
        assert bench.kernel_traffic(parts["file"], "no_such_workload") is None
    assert bench.kernel_traffic("no_such_kernel.cu", "layer1p3b") is None


def test_tensor_peak_follows_the_sampled_clocks():
    """Burst peak when the timed region saw no power capping; burst scaled by
    the sampled median / max SM clock when sw_power_cap was active."""
    peaks = {"hbm_gbs": 6000.0, "bf16_tflops": 1600.0, "bf16_tflops_sustained": 1300.0}
    p, rule = bench.tensor_peak(peaks, {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": []})
    assert p == 1600.0 and "burst" in rule
    p, rule = bench.tensor_peak(peaks, {"sm_mhz": 1300.0, "sm_max_mhz": 1950.0,
                                        "reasons": ["sw_power_cap"]})
    assert abs(p - 1600.0 * 1300.0 / 1950.0) < 1e-9 and "sw_power_cap" in rule
    assert bench.tensor_peak(peaks, None)[0] == 1600.0
    roof, ctx = bench.roofline(peaks, "measured", None, nbytes=6e9, flops=1.6e15, kernel_s=2.0,
                               decode=False, kernel_file="ssd_tc.cu")
    # t_hbm = 1 ms < t_tc = 1 s: tensor-bound, 0.8 PF/s achieved of 1.6
    assert roof["bound"] == "tensor" and abs(roof["frac"] - 0.5) < 1e-12
    roof, _ = bench.roofline(peaks, "measured", None, nbytes=6e9, flops=1.0, kernel_s=2e-3,
                             decode=True, kernel_file="ssd_tc.cu")
    assert roof["bound"] == "hbm" and abs(roof["frac"] - 0.5) < 1e-12


def test_gpus_flag_against_the_launch_environment():
    assert bench.resolve_world(1, {}) == ("run", 1)
    assert bench.resolve_world(4, {}) == ("spawn", 4)
    assert bench.resolve_world(2, {"WORLD_SIZE": "2"}) == ("run", 2)
    how, why = bench.resolve_world(8, {"WORLD_SIZE": "1"})
    assert how == "refuse" and "WORLD_SIZE=1" in why
    assert bench.resolve_world(0, {})[0] == "refuse"


def _rank_worker(rank, world, port, q):
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # rank r ran 100*(r+1) tokens per step for 20 steps in 10+5r ms, its
        # main kernel averaging 0.4+0.1r ms, with 40 launches each
        q.put((rank, bench.combine_ranks(2000.0 * (rank + 1), 10.0 + 5.0 * rank,
                                         0.4 + 0.1 * rank, 40)))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_bench_rank_path_two_gloo_ranks():
    """The bench's per-rank figures combined over two gloo ranks: all ranks'
    tokens, the slowest rank's time, every rank's launches."""
    import socket

    import torch.multiprocessing as mp
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    got = dict(q.get(timeout=10) for _ in range(2))
    for r in range(2):
        tokens, ms, kernel_ms, launches = got[r]
        assert tokens == 6000.0 and ms == 15.0 and abs(kernel_ms - 0.5) < 1e-12
        assert launches == 80
