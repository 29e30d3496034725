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
    """The bench reports the committed DRAM traffic only while the kernel's
    code (comments aside) is the one the capture was taken on; otherwise
    traffic is null."""
    src = open(os.path.join(ROOT, "bidirectional_mamba_ssm_b200", "csrc", "ssd_tc.cu")).read()
    line = open(os.path.join(ROOT, "profiles", "traffic.txt")).read()
    parts = dict(kv.split("=", 1) for kv in line.split() if "=" in kv)
    want = float(parts["dram_bytes_per_launch"]) if parts["code_sha"] == bench.code_sha(src) else None
    assert bench.kernel_traffic("ssd_tc.cu") == want
    assert bench.kernel_traffic("no_such_kernel.cu") is None
