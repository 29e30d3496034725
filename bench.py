#!/usr/bin/env python
"""Throughput of the bidirectional Mamba-2 mixer core on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload long131k|layer1p3b|decode|decode_pool|untied1p3b|mixer1p3b|
                                sweep|tiny|backward1p3b]
                    [--no-cpu-baseline]

One step = one bimamba_ssd_fwd_rev call over one batch of the workload
(conv+SiLU both ways, forward and reverse SSD scans, summed output), inputs
resident in HBM.  Default workload: the largest single-GPU configuration,
one 131072-token sequence, 64 heads x headdim 64, d_state 128, bf16
activations, fp32 state; the same line carries the 1.3B-layer workload
(b8 x L4096) as its "layer1p3b" field.  Other workloads: the 1.3B layer
alone; cached block decode (32 streams x 64-token block, HBM-cold: the
timed steps rotate over state/input sets larger than L2); the layer with
untied directions and concatenated outputs; and a sweep of one sequence at
1k..256k tokens, prefill and cached decode at each length (the line's value
at 256k, a "sweep" field with every length).
Every rank runs its own copy of the workload (independent sequences, no
data-path collective): scaling is weak, value = all ranks' tokens / the
slowest rank's time.  Rank 0 prints one JSON line.  `--gpus N` without a
torchrun environment launches N local ranks itself (torch.distributed.run);
under torchrun, N must equal WORLD_SIZE.

--impl reference times the CPU oracle (the double-precision sequential
recurrence under oracle/) on the host cores, a bounded sample per step, and
prints the same line with "impl": "reference".
"""
from __future__ import annotations

import argparse
import hashlib
import re
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "BiMamba-2 scan tokens/s (fwd+rev) on 1 B200; % of HBM/tensor roofline"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse_args():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=["long131k", "layer1p3b", "decode", "decode_pool",
                                           "untied1p3b", "mixer1p3b", "sweep", "tiny",
                                           "backward1p3b"],
                    default="long131k")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=8)
    ap.add_argument("--batch", type=int, default=None,
                    help="sequences (decode: streams) per GPU; default: the workload's own")
    return ap.parse_args()


# --------------------------------------------------------------------------- workloads
SWEEP_LENGTHS = (1024, 4096, 16384, 65536, 262144)


def workload_spec(name):
    from bidirectional_mamba_ssm_b200 import inputs as I
    if name == "layer1p3b":
        return I.LAYER_1P3B, I.LAYER_1P3B.batch, I.LAYER_1P3B.seqlen
    if name == "long131k":
        return I.LONG_131K, 1, I.LONG_131K.seqlen
    if name in ("decode", "decode_pool"):
        return I.LAYER_1P3B, I.DECODE_STREAMS, I.DECODE_BLOCK
    if name == "mixer1p3b":   # the layer with its in/out projections around the mixer
        return I.LAYER_1P3B, I.LAYER_1P3B.batch, I.LAYER_1P3B.seqlen
    if name == "untied1p3b":   # the same layer with untied directions, outputs concatenated
        return I.LAYER_1P3B, I.LAYER_1P3B.batch, I.LAYER_1P3B.seqlen
    if name == "sweep":   # one sequence, prefill at 1k..256k tokens; the line's value at 256k
        return I.LONG_131K, 1, SWEEP_LENGTHS[-1]
    if name == "backward1p3b":   # gradients of the mixer core at the 1.3B-layer shape
        return I.LAYER_1P3B, I.LAYER_1P3B.batch, I.LAYER_1P3B.seqlen
    if name == "tiny":   # the small fp32 case (b1 L256 H4x32 N16): launch-bound, latency is the figure
        return I.TINY_F32, 1, I.TINY_F32.seqlen
    raise ValueError(name)


D_MODEL = 2048   # the 1.3B model's width ("DiffuMamba" blog, network-architecture listing)
POOL_STREAMS = 256   # cached streams held by the pooled-decode workload


def gemm_counts(w, tokens, d_model=D_MODEL):
    """Algorithmic bytes and flops of the two projections of one step:
    in  [xbc | dt] = u (tokens, d_model) . W_in^T (ch + H, d_model)
    out out = y (tokens, H*P) . W_out^T (d_model, H*P)
    bytes: each operand and result once (bf16)."""
    ch = w.heads * w.headdim + 2 * w.d_state
    n_in, k_out = ch + w.heads, w.heads * w.headdim
    f_in = 2 * tokens * n_in * d_model
    f_out = 2 * tokens * d_model * k_out
    b_in = 2 * (tokens * d_model + n_in * d_model + tokens * n_in)
    b_out = 2 * (tokens * k_out + d_model * k_out + tokens * d_model)
    return (b_in, f_in), (b_out, f_out)


def algorithmic(w, batch, seqlen, decode=False, untied=False):
    """Algorithmic bytes and flops of one step: the bytes the operation must
    move through HBM once and the flops of its chunked form, counted with a
    fixed chunk length so that the kernel's own chunking cannot change them.

    bytes/token = raw xBC in (H*P + 2N) + dt (H) + y out (H*P), in the
    activation dtype; decode adds the fp32 state read (H*P*N*4 per stream)
    and the conv tail (4 tokens of xBC) per stream.  Untied directions read
    both streams' xBC and dt and write both halves of the concatenated y.
    flops/token = 2*(2*Q*N + H*(Q*P + 4*P*N)) with Q = 64 fixed.
    """
    esz = 2 if w.dtype == "bf16" else 4
    H, P, N = w.heads, w.headdim, w.d_state
    per_tok = esz * ((H * P + 2 * N) + H + H * P) * (2 if untied else 1)
    tokens = batch * seqlen
    nbytes = per_tok * tokens
    if decode:
        nbytes += batch * (H * P * N * 4 + 4 * (H * P + 2 * N) * esz)
    Q = 64
    flops = 2 * (2 * Q * N + H * (Q * P + 4 * P * N)) * tokens
    return nbytes, flops


def backward_counts(w, tokens):
    """Algorithmic bytes and flops of one backward call of the mixer core.
    bytes: raw xBC, dt and dy read (bf16), d(xBC) and d(dt) written (fp32).
    flops: the adjoint's products per chunk of Q = 64 (the convention the
    forward's count uses; the kernel's chunks are 128 long) and per direction
    and head -- C.B^T, dY.X^T (Q^2 N, Q^2 P), X.dS, dY.S_in (Q P N each), W^T.dY
    (Q^2 P), B.dS^T (Q N P), T^T.C, T.B (Q^2 N each), the state adjoint (P N Q)
    -- i.e. Q(3N + 2P) + 5PN multiply-adds per token, head and direction."""
    H, P, N = w.heads, w.headdim, w.d_state
    Q = 64
    ch = H * P + 2 * N
    nbytes = tokens * (2 * (ch + H + H * P) + 4 * (ch + H))
    flops = tokens * 2 * 2 * H * (Q * (3 * N + 2 * P) + 5 * P * N)
    return nbytes, flops


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in FALLBACK_PEAKS}, "measured"
    except (OSError, KeyError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


def code_sha(text):
    """sha256[:16] of a C/CUDA source with its comments and whitespace
    removed: the same for two versions that differ only in comments."""
    text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
    text = re.sub(r"//[^\n]*", " ", text)
    text = re.sub(r"\s+", " ", text).strip()
    return hashlib.sha256(text.encode()).hexdigest()[:16]


def kernel_traffic(kernel_file, workload):
    """dram bytes per timed call (the launches the kernel events bracket) of
    this workload from the committed ncu summary, if it was taken on the
    current code of the kernel (code_sha recorded there); else None."""
    path = os.path.join(ROOT, "profiles", "traffic.txt")
    src = os.path.join(ROOT, "bidirectional_mamba_ssm_b200", "csrc", kernel_file)
    try:
        sha = code_sha(open(src).read())
        for line in open(path):
            parts = dict(kv.split("=", 1) for kv in line.split() if "=" in kv)
            if (parts.get("file") == kernel_file and parts.get("workload") == workload
                    and parts.get("code_sha") == sha):
                return float(parts["dram_bytes_per_launch"])
    except OSError:
        pass
    return None


# --------------------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.rows = []
        self.proc = None
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", gpu_id, "--query-gpu=" + self.FIELDS,
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except OSError:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.rows.append([c.strip() for c in line.split(",")])

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.t.join(timeout=2)
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in self.rows:
            try:
                sm.append(float(r[1]))
                smax.append(float(r[2]))
            except (ValueError, IndexError):
                continue
            for n, v in zip(names, r[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax),
                "reasons": sorted(reasons), "samples": len(sm)}


# --------------------------------------------------------------------------- peaks
def tensor_peak(peaks, clocks):
    """The bf16 tensor peak a kernel timed inside this run is held against.

    The burst figure (a cuBLAS GEMM timed alone, at full clock) applies when
    the clocks sampled during the timed region show no power capping; when
    sw_power_cap was active the burst figure is scaled by the sampled median
    SM clock over the maximum clock.  Returns (TFLOP/s, rule)."""
    burst = peaks["bf16_tflops"]
    if not clocks:
        return burst, "burst (no clock samples)"
    if "sw_power_cap" in clocks.get("reasons", []):
        f = clocks["sm_mhz"] / max(clocks["sm_max_mhz"], 1.0)
        return burst * f, f"burst x median/max SM clock ({f:.3f}): sw_power_cap active"
    return burst, "burst: no sw_power_cap in the clock samples"


def roofline(peaks, peak_kind, clocks, nbytes, flops, kernel_s, decode, kernel_file, workload=None):
    t_hbm = nbytes / (peaks["hbm_gbs"] * 1e9)
    tpeak, rule = tensor_peak(peaks, clocks)
    t_tc = flops / (tpeak * 1e12)
    if decode or t_hbm >= t_tc:
        roof = {"bound": "hbm", "achieved": nbytes / kernel_s / 1e9, "peak": peaks["hbm_gbs"],
                "unit": "GB/s", "peak_source": f"{peak_kind} (copy)"}
    else:
        roof = {"bound": "tensor", "achieved": flops / kernel_s / 1e12, "peak": tpeak,
                "unit": "TFLOP/s", "peak_source": f"{peak_kind} ({rule})"}
    roof["frac"] = roof["achieved"] / roof["peak"]
    roof["traffic"] = kernel_traffic(kernel_file, workload)
    roof["kernel"] = kernel_file
    ctx = {"achieved_gbs": nbytes / kernel_s / 1e9, "peak_gbs": peaks["hbm_gbs"],
           "frac": nbytes / kernel_s / 1e9 / peaks["hbm_gbs"], "algorithmic_bytes": nbytes,
           "algorithmic_flops": flops, "t_hbm_us": t_hbm * 1e6, "t_tensor_us": t_tc * 1e6,
           "tensor_peak_tflops": tpeak}
    return roof, ctx


# --------------------------------------------------------------------------- ranks
def resolve_world(gpus, env):
    """How this process runs `--gpus gpus` given its environment `env`:
    ("run", world) inside a torchrun rank or for one GPU, ("spawn", gpus) to
    launch gpus local ranks, ("refuse", why) when they disagree."""
    if gpus < 1:
        return "refuse", f"--gpus {gpus}: need at least one GPU"
    ws = env.get("WORLD_SIZE")
    if ws is None:
        return ("spawn", gpus) if gpus > 1 else ("run", 1)
    if int(ws) != gpus:
        return "refuse", f"--gpus {gpus} but WORLD_SIZE={ws}: launch one rank per GPU"
    return "run", int(ws)


def spawn_ranks(n):
    """Re-run this command as n local ranks under torch.distributed.run."""
    import socket
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={n}",
           "--master-addr", "127.0.0.1", "--master-port", str(port),
           os.path.abspath(__file__), *sys.argv[1:]]
    return subprocess.call(cmd)


def combine_ranks(tokens, ms_total, per_call_ms, launches, device=None):
    """Whole-job figures from each rank's own: all ranks' tokens, the slowest
    rank's elapsed time and main-kernel time, every rank's launches."""
    from bidirectional_mamba_ssm_b200 import replicas
    tokens, ms_total, _ = replicas.aggregate(tokens, ms_total, device=device)
    _, per_call_ms, _ = replicas.aggregate(0, per_call_ms, device=device)
    launches, _, _ = replicas.aggregate(launches, 1.0, device=device)
    return tokens, ms_total, per_call_ms, int(launches)


# --------------------------------------------------------------------------- our arm
DECODE_SETS = 4   # state/input sets the timed decode steps rotate over (> L2 in all)


def build_step(lib, I, w, name, batch, seqlen, rank, dev):
    """Inputs on the device and the step closure of one workload.  A step
    takes `ev`, a (start, stop) pair of events (or None), and hands it to the
    library's timing hook around the call whose main kernel the roofline
    reports."""
    import torch
    H, P, N = w.heads, w.headdim, w.d_state
    decode = name == "decode"
    untied = name == "untied1p3b"
    g = I.make_inputs(w, seed=rank, device=dev, seqlen=seqlen, batch=batch,
                      conv_bias=name in ("decode", "decode_pool", "backward1p3b"))
    gr = I.make_inputs(w, seed=10000 + rank, device=dev, seqlen=seqlen, batch=batch) if untied else None
    adt = I.torch_dtype(w.dtype)
    y = torch.empty((batch, seqlen, (2 if untied else 1) * H * P), dtype=adt, device=dev)
    dims = lib.make_dims(batch, seqlen, H, P, N, adt)
    ws = lib.new_workspace(dims, device=dev)
    extra = {}

    def hook(ev):
        lib.bimamba_set_timing_events(*(ev if ev is not None else (None, None)))

    if decode:
        state, tail = decode_cache(lib, I, w, batch, I.DECODE_PREFIX, g, rank, dev)
        # Sets of (state, tail, block inputs, y) at distinct addresses: each
        # timed step reads the set the previous DECODE_SETS - 1 steps did not
        # touch, ~100 MB each, so its 64 MiB of cached state comes from HBM.
        sets = [(state, tail, g["xbc"], g["dt"], y)]
        for _ in range(DECODE_SETS - 1):
            sets.append((state.clone(), tail.clone(), g["xbc"].clone(), g["dt"].clone(),
                         torch.empty_like(y)))
        it = [0]
        extra.update(state=state, tail=tail)

        def step(ev=None):
            st, tl, xb, dtb, yy = sets[it[0] % DECODE_SETS]
            it[0] += 1
            hook(ev)
            lib.bimamba_block_decode(xb, dtb, g["A"], g["D"], g["conv_w"], g["conv_b"], st, tl, yy,
                                     None, None, ws, heads=H, headdim=P, d_state=N)
            hook(None)
    elif name == "decode_pool":
        # a pool of cached streams; each step decodes the next `batch` of them
        # (slots rotate through the pool, so the states come from HBM) and
        # commits every row's state and conv tail back in place
        pool = I.make_state(POOL_STREAMS, H, P, N, seed=50 + rank, scale=0.05, device=dev)
        tails = I.make_tail(POOL_STREAMS, 4, w.channels, "bf16", seed=51 + rank, bc_split=H * P,
                            bc_scale=w.bc_scale, device=dev)
        groups = POOL_STREAMS // batch
        slot_sets = [torch.arange(i * batch, (i + 1) * batch, dtype=torch.int32, device=dev)
                     for i in range(groups)]
        it = [0]

        def step(ev=None):
            sl = slot_sets[it[0] % groups]
            it[0] += 1
            hook(ev)
            lib.bimamba_block_decode_pool(g["xbc"], g["dt"], g["A"], g["D"], g["conv_w"], g["conv_b"],
                                          pool, tails, sl, None, y, ws, heads=H, headdim=P, d_state=N)
            hook(None)
    elif name == "mixer1p3b":
        tokens = batch * seqlen
        pr = I.make_projections(D_MODEL, H, P, N, tokens, seed=rank, device=dev)
        xbc = torch.empty((batch, seqlen, w.channels), dtype=torch.bfloat16, device=dev)
        dtv = torch.empty((batch, seqlen, H), dtype=torch.bfloat16, device=dev)
        out = torch.empty((tokens, D_MODEL), dtype=torch.bfloat16, device=dev)
        del pr["y"]
        extra.update(proj=pr)

        def step(ev=None):
            hook(ev)   # the in-projection GEMM is the roofline's kernel
            lib.bimamba_in_proj(pr["u"], pr["w_in"], pr["dt_bias"], xbc, dtv, heads=H, headdim=P,
                                d_state=N)
            hook(None)
            lib.bimamba_ssd_fwd_rev(xbc, dtv, g["A"], g["D"], g["conv_w"], None, None, None, y, ws,
                                    heads=H, headdim=P, d_state=N)
            lib.bimamba_out_proj(y.view(tokens, H * P), pr["w_out"], out)
    elif name == "backward1p3b":
        gen = torch.Generator(device=dev)
        gen.manual_seed(7 + rank)
        dyv = torch.randn((batch, seqlen, H * P), generator=gen, device=dev).to(torch.bfloat16)
        bws = torch.empty(max(256, lib.bimamba_backward_workspace_bytes(dims)), dtype=torch.uint8,
                          device=dev)
        extra.update(dy=dyv, bws=bws)

        def step(ev=None):
            hook(ev)   # the chunked adjoint kernel is the roofline's kernel
            lib.bimamba_ssd_fwd_rev_backward(g["xbc"], g["dt"], g["A"], g["D"], g["conv_w"],
                                             g["conv_b"], None, dyv, heads=H, headdim=P,
                                             d_state=N, workspace=bws)
            hook(None)
    elif untied:
        def step(ev=None):
            hook(ev)
            lib.bimamba_ssd_fwd_rev_untied(g, gr, None, None, y, ws, heads=H, headdim=P,
                                           d_state=N, concat=True)
            hook(None)
    else:
        def step(ev=None):
            hook(ev)
            lib.bimamba_ssd_fwd_rev(g["xbc"], g["dt"], g["A"], g["D"], g["conv_w"], None, None,
                                    None, y, ws, heads=H, headdim=P, d_state=N)
            hook(None)
    return step, g, gr, dims, ws, extra


def decode_cache(lib, I, w, streams, prefix, g, rank, dev, distinct=None):
    """The cached forward state and conv tail of `streams` streams, each from
    a forward scan over a seeded `prefix`-token prefix.  distinct = how many
    streams get their own prefix (the rest repeat them; the step's cost does
    not depend on the state's values); default all."""
    import torch
    H, P, N = w.heads, w.headdim, w.d_state
    state = torch.empty((streams, H, P, N), device=dev)
    tail = torch.empty((streams, 4, w.channels), dtype=torch.bfloat16, device=dev)
    pdims = lib.make_dims(1, prefix, H, P, N, torch.bfloat16)
    pws = lib.new_workspace(pdims, device=dev)
    py = torch.empty((1, prefix, H * P), dtype=torch.bfloat16, device=dev)
    k = streams if distinct is None else min(distinct, streams)
    for s in range(k):
        pre = I.make_inputs(w, seed=1000 + streams * rank + s, device=dev, seqlen=prefix, batch=1)
        lib.bimamba_ssd_fwd_rev(pre["xbc"], pre["dt"], g["A"], g["D"], g["conv_w"], g["conv_b"],
                                None, state[s:s + 1], py, pws, heads=H, headdim=P, d_state=N)
        tail[s] = pre["xbc"][0, -4:]
        del pre
    for s in range(k, streams):
        state[s] = state[s % k]
        tail[s] = tail[s % k]
    torch.cuda.synchronize()
    return state, tail


def time_steps(args, lib, step, stream, world, dev):
    """Warm-up, then exactly args.steps timed steps between barriers and
    synchronisations; CUDA events around the whole region and, through the
    library's timing hook, around each step's main kernel."""
    import torch
    import torch.distributed as dist
    t0 = time.time()
    n = 0
    while n < args.warmup or time.time() - t0 < 1.0:   # and >= ~1 s of load for the sampler
        step()
        n += 1
        if n % 10 == 0:
            torch.cuda.synchronize()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    kev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)]
    for a, b_ in kev:       # materialise the event handles before handing them over
        a.record(stream)
        b_.record(stream)
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    launches0 = lib.bimamba_launch_count()
    start.record(stream)
    for i in range(args.steps):
        step(kev[i])
    end.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    launches = lib.bimamba_launch_count() - launches0
    assert lib.bimamba_get_error() == lib.BIMAMBA_OK
    return start.elapsed_time(end), statistics.mean(a.elapsed_time(b_) for a, b_ in kev), launches


def measure(args, lib, I, name, rank, world, dev, gpu_id, want_e2e=True):
    """One workload's figures: whole-job tokens/s, the dominant kernel's
    roofline, clocks during the timed region, launches, and (want_e2e) the
    end-to-end figure through host buffers."""
    import torch
    stream = torch.cuda.current_stream()
    w, batch, seqlen = workload_spec(name)
    if args.batch is not None:
        batch = args.batch
    decode = name in ("decode", "decode_pool")
    untied = name == "untied1p3b"
    H, P, N = w.heads, w.headdim, w.d_state
    step, g, gr, dims, ws, extra = build_step(lib, I, w, name, batch, seqlen, rank, dev)
    torch.cuda.synchronize()
    assert lib.bimamba_get_error() == lib.BIMAMBA_OK
    sampler = ClockSampler(gpu_id)
    ms_total, per_call_ms, launches = time_steps(args, lib, step, stream, world, dev)
    clocks = sampler.stop()
    tokens = batch * seqlen
    tok_all, ms_total, per_call_ms, launches = combine_ranks(tokens * args.steps, ms_total,
                                                             per_call_ms, launches, device=dev)
    ms_step = ms_total / args.steps
    value = tok_all / args.steps / (ms_step / 1e3)
    peaks, peak_kind = load_peaks()
    nbytes, flops = algorithmic(w, batch, seqlen, decode, untied)
    kernel_file = "ssd_tc.cu" if (P, N) == (64, 128) else "scan_seq.cu"
    if decode:
        kernel_file = "decode_tc.cu"
    if name == "decode_pool":   # the commit writes every row's state and conv tail back
        nbytes += batch * (H * P * N * 4 + 4 * w.channels * 2)
    if name == "mixer1p3b":
        (nbytes, flops), _ = gemm_counts(w, batch * seqlen)
        kernel_file = "gemm_tc.cu"
    roof, ctx = roofline(peaks, peak_kind, clocks, nbytes, flops, per_call_ms / 1e3, decode,
                         kernel_file, name)
    if name == "backward1p3b":
        # the adjoint's products on tcgen05 (bf16 operands): held against the
        # bf16 tensor peak over the adjoint kernel's time
        nbytes, flops = backward_counts(w, batch * seqlen)
        roof, ctx = roofline(peaks, peak_kind, clocks, nbytes, flops, per_call_ms / 1e3, False,
                             "backward_tc.cu", name)
        ctx["note"] = ("flops: the adjoint's products at the Q = 64 convention over the adjoint "
                       "kernel's time; bytes: the whole call (conv, state pass, adjoint, conv backward)")
    if name == "decode":
        wl = (f"cached block decode: {batch} streams x {seqlen}-token block, H64x64 N128 bf16, "
              f"65536-token prefix state")
        l2 = (f"HBM-cold: steps rotate over {DECODE_SETS} sets of state + block inputs + y "
              f"(~{DECODE_SETS * 100} MB > 126 MB L2)")
    elif name == "decode_pool":
        wl = (f"pooled cached decode: {batch} of {POOL_STREAMS} cached streams per step x "
              f"{seqlen}-token block, H64x64 N128 bf16, every row's state and tail committed")
        l2 = (f"HBM-cold: consecutive steps take different slots of a {POOL_STREAMS * 2} MiB "
              f"state pool")
    elif name == "mixer1p3b":
        wl = (w.name + f", with its projections: in {D_MODEL}->{w.channels}+{H} (softplus dt), "
              f"mixer core, out {H * P}->{D_MODEL}")
        l2 = "inputs larger than L2"
    elif name == "backward1p3b":
        wl = (w.name + ", backward of the mixer core: gradients of xBC, dt, A, D, conv taps and "
              "bias from dy")
        l2 = "inputs larger than L2"
    elif name == "tiny":
        wl = w.name + " (launch-bound: the figure is the call's latency, not a roofline fraction)"
        l2 = "L2-resident (0.3 MB per call)"
        roof["note"] = "launch-bound small case: report latency (latency_us), no roofline claim"
    else:
        wl = w.name + (", untied directions, outputs concatenated" if untied else "")
        l2 = "inputs larger than L2 (xbc + y per step > 126 MB)"
    out = {"value": value, "ms_per_step": ms_step, "workload": wl, "batch_per_gpu": batch,
           "seqlen": seqlen, "l2": l2, "roofline": roof, "roofline_hbm_context": ctx,
           "clocks": clocks, "gpu_launches": launches, "main_kernel_ms": per_call_ms}
    if name == "tiny":
        out["latency_us"] = {"call": ms_step * 1e3, "kernel": per_call_ms * 1e3}
    if want_e2e and name == "backward1p3b":
        out["e2e"] = run_e2e_backward(args, lib, w, g, extra, dev)
    elif want_e2e:
        out["e2e"] = run_e2e(args, lib, w, name, g, batch, seqlen, dims, ws, extra, dev, world, gr)
    del step, g, gr, ws, extra
    torch.cuda.empty_cache()
    return out


def run_ours(args, world):
    import torch
    import torch.distributed as dist
    from datetime import timedelta

    from bidirectional_mamba_ssm_b200 import _lib as lib
    from bidirectional_mamba_ssm_b200 import inputs as I

    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        dist.init_process_group("nccl", timeout=timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local)
    uuid = str(torch.cuda.get_device_properties(dev).uuid)
    gpu_id = uuid if uuid.startswith("GPU-") else "GPU-" + uuid

    main_name = "long131k" if args.workload == "sweep" else args.workload
    m = measure(args, lib, I, main_name, rank, world, dev, gpu_id)
    w, _, _ = workload_spec(main_name)
    result = {
        "metric": METRIC, "value": m["value"], "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": m["ms_per_step"],
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": w.dtype,
        "data": "synthetic",
        "config": {"workload": m["workload"], "batch_per_gpu": m["batch_per_gpu"],
                   "seqlen": m["seqlen"], "heads": w.heads, "headdim": w.headdim,
                   "d_state": w.d_state, "state_dtype": "f32", "l2": m["l2"],
                   "parallelism": f"independent replicas x{world} (no data-path collective)"},
        "roofline": m["roofline"], "roofline_hbm_context": m["roofline_hbm_context"],
        "e2e": m["e2e"], "clocks": m["clocks"], "gpu_launches": m["gpu_launches"],
    }
    if "latency_us" in m:
        result["latency_us"] = m["latency_us"]
    if args.workload == "long131k" and args.batch is None:
        # the 1.3B-layer workload (b8 x L4096) measured in the same run
        lm = measure(args, lib, I, "layer1p3b", rank, world, dev, gpu_id, want_e2e=False)
        result["layer1p3b"] = {k: lm[k] for k in ("value", "ms_per_step", "workload",
                                                  "batch_per_gpu", "seqlen", "roofline",
                                                  "clocks", "gpu_launches")}
    if args.workload == "sweep":
        result["config"]["workload"] = (m["workload"] + f"; plus a sweep of one sequence, prefill "
                                        f"and 32-stream 64-token cached decode at "
                                        f"{SWEEP_LENGTHS[0]}..{SWEEP_LENGTHS[-1]} tokens")
        result["sweep"] = run_sweep(args, lib, w, dev, rank, gpu_id)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        result["cpu_baseline"] = cpu_baseline(w, main_name)
    if rank == 0:
        print(json.dumps(result), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def run_sweep(args, lib, w, dev, rank, gpu_id):
    """Per context length L: the prefill (one L-token sequence through
    bimamba_ssd_fwd_rev) and one cached 64-token block decode step of 32
    streams whose state came from a forward scan over an L-token prefix.
    The prefill's cost should grow linearly in L (flat per token), the
    decode step's not at all (the cached state is O(1) in L).  Every timed
    call starts with L2 flushed (a 256 MB write between calls, outside the
    timed region), so the short lengths, whose inputs would fit in L2, are
    timed cold like the long ones; the figure is the median of the calls."""
    import torch
    from bidirectional_mamba_ssm_b200 import inputs as I
    H, P, N = w.heads, w.headdim, w.d_state
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()
    S, blk = I.DECODE_STREAMS, I.DECODE_BLOCK
    dw, _, _ = workload_spec("decode")
    gd = I.make_inputs(dw, seed=rank, device=dev, seqlen=blk, batch=S, conv_bias=True)
    yd = torch.empty((S, blk, H * P), dtype=torch.bfloat16, device=dev)
    wsd = lib.new_workspace(lib.make_dims(S, blk, H, P, N, torch.bfloat16), device=dev)
    peaks, _ = load_peaks()
    sampler = ClockSampler(gpu_id)

    def cold_median(call):
        for _ in range(max(3, args.warmup)):
            call()
        times = []
        for _ in range(max(5, min(args.steps, 20))):
            flush.fill_(1)
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record(stream)
            call()
            b.record(stream)
            b.synchronize()
            times.append(a.elapsed_time(b))
        assert lib.bimamba_get_error() == lib.BIMAMBA_OK
        return statistics.median(times)

    rows = []
    for L in SWEEP_LENGTHS:
        g = I.make_inputs(w, seed=7, device=dev, seqlen=L, batch=1)
        y = torch.empty((1, L, H * P), dtype=torch.bfloat16, device=dev)
        ws = lib.new_workspace(lib.make_dims(1, L, H, P, N, torch.bfloat16), device=dev)
        ms = cold_median(lambda: lib.bimamba_ssd_fwd_rev(
            g["xbc"], g["dt"], g["A"], g["D"], g["conv_w"], None, None, None, y, ws, heads=H,
            headdim=P, d_state=N))
        del g, y, ws
        torch.cuda.empty_cache()
        # cached state after an L-token prefix (two distinct prefixes, repeated over the streams)
        state, tail = decode_cache(lib, I, dw, S, L, gd, rank, dev, distinct=2)
        dms = cold_median(lambda: lib.bimamba_block_decode(
            gd["xbc"], gd["dt"], gd["A"], gd["D"], gd["conv_w"], gd["conv_b"], state, tail, yd,
            None, None, wsd, heads=H, headdim=P, d_state=N))
        del state, tail
        torch.cuda.empty_cache()
        _, flops = algorithmic(w, 1, L)
        dbytes, _ = algorithmic(dw, S, blk, decode=True)
        plan = lib.bimamba_launch_plan(lib.make_dims(1, L, H, P, N, torch.bfloat16))
        rows.append({"seqlen": L, "ms_per_step": ms, "ns_per_token": ms * 1e6 / L,
                     "tokens_per_s": L / (ms / 1e3), "flops": flops,
                     "segments": plan["segments"], "state_only_items": plan["items"],
                     "decode_ms_per_step": dms, "decode_tokens_per_s": S * blk / (dms / 1e3),
                     "decode_hbm_frac": dbytes / (dms / 1e3) / 1e9 / peaks["hbm_gbs"]})
    clocks = sampler.stop()
    tpeak, rule = tensor_peak(peaks, clocks)
    for r in rows:
        r["tensor_frac"] = r.pop("flops") / (r["ms_per_step"] / 1e3) / 1e12 / tpeak
        r["tensor_peak_rule"] = rule
    return rows


def run_e2e_backward(args, lib, w, g, extra, dev):
    """The backward through the public API from pinned host buffers: every
    step uploads xBC, dt and dy, runs the call and reads d(xBC) back (one
    stream, not pipelined)."""
    import torch
    H, P, N = w.heads, w.headdim, w.d_state
    hin = [t.cpu().pin_memory() for t in (g["xbc"], g["dt"], extra["dy"])]
    din = [torch.empty_like(t, device=dev) for t in hin]
    hout = torch.empty(g["xbc"].shape, dtype=torch.float32).pin_memory()

    def step():
        for dst, src in zip(din, hin):
            dst.copy_(src, non_blocking=True)
        gr = lib.bimamba_ssd_fwd_rev_backward(din[0], din[1], g["A"], g["D"], g["conv_w"], g["conv_b"],
                                              None, din[2], heads=H, headdim=P, d_state=N,
                                              workspace=extra["bws"])
        hout.copy_(gr["xbc"], non_blocking=True)

    for _ in range(max(1, args.warmup)):
        step()
    torch.cuda.synchronize()
    steps = max(1, args.e2e_steps)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record()
    for _ in range(steps):
        step()
    end.record()
    torch.cuda.synchronize()
    ms = start.elapsed_time(end) / steps
    tokens = g["xbc"].shape[0] * g["xbc"].shape[1]
    return {"value": tokens / (ms / 1e3), "unit": "tokens/s",
            "h2d_bytes_per_step": sum(t.numel() * t.element_size() for t in hin),
            "d2h_bytes_per_step": hout.numel() * hout.element_size(), "ms_per_step": ms}


def run_e2e(args, lib, w, name, g, batch, seqlen, dims, ws, extra, dev, world, gr=None):
    """Same metric through the public API from pinned HOST buffers.  Every step
    copies its inputs host->device (the raw xbc and dt of each stream; the
    layer input u for the workload with projections), runs the call(s), and
    copies the result (y, or the layer output) back to the host.  Steps are
    pipelined the way a serving loop would run them: step i+1's upload, step
    i's kernels and step i-1's download run on three streams with two device
    buffer sets, ordered by events."""
    import torch
    H, P, N = w.heads, w.headdim, w.d_state
    untied = gr is not None
    tokens = batch * seqlen
    if name == "mixer1p3b":
        pr = extra["proj"]
        hin = [pr["u"].cpu().pin_memory()]
        out_shape = (tokens, D_MODEL)
        mid = [(torch.empty((batch, seqlen, w.channels), dtype=torch.bfloat16, device=dev),
                torch.empty((batch, seqlen, H), dtype=torch.bfloat16, device=dev),
                torch.empty((batch, seqlen, H * P), dtype=torch.bfloat16, device=dev)) for _ in range(2)]
    else:
        srcs = [g] + ([gr] if untied else [])
        hin = [t.cpu().pin_memory() for d in srcs for t in (d["xbc"], d["dt"])]
        out_shape = (batch, seqlen, (2 if untied else 1) * H * P)
    if name == "decode_pool":
        pool = I_make_pool(w, dev)
        slot_sets = [torch.arange(i * batch, (i + 1) * batch, dtype=torch.int32, device=dev)
                     for i in range(POOL_STREAMS // batch)]
    odt = torch.float32 if w.dtype == "f32" else torch.bfloat16
    hy = torch.empty(out_shape, dtype=odt).pin_memory()
    din = [[torch.empty_like(t, device=dev) for t in hin] for _ in range(2)]
    dy = [torch.empty(out_shape, dtype=odt, device=dev) for _ in range(2)]
    wss = [ws, lib.new_workspace(dims, device=dev)]
    s_up, s_run, s_down = (torch.cuda.Stream(device=dev) for _ in range(3))
    up_done = [torch.cuda.Event() for _ in range(2)]
    run_done = [torch.cuda.Event() for _ in range(2)]
    down_done = [torch.cuda.Event() for _ in range(2)]
    for e in run_done + down_done:
        e.record(torch.cuda.current_stream())
    kw = dict(heads=H, headdim=P, d_state=N, stream=s_run)

    def step(i):
        j = i & 1
        s_up.wait_event(run_done[j])            # buffers j free once step i-2 has run
        with torch.cuda.stream(s_up):
            for dst, src in zip(din[j], hin):
                dst.copy_(src, non_blocking=True)
        up_done[j].record(s_up)
        s_run.wait_event(up_done[j])
        s_run.wait_event(down_done[j])          # output buffer j read back by step i-2
        if name == "mixer1p3b":
            xb, dtb, yb = mid[j]
            lib.bimamba_in_proj(din[j][0], pr["w_in"], pr["dt_bias"], xb, dtb, heads=H, headdim=P,
                                d_state=N, stream=s_run)
            lib.bimamba_ssd_fwd_rev(xb, dtb, g["A"], g["D"], g["conv_w"], None, None, None, yb,
                                    wss[j], **kw)
            lib.bimamba_out_proj(yb.view(tokens, H * P), pr["w_out"], dy[j], stream=s_run)
        elif name == "decode":
            lib.bimamba_block_decode(din[j][0], din[j][1], g["A"], g["D"], g["conv_w"], g["conv_b"],
                                     extra["state"], extra["tail"], dy[j], None, None, wss[j], **kw)
        elif name == "decode_pool":
            lib.bimamba_block_decode_pool(din[j][0], din[j][1], g["A"], g["D"], g["conv_w"],
                                          g["conv_b"], pool[0], pool[1],
                                          slot_sets[i % len(slot_sets)], None, dy[j], wss[j], **kw)
        elif untied:
            fwd = dict(g, xbc=din[j][0], dt=din[j][1])
            rev = dict(gr, xbc=din[j][2], dt=din[j][3])
            lib.bimamba_ssd_fwd_rev_untied(fwd, rev, None, None, dy[j], wss[j], concat=True, **kw)
        else:
            lib.bimamba_ssd_fwd_rev(din[j][0], din[j][1], g["A"], g["D"], g["conv_w"], None, None,
                                    None, dy[j], wss[j], **kw)
        run_done[j].record(s_run)
        s_down.wait_event(run_done[j])
        with torch.cuda.stream(s_down):
            hy.copy_(dy[j], non_blocking=True)
        down_done[j].record(s_down)

    for i in range(2):
        step(i)
    torch.cuda.synchronize()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record(s_up)
    for i in range(args.e2e_steps):
        step(i)
    s_up.wait_stream(s_down)
    b.record(s_up)
    torch.cuda.synchronize()
    ms = a.elapsed_time(b) / args.e2e_steps
    from bidirectional_mamba_ssm_b200 import replicas
    _, ms, _ = replicas.aggregate(0, ms, device=dev)
    h2d = sum(t.numel() * t.element_size() for t in hin)
    d2h = hy.numel() * hy.element_size()
    return {"value": batch * seqlen * world / (ms / 1e3), "unit": "tokens/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": ms,
            "pipelined": "upload / kernels / download overlapped across steps (3 streams)"}


def I_make_pool(w, dev):
    """A pool of POOL_STREAMS cached streams (seeded states and conv tails)."""
    from bidirectional_mamba_ssm_b200 import inputs as I
    pool = I.make_state(POOL_STREAMS, w.heads, w.headdim, w.d_state, seed=60, scale=0.05, device=dev)
    tails = I.make_tail(POOL_STREAMS, 4, w.channels, "bf16", seed=61, bc_split=w.heads * w.headdim,
                        bc_scale=w.bc_scale, device=dev)
    return pool, tails


# --------------------------------------------------------------------------- CPU oracle
def oracle_sample_step(w, workload, seq_tokens, seed=0):
    """Run the oracle once on one sequence prefix of `seq_tokens` tokens of
    the workload (all heads, both directions, conv fused; with the
    projections for the layer workload); return seconds."""
    import numpy as np
    import oracle
    from bidirectional_mamba_ssm_b200 import inputs as I
    decode = workload in ("decode", "decode_pool")
    cpu = I.make_inputs(w, seed=seed, seqlen=seq_tokens, batch=1,
                        conv_bias=decode or workload == "backward1p3b")
    n = {k: (None if v is None else v.float().double().numpy()) for k, v in cpu.items()}
    kw = dict(heads=w.heads, headdim=w.headdim, d_state=w.d_state)
    if workload == "untied1p3b":
        cr = I.make_inputs(w, seed=seed + 10000, seqlen=seq_tokens, batch=1)
        r = {k: (None if v is None else v.float().double().numpy()) for k, v in cr.items()}
    if workload == "mixer1p3b":
        pr = I.make_projections(D_MODEL, w.heads, w.headdim, w.d_state, seq_tokens, seed=seed)
    t0 = time.perf_counter()
    if workload == "untied1p3b":
        oracle.bimamba_untied(n["xbc"], r["xbc"], n["dt"], r["dt"], n["A"], r["A"], n["D"], r["D"],
                              n["conv_w"], r["conv_w"], None, None, concat=True, **kw)
    elif workload == "mixer1p3b":
        xbc, dt = oracle.in_proj(pr["u"], pr["w_in"], pr["dt_bias"], **kw)
        y = oracle.bimamba(xbc[None], dt[None], n["A"], n["D"], n["conv_w"], None, **kw)
        oracle.out_proj(y[0], pr["w_out"])
    elif workload == "backward1p3b":
        dy = np.random.default_rng(seed).standard_normal((1, seq_tokens, w.heads * w.headdim))
        oracle.bimamba_mixer_backward(n["xbc"], n["dt"], n["A"], n["D"], n["conv_w"], n["conv_b"], dy,
                                      **kw)
    elif decode:
        state = np.zeros((1, w.heads, w.headdim, w.d_state))
        tail = np.zeros((1, 4, w.channels))
        oracle.block_decode(n["xbc"], n["dt"], n["A"], n["D"], n["conv_w"], n["conv_b"], state,
                            tail, want_commit=workload == "decode_pool", **kw)
    else:
        oracle.bimamba(n["xbc"], n["dt"], n["A"], n["D"], n["conv_w"], None, **kw)
    return time.perf_counter() - t0


def cpu_baseline(w, workload):
    """The oracle, as it stands, on host cores: whole sequences of the
    workload's length (capped at 4096 tokens) until ~10 s of CPU time."""
    import oracle
    seq = (64 if workload in ("decode", "decode_pool", "backward1p3b")
           else (256 if workload == "tiny" else 1024))
    tokens, secs, reps = 0, 0.0, 0
    while secs < 10.0 and reps < 64:
        secs += oracle_sample_step(w, workload, seq, seed=reps)
        tokens += seq
        reps += 1
    return {"value": tokens / secs, "unit": "tokens/s", "cores": oracle.num_threads(),
            "kind": "oracle",
            "sample": f"{reps} sequence(s) x {seq} tokens of the workload, all {w.heads} heads, "
                      f"both directions, conv fused; double precision; {secs:.1f} s"}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle
    w, batch, seqlen = workload_spec(args.workload)
    seq = 64 if args.workload in ("decode", "decode_pool", "backward1p3b") else 256
    for i in range(args.warmup):
        oracle_sample_step(w, args.workload, seq, seed=i)
    total = 0.0
    for i in range(args.steps):
        total += oracle_sample_step(w, args.workload, seq, seed=100 + i)
    ms = total / args.steps * 1e3
    value = seq / (ms / 1e3)
    cores = oracle.num_threads()
    sample = (f"one sequence x {seq} tokens of the workload per step (all {w.heads} heads, both "
              f"directions, conv fused), double precision")
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": int(os.environ.get("WORLD_SIZE", "1")), "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": {"decode": "cached block decode",
                                "decode_pool": "pooled cached decode",
                                "untied1p3b": w.name + ", untied directions, outputs concatenated",
                                "mixer1p3b": w.name + ", with its in/out projections",
                                "backward1p3b": w.name + ", backward of the mixer core"}
                   .get(args.workload, w.name),
                   "batch_per_gpu": batch, "seqlen": seqlen, "heads": w.heads,
                   "headdim": w.headdim, "d_state": w.d_state},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }), flush=True)


def main():
    args = parse_args()
    if args.impl == "reference":
        run_reference(args)
        return
    how, arg = resolve_world(args.gpus, os.environ)
    if how == "refuse":
        print(f"bench.py: {arg}", file=sys.stderr)
        sys.exit(2)
    if how == "spawn":
        sys.exit(spawn_ranks(arg))
    run_ours(args, arg)


if __name__ == "__main__":
    main()
