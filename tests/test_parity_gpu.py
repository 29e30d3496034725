"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle.

Small cases span several chunks/tiles and a ragged tail; the full-size
workloads run in the launch configuration the benchmark times and are
compared on sampled heads / streams that the oracle computes in seconds.
Every case with a learned-looking decay range also runs with long-memory
decays (A in [-1e-2, -1e-3]) so that cross-chunk state errors cannot hide.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from bidirectional_mamba_ssm_b200 import inputs as inp_mod
from parity_util import TOL, head_subset, rel_err, to_np, y_cols

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lib():
    from bidirectional_mamba_ssm_b200 import _lib
    return _lib


def _dev(d):
    return {k: (None if v is None else v.cuda()) for k, v in d.items()}


def _np_inputs(d):
    return {k: to_np(v) for k, v in d.items()}


def _run_scan(lib, w, g, init=None, want_final=False):
    bsz, L, _ = g["xbc"].shape
    H, P, N = w.heads, w.headdim, w.d_state
    y = torch.full((bsz, L, H * P), float("nan"), dtype=g["xbc"].dtype, device="cuda")
    fin = torch.full((bsz, H, P, N), float("nan"), device="cuda") if want_final else None
    dims = lib.make_dims(bsz, L, H, P, N, g["xbc"].dtype)
    ws = lib.new_workspace(dims)
    lib.bimamba_ssd_fwd_rev(g["xbc"], g["dt"], g["A"], g["D"], g["conv_w"], g["conv_b"], init,
                            fin, y, ws, heads=H, headdim=P, d_state=N)
    assert lib.bimamba_get_error() == lib.BIMAMBA_OK
    return y, fin


# ----------------------------------------------------------------- conv
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("rev", [False, True])
@pytest.mark.parametrize("use_tail", [False, True])
@pytest.mark.parametrize("L", [1, 3, 37, 130])
def test_conv_index_logic_bit_exact(lib, dtype, rev, use_tail, L):
    """Integer inputs and taps, identity activation: every sum is exact in
    fp32 and bf16, so the padding / tap order / reflection must match the
    oracle bit for bit."""
    if rev and use_tail:
        pytest.skip("the tail is forward-only")
    g = torch.Generator().manual_seed(L * 7 + rev)
    bsz, ch = 2, 48
    td = inp_mod.torch_dtype(dtype)
    u = torch.randint(-8, 9, (bsz, L, ch), generator=g).to(td)
    w = torch.randint(-2, 3, (ch, 4), generator=g).float()
    bias = torch.randint(-3, 4, (ch,), generator=g).float()
    tail = torch.randint(-8, 9, (bsz, 4, ch), generator=g).to(td) if use_tail else None
    out = torch.empty_like(u, device="cuda")
    lib.bimamba_conv_silu(u.cuda(), out, w.cuda(), bias.cuda(),
                          None if tail is None else tail.cuda(), reverse=rev, silu=False)
    ref = oracle.conv(u, w, bias, tail=tail, reverse=rev, silu=False)
    np.testing.assert_array_equal(to_np(out), ref)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("rev", [False, True])
def test_conv_silu_values(lib, dtype, rev):
    g = torch.Generator().manual_seed(3)
    td = inp_mod.torch_dtype(dtype)
    u = torch.randn((3, 200, 72), generator=g).to(td)
    w = torch.randn((72, 4), generator=g) * 0.5
    b = torch.randn((72,), generator=g) * 0.1
    out = torch.empty_like(u, device="cuda")
    lib.bimamba_conv_silu(u.cuda(), out, w.cuda(), b.cuda(), reverse=rev, silu=True)
    ref = oracle.conv(u, w, b, reverse=rev, silu=True)
    assert rel_err(to_np(out), ref) <= (1e-6 if dtype == "f32" else 8e-3)


# ----------------------------------------------------------------- scan
SMALL = [
    # dtype, batch, L, H, P, N
    ("f32", 1, 256, 4, 32, 16),     # the tiny fp32 workload's shape
    ("f32", 2, 129, 3, 16, 32),
    ("f32", 1, 1, 2, 8, 8),
    ("bf16", 2, 300, 4, 64, 128),   # several 64/128-token chunks + ragged tail
    ("bf16", 1, 127, 2, 64, 128),
    ("bf16", 3, 65, 2, 64, 128),
    ("bf16", 1, 2, 2, 64, 128),
    ("bf16", 2, 520, 3, 64, 64),
    ("bf16", 1, 200, 2, 32, 128),
]


@pytest.mark.parametrize("case", SMALL, ids=lambda c: "-".join(map(str, c)))
@pytest.mark.parametrize("memory", ["short", "long"])
@pytest.mark.parametrize("variant", ["conv", "conv+bias+init", "noconv"])
def test_scan_small(lib, case, memory, variant):
    dtype, bsz, L, H, P, N = case
    w = inp_mod.Workload("t", bsz, L, H, P, N, dtype=dtype,
                         bc_scale=1.0 if dtype == "f32" else 1.0 / math.sqrt(N))
    a = (1.0, 16.0) if memory == "short" else (1e-3, 1e-2)
    cpu = inp_mod.make_inputs(w, seed=L + H, a_range=a, conv_bias="bias" in variant)
    if variant == "noconv":
        cpu["conv_w"] = None
        cpu["conv_b"] = None
    init = inp_mod.make_state(bsz, H, P, N, seed=9, scale=0.5) if "init" in variant else None
    y, fin = _run_scan(lib, w, _dev(cpu), None if init is None else init.cuda(), want_final=True)
    n = _np_inputs(cpu)
    ry, rfin = oracle.bimamba(n["xbc"], n["dt"], n["A"], n["D"], n["conv_w"], n["conv_b"],
                              heads=H, headdim=P, d_state=N, init=to_np(init), want_final=True)
    tol = TOL[dtype]
    for b in range(bsz):
        assert rel_err(to_np(y)[b], ry[b]) <= tol, b
        assert rel_err(to_np(fin)[b], rfin[b]) <= tol, b


def test_tiny_f32_workload(lib):
    w = inp_mod.TINY_F32
    cpu = inp_mod.make_inputs(w, seed=0)
    y, fin = _run_scan(lib, w, _dev(cpu), want_final=True)
    n = _np_inputs(cpu)
    ry, rfin = oracle.bimamba(n["xbc"], n["dt"], n["A"], n["D"], n["conv_w"], None, heads=w.heads,
                              headdim=w.headdim, d_state=w.d_state, want_final=True)
    assert rel_err(to_np(y), ry) <= TOL["f32"]
    assert rel_err(to_np(fin), rfin) <= TOL["f32"]


def _sampled_full_size(lib, w, heads, batches, seed=0):
    cpu = inp_mod.make_inputs(w, seed=seed)
    y, fin = _run_scan(lib, w, _dev(cpu), want_final=True)
    y = y.cpu()
    fin = fin.cpu()
    n = _np_inputs({k: v for k, v in cpu.items()})
    sub, _ = head_subset(n, heads, w.heads, w.headdim, w.d_state)
    cols = y_cols(heads, w.headdim)
    for b in batches:
        ry, rfin = oracle.bimamba(sub["xbc"][b:b + 1], sub["dt"][b:b + 1], sub["A"], sub["D"],
                                  sub["conv_w"], None, heads=len(heads), headdim=w.headdim,
                                  d_state=w.d_state, want_final=True)
        got = to_np(y[b:b + 1])[..., cols]
        assert rel_err(got, ry) <= TOL[w.dtype], (b, rel_err(got, ry))
        assert rel_err(to_np(fin[b:b + 1, heads]), rfin) <= TOL[w.dtype]


def test_layer_1p3b_sampled_heads(lib):
    """b8 L4096 H64x64 N128 bf16, as benchmarked; 3 heads x 8 sequences checked."""
    _sampled_full_size(lib, inp_mod.LAYER_1P3B, heads=[0, 29, 63], batches=range(8))


@pytest.mark.slow
def test_long_131k_sampled_heads(lib):
    """b1 L131072 bf16; 2 heads checked over the whole sequence."""
    _sampled_full_size(lib, inp_mod.LONG_131K, heads=[5, 50], batches=[0])


def test_empty_sequence_passes_state_through(lib):
    H, P, N = 2, 64, 128
    init = inp_mod.make_state(2, H, P, N, seed=4).cuda()
    fin = torch.full_like(init, float("nan"))
    dims = lib.make_dims(2, 0, H, P, N, torch.bfloat16)
    e = torch.empty(16, dtype=torch.bfloat16, device="cuda")
    f = torch.zeros(H, device="cuda")
    lib.bimamba_ssd_fwd_rev(e, e, f, f, None, None, init, fin, e, lib.new_workspace(dims),
                            heads=H, headdim=P, d_state=N, dims=dims)
    torch.cuda.synchronize()
    assert torch.equal(fin, init)
    lib.bimamba_ssd_fwd_rev(e, e, f, f, None, None, None, fin, e, lib.new_workspace(dims),
                            heads=H, headdim=P, d_state=N, dims=dims)
    torch.cuda.synchronize()
    assert torch.count_nonzero(fin).item() == 0


# ----------------------------------------------------------------- decode
def _decode_case(lib, dtype, S, blk, prefix, H, P, N, a, commit=True, seed=0):
    w = inp_mod.Workload("d", S, prefix + blk, H, P, N, dtype=dtype,
                         bc_scale=1.0 if dtype == "f32" else 1.0 / math.sqrt(N))
    cpu = inp_mod.make_inputs(w, seed=seed, a_range=a, conv_bias=True)
    n = _np_inputs(cpu)
    ch = w.channels
    # prefix summary from the oracle: forward state and the last 4 raw tokens
    if prefix:
        _, state = oracle.bimamba(n["xbc"][:, :prefix], n["dt"][:, :prefix], n["A"], n["D"],
                                  n["conv_w"], n["conv_b"], heads=H, headdim=P, d_state=N,
                                  want_final=True)
    else:
        state = np.zeros((S, H, P, N))
    tail = np.zeros((S, 4, ch))
    k = min(prefix, 4)
    if k:
        tail[:, 4 - k:] = n["xbc"][:, prefix - k:prefix]
    td = inp_mod.torch_dtype(dtype)
    blk_x = cpu["xbc"][:, prefix:].contiguous().cuda()
    blk_dt = cpu["dt"][:, prefix:].contiguous().cuda()
    st_t = torch.from_numpy(state).float().cuda()
    tail_t = torch.from_numpy(tail).to(td).cuda()
    y = torch.full((S, blk, H * P), float("nan"), dtype=td, device="cuda")
    so = torch.full_like(st_t, float("nan")) if commit else None
    to = torch.zeros_like(tail_t) if commit else None
    dims = lib.make_dims(S, blk, H, P, N, td)
    lib.bimamba_block_decode(blk_x, blk_dt, cpu["A"].cuda(), cpu["D"].cuda(), cpu["conv_w"].cuda(),
                             cpu["conv_b"].cuda(), st_t, tail_t, y, so, to,
                             lib.new_workspace(dims), heads=H, headdim=P, d_state=N)
    assert lib.bimamba_get_error() == lib.BIMAMBA_OK
    ry, rso, rto = oracle.block_decode(n["xbc"][:, prefix:], n["dt"][:, prefix:], n["A"], n["D"],
                                       n["conv_w"], n["conv_b"], state, to_np(tail_t), heads=H,
                                       headdim=P, d_state=N, want_commit=True)
    tol = TOL[dtype]
    for s in range(S):
        assert rel_err(to_np(y)[s], ry[s]) <= tol
        if commit:
            assert rel_err(to_np(so)[s], rso[s]) <= tol
    if commit:
        np.testing.assert_array_equal(to_np(to), rto)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("blk,prefix", [(64, 200), (64, 0), (17, 2), (3, 70), (130, 9)])
@pytest.mark.parametrize("memory", ["short", "long"])
def test_block_decode_small(lib, dtype, blk, prefix, memory):
    a = (1.0, 16.0) if memory == "short" else (1e-3, 1e-2)
    P, N = (32, 16) if dtype == "f32" else (64, 128)
    _decode_case(lib, dtype, 3, blk, prefix, 2, P, N, a)


def test_block_decode_without_commit(lib):
    _decode_case(lib, "bf16", 2, 64, 100, 2, 64, 128, (1e-3, 1e-2), commit=False)


def test_block_decode_32_streams_65k_prefix_sampled(lib):
    """32 streams x 64-token block x 64 heads, bf16, as benchmarked.  Streams
    (3, 30) x heads (7, 40) carry a state the oracle computed over a seeded
    65536-token prefix; the rest carry seeded random states."""
    w = inp_mod.LAYER_1P3B
    S, blk, pre = inp_mod.DECODE_STREAMS, inp_mod.DECODE_BLOCK, inp_mod.DECODE_PREFIX
    H, P, N = w.heads, w.headdim, w.d_state
    blk_in = inp_mod.make_inputs(w, seed=0, seqlen=blk, batch=S, conv_bias=True)
    state = inp_mod.make_state(S, H, P, N, seed=3, scale=0.05)
    tail = inp_mod.make_tail(S, 4, w.channels, "bf16", seed=4, bc_split=H * P, bc_scale=w.bc_scale)
    heads, streams = [7, 40], [3, 30]
    n_blk = _np_inputs(blk_in)
    sub, _ = head_subset(n_blk, heads, H, P, N)
    for s in streams:
        pw = inp_mod.Workload("prefix", 1, pre, len(heads), P, N, dtype="bf16", bc_scale=w.bc_scale)
        pin = _np_inputs(inp_mod.make_inputs(pw, seed=100 + s))
        act = oracle.conv(pin["xbc"], sub["conv_w"], sub["conv_b"])
        x = act[..., :len(heads) * P].reshape(1, pre, len(heads), P)
        Bm = act[..., len(heads) * P:len(heads) * P + N].reshape(1, pre, 1, N)
        Cm = act[..., len(heads) * P + N:].reshape(1, pre, 1, N)
        _, fin = oracle.scan(x, Bm, Cm, pin["dt"], sub["A"], sub["D"], want_final=True)
        state[s, heads] = torch.from_numpy(fin[0]).float()
        # conv tail: the prefix's last 4 raw tokens on the sampled channels
        t = tail[s].float().numpy()
        cols = np.concatenate([np.concatenate([np.arange(h * P, (h + 1) * P) for h in heads]),
                               np.arange(H * P, H * P + 2 * N)])
        t[:, cols] = pin["xbc"][0, -4:]
        tail[s] = torch.from_numpy(t).to(torch.bfloat16)
    g = _dev(blk_in)
    st_d, tail_d = state.cuda(), tail.cuda()
    y = torch.full((S, blk, H * P), float("nan"), dtype=torch.bfloat16, device="cuda")
    so = torch.empty_like(st_d)
    to = torch.empty_like(tail_d)
    dims = lib.make_dims(S, blk, H, P, N, torch.bfloat16)
    lib.bimamba_block_decode(g["xbc"], g["dt"], g["A"], g["D"], g["conv_w"], g["conv_b"], st_d,
                             tail_d, y, so, to, lib.new_workspace(dims), heads=H, headdim=P,
                             d_state=N)
    assert lib.bimamba_get_error() == lib.BIMAMBA_OK
    ycols = y_cols(heads, P)
    n_tail = to_np(tail)
    for s in streams:
        tcols = np.concatenate([ycols, np.arange(H * P, H * P + 2 * N)])
        ry, rso, _ = oracle.block_decode(sub["xbc"][s:s + 1], sub["dt"][s:s + 1], sub["A"],
                                         sub["D"], sub["conv_w"], sub["conv_b"],
                                         to_np(state[s:s + 1, heads]), n_tail[s:s + 1][..., tcols],
                                         heads=len(heads), headdim=P, d_state=N, want_commit=True)
        assert rel_err(to_np(y[s:s + 1])[..., ycols], ry) <= TOL["bf16"]
        assert rel_err(to_np(so[s:s + 1, heads]), rso) <= TOL["bf16"]
    np.testing.assert_array_equal(to_np(to), to_np(blk_in["xbc"][:, -4:]))


# ------------------------------------------------- tensor-core path edges
TC_EDGES = [1, 3, 64, 128, 129, 255, 256, 257]


@pytest.mark.parametrize("L", TC_EDGES)
@pytest.mark.parametrize("variant", ["plain", "init+bias"])
def test_tensor_core_path_chunk_boundaries(lib, L, variant):
    """bf16, headdim 64, d_state 128 (the chunked tensor-core kernel) at
    lengths around the 128-token chunk size, long-memory decays so that
    state carried across chunk boundaries dominates."""
    bsz, H, P, N = 2, 4, 64, 128
    w = inp_mod.Workload("edge", bsz, L, H, P, N, dtype="bf16", bc_scale=1.0 / math.sqrt(N))
    cpu = inp_mod.make_inputs(w, seed=1000 + L, a_range=(1e-3, 1e-2), conv_bias="bias" in variant)
    init = inp_mod.make_state(bsz, H, P, N, seed=L, scale=0.3) if "init" in variant else None
    y, fin = _run_scan(lib, w, _dev(cpu), None if init is None else init.cuda(), want_final=True)
    n = _np_inputs(cpu)
    ry, rfin = oracle.bimamba(n["xbc"], n["dt"], n["A"], n["D"], n["conv_w"], n["conv_b"],
                              heads=H, headdim=P, d_state=N, init=to_np(init), want_final=True)
    for b in range(bsz):
        assert rel_err(to_np(y)[b], ry[b]) <= TOL["bf16"], (L, b)
        assert rel_err(to_np(fin)[b], rfin[b]) <= TOL["bf16"], (L, b)


def test_odd_head_count_uses_a_valid_path(lib):
    """Three heads cannot be paired: the library must still compute it."""
    w = inp_mod.Workload("odd", 1, 150, 3, 64, 128, dtype="bf16", bc_scale=1.0 / math.sqrt(128))
    cpu = inp_mod.make_inputs(w, seed=3)
    y, _ = _run_scan(lib, w, _dev(cpu))
    n = _np_inputs(cpu)
    ry = oracle.bimamba(n["xbc"], n["dt"], n["A"], n["D"], n["conv_w"], None, heads=3,
                        headdim=64, d_state=128)
    assert rel_err(to_np(y), ry) <= TOL["bf16"]


@pytest.mark.parametrize("blk,prefix", [(1, 5), (128, 300), (200, 64), (900, 100)])
def test_block_decode_multi_chunk_blocks(lib, blk, prefix):
    """Decode blocks of 1, 128, 200 and 900 tokens (one, one full, two and
    eight chunks; the 900-token block is walked as segments, so the cached
    state, the conv tail and the commit meet segment boundaries)."""
    _decode_case(lib, "bf16", 2, blk, prefix, 4, 64, 128, (1e-3, 1e-2))


# ------------------------------------------------------- segmented walks
SEGMENTED = [
    # batch, L, H, variant, heads the oracle checks (None: all)
    (1, 1300, 2, "plain", None),          # 11 one-chunk segments, 10 state-only items
    (2, 700, 4, "init+bias", None),       # 6 one-chunk segments, initial state chained
    (1, 1100, 64, "init+bias", [0, 17, 62, 63]),   # 2 segments of 6 chunks, items of 3
]


@pytest.mark.parametrize("case", SEGMENTED, ids=lambda c: f"b{c[0]}-L{c[1]}-H{c[2]}-{c[3]}")
@pytest.mark.parametrize("memory", ["short", "long"])
def test_segmented_walks(lib, case, memory):
    """Few (sequence, head pair) tasks: each direction's walk is split into
    segments that start from states chained out of a state-only pass.  With
    long-memory decays the chained state dominates every segment's output."""
    bsz, L, H, variant, heads = case
    P, N = 64, 128
    plan = lib.bimamba_launch_plan(lib.make_dims(bsz, L, H, P, N, torch.bfloat16))
    assert plan["tensor_core"] and plan["segments"] > 1 and plan["items"] > 0, plan
    w = inp_mod.Workload("seg", bsz, L, H, P, N, dtype="bf16", bc_scale=1.0 / math.sqrt(N))
    a = (1.0, 16.0) if memory == "short" else (1e-3, 1e-2)
    cpu = inp_mod.make_inputs(w, seed=L + H, a_range=a, conv_bias="bias" in variant)
    init = inp_mod.make_state(bsz, H, P, N, seed=11, scale=0.3) if "init" in variant else None
    y, fin = _run_scan(lib, w, _dev(cpu), None if init is None else init.cuda(), want_final=True)
    n = _np_inputs(cpu)
    heads = list(range(H)) if heads is None else heads
    sub, _ = head_subset(n, heads, H, P, N)
    ry, rfin = oracle.bimamba(sub["xbc"], sub["dt"], sub["A"], sub["D"], sub["conv_w"],
                              sub["conv_b"], heads=len(heads), headdim=P, d_state=N,
                              init=None if init is None else to_np(init[:, heads]),
                              want_final=True)
    cols = y_cols(heads, P)
    for b in range(bsz):
        assert rel_err(to_np(y)[b][..., cols], ry[b]) <= TOL["bf16"], b
        assert rel_err(to_np(fin)[b][heads], rfin[b]) <= TOL["bf16"], b


def test_repeated_calls_reuse_the_workspace(lib):
    """The handshake counters must come back to zero: three calls on one
    workspace give the same result."""
    w = inp_mod.Workload("rep", 2, 300, 4, 64, 128, dtype="bf16", bc_scale=1.0 / math.sqrt(128))
    g = _dev(inp_mod.make_inputs(w, seed=5))
    dims = lib.make_dims(2, 300, 4, 64, 128, torch.bfloat16)
    ws = lib.new_workspace(dims)
    outs = []
    for _ in range(3):
        y = torch.empty((2, 300, 256), dtype=torch.bfloat16, device="cuda")
        lib.bimamba_ssd_fwd_rev(g["xbc"], g["dt"], g["A"], g["D"], g["conv_w"], None, None, None, y,
                                ws, heads=4, headdim=64, d_state=128)
        outs.append(y)
    assert lib.bimamba_get_error() == lib.BIMAMBA_OK
    nflags = 2 * 2 * 3    # batch x head pairs x chunks, two counters each
    assert torch.count_nonzero(ws[: 4 * 2 * nflags]).item() == 0
    for o in outs[1:]:
        assert rel_err(to_np(o), to_np(outs[0])) <= 1e-2


# ------------------------------------------------------- untied directions
UNTIED = [
    # dtype, batch, L, H, P, N
    ("f32", 2, 129, 3, 16, 32),      # sequential fp32 path
    ("bf16", 2, 300, 4, 64, 128),    # tensor-core path, several chunks and a ragged tail
    ("bf16", 1, 1300, 2, 64, 128),   # tensor-core path, segmented walk (state-only items)
    ("bf16", 1, 200, 3, 32, 64),     # sequential path for bf16 shapes the tensor cores do not take
]


def _untied_inputs(w, a, seed):
    f = inp_mod.make_inputs(w, seed=seed, a_range=a, conv_bias=True)
    r = inp_mod.make_inputs(w, seed=seed + 1, a_range=a, conv_bias=True)
    return f, r


@pytest.mark.parametrize("case", UNTIED, ids=lambda c: "-".join(map(str, c)))
@pytest.mark.parametrize("fusion", ["sum", "concat"])
@pytest.mark.parametrize("memory", ["short", "long"])
@pytest.mark.parametrize("convs", ["both", "forward-only"])
def test_untied_directions(lib, case, fusion, memory, convs):
    """Each stream with its own x/B/C, dt, A, D and conv parameters; outputs
    summed or concatenated [forward | reverse] per token."""
    dtype, bsz, L, H, P, N = case
    w = inp_mod.Workload("u", bsz, L, H, P, N, dtype=dtype,
                         bc_scale=1.0 if dtype == "f32" else 1.0 / math.sqrt(N))
    a = (1.0, 16.0) if memory == "short" else (1e-3, 1e-2)
    f, r = _untied_inputs(w, a, seed=L + 31 * H)
    if convs == "forward-only":
        r["conv_w"] = None
        r["conv_b"] = None
    init = inp_mod.make_state(bsz, H, P, N, seed=17, scale=0.3)
    concat = fusion == "concat"
    td = inp_mod.torch_dtype(dtype)
    y = torch.full((bsz, L, (2 if concat else 1) * H * P), float("nan"), dtype=td, device="cuda")
    fin = torch.full((bsz, H, P, N), float("nan"), device="cuda")
    ws = lib.new_workspace(lib.make_dims(bsz, L, H, P, N, td))
    lib.bimamba_ssd_fwd_rev_untied(_dev(f), _dev(r), init.cuda(), fin, y, ws, heads=H, headdim=P,
                                   d_state=N, concat=concat)
    assert lib.bimamba_get_error() == lib.BIMAMBA_OK
    nf, nr = _np_inputs(f), _np_inputs(r)
    ry, rfin = oracle.bimamba_untied(nf["xbc"], nr["xbc"], nf["dt"], nr["dt"], nf["A"], nr["A"],
                                     nf["D"], nr["D"], nf["conv_w"], nr["conv_w"], nf["conv_b"],
                                     nr["conv_b"], heads=H, headdim=P, d_state=N, init=to_np(init),
                                     concat=concat, want_final=True)
    tol = TOL[dtype]
    for b in range(bsz):
        if concat:
            # each half against its own stream's scale
            assert rel_err(to_np(y)[b][..., :H * P], ry[b][..., :H * P]) <= tol, b
            assert rel_err(to_np(y)[b][..., H * P:], ry[b][..., H * P:]) <= tol, b
        else:
            assert rel_err(to_np(y)[b], ry[b]) <= tol, b
        assert rel_err(to_np(fin)[b], rfin[b]) <= tol, b


def test_untied_1p3b_concat_sampled_heads(lib):
    """b8 L4096 H64x64 N128 bf16 untied, concatenated, as benchmarked; 2 heads x
    2 sequences checked."""
    w = inp_mod.LAYER_1P3B
    f = inp_mod.make_inputs(w, seed=0)
    r = inp_mod.make_inputs(w, seed=1)
    H, P, N = w.heads, w.headdim, w.d_state
    y = torch.full((w.batch, w.seqlen, 2 * H * P), float("nan"), dtype=torch.bfloat16, device="cuda")
    ws = lib.new_workspace(lib.make_dims(w.batch, w.seqlen, H, P, N, torch.bfloat16))
    lib.bimamba_ssd_fwd_rev_untied(_dev(f), _dev(r), None, None, y, ws, heads=H, headdim=P,
                                   d_state=N, concat=True)
    assert lib.bimamba_get_error() == lib.BIMAMBA_OK
    y = y.cpu()
    heads = [3, 60]
    nf, nr = _np_inputs(f), _np_inputs(r)
    sf, _ = head_subset(nf, heads, H, P, N)
    sr, _ = head_subset(nr, heads, H, P, N)
    cols = y_cols(heads, P)
    for b in (0, 7):
        sl = slice(b, b + 1)
        ry = oracle.bimamba_untied(sf["xbc"][sl], sr["xbc"][sl], sf["dt"][sl], sr["dt"][sl], sf["A"],
                                   sr["A"], sf["D"], sr["D"], sf["conv_w"], sr["conv_w"], None, None,
                                   heads=len(heads), headdim=P, d_state=N, concat=True)
        got = to_np(y[sl])
        hp = len(heads) * P
        assert rel_err(got[..., cols], ry[..., :hp]) <= TOL["bf16"], b
        assert rel_err(got[..., H * P + cols], ry[..., hp:]) <= TOL["bf16"], b


# ------------------------------------------------------- sequence shards
SHARDED = [
    # batch, shard lengths, H, variant, heads the oracle checks (None: all)
    (2, (334, 333, 333), 4, "init+bias", None),        # 3 ranks, ragged shards
    (1, (700, 5, 600, 130), 2, "plain", None),         # 4 ranks; a 5-token shard; segmented shards
    (1, (1500, 1700), 64, "init+bias", [0, 41, 63]),   # 64 heads: items inside each shard too
]


def _run_shards(lib, g, lens, H, P, N, init):
    """Every rank's two calls, one rank after the other on this GPU (no rank
    waits on another inside a kernel); the all-gather becomes a stack."""
    full_x, full_dt = g["xbc"], g["dt"]
    bsz, total, ch = full_x.shape
    starts = [sum(lens[:r]) for r in range(len(lens))]
    zeros = torch.zeros((bsz, 4, ch), dtype=full_x.dtype, device="cuda")
    parts = []
    for r, (s0, n) in enumerate(zip(starts, lens)):
        # fresh allocations (a rank holds its own shard); slices of one tensor
        # can start off the 16-byte alignment the library requires
        x = full_x[:, s0:s0 + n].clone()
        dt = full_dt[:, s0:s0 + n].clone()
        tail = full_x[:, s0 - 4:s0].clone() if r > 0 else zeros
        head = full_x[:, s0 + n:s0 + n + 4].clone() if r + 1 < len(lens) else zeros
        ws = lib.new_workspace(lib.make_dims(bsz, n, H, P, N, torch.bfloat16))
        st = torch.full((2, bsz, H, P, N), float("nan"), device="cuda")
        dc = torch.full((2, bsz, H), float("nan"), device="cuda")
        lib.bimamba_shard_states(x, dt, g["A"], g["conv_w"], g["conv_b"], tail, head, st, dc, ws,
                                 heads=H, headdim=P, d_state=N)
        parts.append((x, dt, tail, head, ws, st, dc))
    all_states = torch.stack([p_[5] for p_ in parts])
    all_decays = torch.stack([p_[6] for p_ in parts])
    ys, fin = [], None
    for r, (x, dt, tail, head, ws, _, _) in enumerate(parts):
        y = torch.full((bsz, lens[r], H * P), float("nan"), dtype=torch.bfloat16, device="cuda")
        f = torch.full((bsz, H, P, N), float("nan"), device="cuda")
        lib.bimamba_ssd_fwd_rev_shard(x, dt, g["A"], g["D"], g["conv_w"], g["conv_b"], tail, head,
                                      init, all_states, all_decays, r, len(lens), f, y, ws,
                                      heads=H, headdim=P, d_state=N)
        ys.append(y)
        fin = f
    assert lib.bimamba_get_error() == lib.BIMAMBA_OK
    return torch.cat(ys, dim=1), fin, all_decays


@pytest.mark.parametrize("case", SHARDED, ids=lambda c: f"b{c[0]}-{len(c[1])}ranks-H{c[2]}-{c[3]}")
@pytest.mark.parametrize("memory", ["short", "long"])
def test_sequence_shards_equal_the_whole_sequence(lib, case, memory):
    """One sequence cut into shards: each rank's state-only pass, the exchange
    (here a stack) and each rank's shard call together give the oracle's
    output over the whole sequence and its final forward state."""
    bsz, lens, H, variant, heads = case
    P, N = 64, 128
    L = sum(lens)
    w = inp_mod.Workload("shard", bsz, L, H, P, N, dtype="bf16", bc_scale=1.0 / math.sqrt(N))
    a = (1.0, 16.0) if memory == "short" else (1e-3, 1e-2)
    cpu = inp_mod.make_inputs(w, seed=L + 7 * H, a_range=a, conv_bias="bias" in variant)
    init = inp_mod.make_state(bsz, H, P, N, seed=23, scale=0.3) if "init" in variant else None
    g = _dev(cpu)
    y, fin, decays = _run_shards(lib, g, lens, H, P, N, None if init is None else init.cuda())
    # the decays are log2 of the shards' decay products
    starts = [sum(lens[:r]) for r in range(len(lens))]
    want = torch.stack([(cpu["dt"][:, s:s + n].float() * cpu["A"]).sum(1) for s, n in zip(starts, lens)])
    got = decays.cpu()
    torch.testing.assert_close(got[:, 0], want / math.log(2.0), rtol=2e-4, atol=1e-3)
    # both directions sum the same terms, in opposite orders
    torch.testing.assert_close(got[:, 1], got[:, 0], rtol=1e-5, atol=1e-5)
    n = _np_inputs(cpu)
    heads = list(range(H)) if heads is None else heads
    sub, _ = head_subset(n, heads, H, P, N)
    ry, rfin = oracle.bimamba(sub["xbc"], sub["dt"], sub["A"], sub["D"], sub["conv_w"],
                              sub["conv_b"], heads=len(heads), headdim=P, d_state=N,
                              init=None if init is None else to_np(init[:, heads]), want_final=True)
    cols = y_cols(heads, P)
    for b in range(bsz):
        assert rel_err(to_np(y)[b][..., cols], ry[b]) <= TOL["bf16"], b
        assert rel_err(to_np(fin)[b][heads], rfin[b]) <= TOL["bf16"], b
