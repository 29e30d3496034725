"""GPU parity of the conv index logic INSIDE the scan kernels, and of the
method's closed-form decay extremes (A = 0, A -> -inf), against the oracle.

The stand-alone conv entry point is checked bit for bit elsewhere; the scan
never calls it.  The scan convolves on its own: the x channels while staging
each chunk (TMA box with the 3-token halo, reflected row index for the
reverse stream), the B/C channels in a prepass, the decode path from the conv
tail, sequence shards from their halos, and the sequential kernel in its own
staging.  These tests make a one-token slip in any of them an O(1) error:

  * one-hot conv taps (tap j = 1, the rest 0; a "mixed" case gives the x, B
    and C channels different taps), so each activated value is SiLU of exactly
    one raw token: u[t-3+j] forward, u[t+3-j] reverse, zero past either end;
  * A = -1e4, so every decay factor between two different tokens underflows to
    0 and each output row depends on its own token only:
        y_dir[t] = (C'_t . B'_t) dt_t x'_t          (D = 0)
    with positive raw values (x ~ U[1, 3]; B, C constant over their channels
    per token, ~ U[1, 4]) so that the C'.B' factor varies by token and no
    row is a cancelling sum, whose bf16 rounding the per-row metric below
    would magnify;
  * the comparison is per token row (error relative to that row's own
    magnitude), so a shifted source token fails by the size of the row;
  * where a stream's source token lies in the zero padding, its output is
    exactly 0 (SiLU(0) = 0 and every product with it is an exact zero): with
    concatenated untied outputs each stream's padding rows are compared for
    bit equality with 0, and with the summed output the rows where both
    streams read padding.

Sources: the conv tap convention (tap j multiplies u[t-3+j]; reverse = the
mirror image) is the reading of "DiffuMamba" blog, network-architecture
listing (d_conv = 4) and the Japanese technical summary section 2 (forward and
reverse streams added); the decay extremes are the recurrence's own limits.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from bidirectional_mamba_ssm_b200 import inputs as inp_mod
from parity_util import TOL, rel_err, to_np

pytestmark = pytest.mark.gpu

STEEP = -1.0e4
ROW_TOL = {"f32": 1e-4, "bf16": 2e-2}


@pytest.fixture(scope="module")
def lib():
    from bidirectional_mamba_ssm_b200 import _lib
    return _lib


def _dev(d):
    return {k: (None if v is None else v.cuda()) for k, v in d.items()}


def _np(d):
    return {k: to_np(v) for k, v in d.items()}


def one_hot_taps(ch, split, N, taps):
    """(ch, 4) one-hot taps: x channels take taps[0], B taps[1], C taps[2]."""
    w = torch.zeros((ch, 4))
    w[:split, taps[0]] = 1.0
    w[split:split + N, taps[1]] = 1.0
    w[split + N:, taps[2]] = 1.0
    return w


def steep_inputs(dtype, bsz, L, H, P, N, taps, seed):
    """Seeded inputs with one-hot taps, A = -1e4, D = 0, and positive raw
    values so that no output is a sum that cancels: the x channels ~ U[1, 3]
    per channel and token; the B channels of token t all equal beta_t and
    the C channels gamma_t, both ~ U[1, 4], so that C'_t . B'_t =
    N silu(gamma_t) silu(beta_t) varies with the token by up to 16x and has
    no rounding-sensitive cancellation.  A one-token slip then changes a row
    by tens of percent, far above bf16 rounding."""
    w = inp_mod.Workload("idx", bsz, L, H, P, N, dtype=dtype, bc_scale=1.0)
    cpu = inp_mod.make_inputs(w, seed=seed)
    g = torch.Generator().manual_seed(seed + 12345)
    x = torch.rand((bsz, L, H * P), generator=g) * 2.0 + 1.0
    beta = (torch.rand((bsz, L, 1), generator=g) * 3.0 + 1.0).expand(bsz, L, N)
    gamma = (torch.rand((bsz, L, 1), generator=g) * 3.0 + 1.0).expand(bsz, L, N)
    cpu["xbc"] = torch.cat([x, beta, gamma], dim=-1).to(inp_mod.torch_dtype(dtype)).contiguous()
    cpu["A"] = torch.full((H,), STEEP)
    cpu["D"] = torch.zeros(H)
    cpu["conv_w"] = one_hot_taps(w.channels, H * P, N, taps)
    cpu["conv_b"] = None
    return w, cpu


def row_errors(got, ref):
    """Per token row: max |g - r| over the row / the row's max |r| (rows
    whose reference is below 1e-3 of the tensor's max use that floor)."""
    g = np.asarray(got, dtype=np.float64).reshape(-1, got.shape[-1])
    r = np.asarray(ref, dtype=np.float64).reshape(-1, ref.shape[-1])
    floor = 1e-3 * max(float(np.abs(r).max()), 1e-30)
    den = np.maximum(np.abs(r).max(axis=1), floor)
    return np.abs(g - r).max(axis=1) / den


def assert_rows(got, ref, dtype, what):
    e = row_errors(got, ref)
    worst = int(np.argmax(e))
    assert e[worst] <= ROW_TOL[dtype], f"{what}: row {worst} err {e[worst]:.3e}"


def src_in_range(t, L, j, rev):
    s = t + 3 - j if rev else t - 3 + j
    return 0 <= s < L


TAPS = [(0, 0, 0), (1, 1, 1), (2, 2, 2), (3, 3, 3), (1, 3, 0)]
LENGTHS = [1, 2, 3, 127, 128, 129, 131, 4096]
# the chunked tensor-core kernel (bf16, P 64, N 128) and the sequential kernel
PATHS = {"tc": ("bf16", 64, 128), "seq-f32": ("f32", 32, 16), "seq-bf16": ("bf16", 32, 64)}


@pytest.mark.parametrize("path", list(PATHS))
@pytest.mark.parametrize("L", LENGTHS)
@pytest.mark.parametrize("taps", TAPS, ids=lambda t: "taps" + "".join(map(str, t)))
def test_scan_conv_index_one_hot_summed(lib, path, L, taps):
    """bimamba_ssd_fwd_rev: per-row parity, and exact zeros where both streams
    read only padding."""
    dtype, P, N = PATHS[path]
    if path != "tc" and L == 4096:
        L = 1031   # the sequential kernel is slow per token; still > 8 chunks
    bsz, H = 2, 2
    w, cpu = steep_inputs(dtype, bsz, L, H, P, N, taps, seed=L + 13 * taps[0] + 7 * taps[1])
    g = _dev(cpu)
    td = inp_mod.torch_dtype(dtype)
    y = torch.full((bsz, L, H * P), float("nan"), dtype=td, device="cuda")
    ws = lib.new_workspace(lib.make_dims(bsz, L, H, P, N, td))
    lib.bimamba_ssd_fwd_rev(g["xbc"], g["dt"], g["A"], g["D"], g["conv_w"], None, None, None, y,
                            ws, heads=H, headdim=P, d_state=N)
    assert lib.bimamba_get_error() == lib.BIMAMBA_OK
    n = _np(cpu)
    ry = oracle.bimamba(n["xbc"], n["dt"], n["A"], n["D"], n["conv_w"], None, heads=H, headdim=P,
                        d_state=N)
    got = to_np(y)
    assert_rows(got, ry, dtype, f"{path} L{L} taps{taps}")
    for t in range(L):
        if not any(src_in_range(t, L, j, rev) for j in taps for rev in (False, True)):
            assert np.all(got[:, t] == 0.0), t


@pytest.mark.parametrize("path", ["tc", "seq-bf16"])
@pytest.mark.parametrize("L", [1, 3, 129, 131, 4096])
@pytest.mark.parametrize("taps", TAPS, ids=lambda t: "taps" + "".join(map(str, t)))
def test_scan_conv_index_one_hot_per_stream(lib, path, L, taps):
    """Untied call with concatenated outputs: each stream on its own, so the
    forward stream's left padding and the reverse stream's right padding are
    compared with 0 bit for bit."""
    dtype, P, N = PATHS[path]
    if path != "tc" and L == 4096:
        L = 1031
    bsz, H = 1, 2
    w, f = steep_inputs(dtype, bsz, L, H, P, N, taps, seed=3 * L + taps[2])
    _, r = steep_inputs(dtype, bsz, L, H, P, N, taps, seed=3 * L + taps[2] + 1)
    td = inp_mod.torch_dtype(dtype)
    y = torch.full((bsz, L, 2 * H * P), float("nan"), dtype=td, device="cuda")
    ws = lib.new_workspace(lib.make_dims(bsz, L, H, P, N, td))
    lib.bimamba_ssd_fwd_rev_untied(_dev(f), _dev(r), None, None, y, ws, heads=H, headdim=P,
                                   d_state=N, concat=True)
    assert lib.bimamba_get_error() == lib.BIMAMBA_OK
    nf, nr = _np(f), _np(r)
    ry = oracle.bimamba_untied(nf["xbc"], nr["xbc"], nf["dt"], nr["dt"], nf["A"], nr["A"], nf["D"],
                               nr["D"], nf["conv_w"], nr["conv_w"], None, None, heads=H, headdim=P,
                               d_state=N, concat=True)
    got = to_np(y)
    HP = H * P
    assert_rows(got[..., :HP], ry[..., :HP], dtype, "forward stream")
    assert_rows(got[..., HP:], ry[..., HP:], dtype, "reverse stream")
    for t in range(L):
        if not any(src_in_range(t, L, j, False) for j in taps):
            assert np.all(got[:, t, :HP] == 0.0), ("forward", t)
        if not any(src_in_range(t, L, j, True) for j in taps):
            assert np.all(got[:, t, HP:] == 0.0), ("reverse", t)


@pytest.mark.parametrize("path", ["tc", "seq-f32"])
@pytest.mark.parametrize("blk,prefix", [(1, 7), (2, 2), (3, 0), (64, 200), (130, 1), (300, 9)])
@pytest.mark.parametrize("taps", TAPS, ids=lambda t: "taps" + "".join(map(str, t)))
def test_decode_conv_index_one_hot(lib, path, blk, prefix, taps):
    """bimamba_block_decode: the forward stream's conv reads the newest 3 raw
    tokens of the tail before the block; the reverse stream's reads zeros past
    the block end.  The cached state is scaled to zero by the steep decay, so
    each row checks only where its conv read from."""
    dtype, P, N = PATHS[path]
    S, H = 2, 2
    w, cpu = steep_inputs(dtype, S, prefix + blk, H, P, N, taps, seed=blk + 5 * prefix + taps[0])
    n = _np(cpu)
    ch = w.channels
    tail = np.zeros((S, 4, ch))
    k = min(prefix, 4)
    if k:
        tail[:, 4 - k:] = n["xbc"][:, prefix - k:prefix]
    state = inp_mod.make_state(S, H, P, N, seed=8, scale=0.5)
    td = inp_mod.torch_dtype(dtype)
    tail_t = torch.from_numpy(tail).to(td)
    y = torch.full((S, blk, H * P), float("nan"), dtype=td, device="cuda")
    so = torch.full((S, H, P, N), float("nan"), device="cuda")
    dims = lib.make_dims(S, blk, H, P, N, td)
    lib.bimamba_block_decode(cpu["xbc"][:, prefix:].contiguous().cuda(),
                             cpu["dt"][:, prefix:].contiguous().cuda(), cpu["A"].cuda(),
                             cpu["D"].cuda(), cpu["conv_w"].cuda(), None, state.cuda(),
                             tail_t.cuda(), y, so, None, lib.new_workspace(dims), heads=H,
                             headdim=P, d_state=N)
    assert lib.bimamba_get_error() == lib.BIMAMBA_OK
    ry, rso, _ = oracle.block_decode(n["xbc"][:, prefix:], n["dt"][:, prefix:], n["A"], n["D"],
                                     n["conv_w"], None, to_np(state), to_np(tail_t), heads=H,
                                     headdim=P, d_state=N, want_commit=True)
    assert_rows(to_np(y), ry, dtype, f"decode blk{blk} prefix{prefix}")
    assert rel_err(to_np(so), rso) <= TOL[dtype]


@pytest.mark.parametrize("lens", [(4, 5, 130), (130, 4, 5), (5, 130, 4, 4)],
                         ids=lambda c: "-".join(map(str, c)))
@pytest.mark.parametrize("taps", TAPS, ids=lambda t: "taps" + "".join(map(str, t)))
def test_shard_halo_index_one_hot(lib, lens, taps):
    """Sequence shards: the forward stream's conv reads the 3 tokens before a
    shard from its tail halo, the reverse stream's the 3 after it from its
    head halo.  Shards of 4 and 5 tokens put both halos inside one chunk."""
    from test_parity_gpu import _run_shards
    bsz, H, P, N = 1, 2, 64, 128
    L = sum(lens)
    w, cpu = steep_inputs("bf16", bsz, L, H, P, N, taps, seed=L + taps[1])
    y, _, _ = _run_shards(lib, _dev(cpu), lens, H, P, N, None)
    n = _np(cpu)
    ry = oracle.bimamba(n["xbc"], n["dt"], n["A"], n["D"], n["conv_w"], None, heads=H, headdim=P,
                        d_state=N)
    assert_rows(to_np(y), ry, "bf16", f"shards {lens}")


# ------------------------------------------------------------ decay extremes
EXTREME_SHAPES = [
    # dtype, batch, L, H, P, N
    ("bf16", 2, 300, 4, 64, 128),     # tensor-core path, several chunks + ragged tail
    ("bf16", 1, 4100, 2, 64, 128),    # tensor-core path, segmented walk (33 chunks)
    ("bf16", 1, 1100, 64, 64, 128),   # 64 heads: segments of 6 chunks, state-only items
    ("f32", 1, 256, 4, 32, 16),       # sequential fp32 path
    ("bf16", 1, 200, 2, 32, 64),      # sequential bf16 path
]


@pytest.mark.parametrize("case", EXTREME_SHAPES, ids=lambda c: "-".join(map(str, c)))
@pytest.mark.parametrize("A", ["zero", "steep"])
def test_decay_extremes(lib, case, A):
    """A = 0 exactly: every decay factor is 1 and the state never shrinks
    (outputs are prefix / suffix sums); A = -1e4: only the diagonal term
    survives.  With conv, bias and an initial state."""
    dtype, bsz, L, H, P, N = case
    w = inp_mod.Workload("ext", bsz, L, H, P, N, dtype=dtype,
                         bc_scale=1.0 if dtype == "f32" else 1.0 / math.sqrt(N))
    cpu = inp_mod.make_inputs(w, seed=L + H + (A == "zero"), conv_bias=True)
    cpu["A"] = torch.zeros(H) if A == "zero" else torch.full((H,), STEEP)
    init = inp_mod.make_state(bsz, H, P, N, seed=12, scale=0.3)
    g = _dev(cpu)
    td = inp_mod.torch_dtype(dtype)
    y = torch.full((bsz, L, H * P), float("nan"), dtype=td, device="cuda")
    fin = torch.full((bsz, H, P, N), float("nan"), device="cuda")
    ws = lib.new_workspace(lib.make_dims(bsz, L, H, P, N, td))
    lib.bimamba_ssd_fwd_rev(g["xbc"], g["dt"], g["A"], g["D"], g["conv_w"], g["conv_b"],
                            init.cuda(), fin, y, ws, heads=H, headdim=P, d_state=N)
    assert lib.bimamba_get_error() == lib.BIMAMBA_OK
    n = _np(cpu)
    heads = list(range(H)) if H <= 4 else [0, 21, 63]
    from parity_util import head_subset, y_cols
    sub, _ = head_subset(n, heads, H, P, N)
    ry, rfin = oracle.bimamba(sub["xbc"], sub["dt"], sub["A"], sub["D"], sub["conv_w"],
                              sub["conv_b"], heads=len(heads), headdim=P, d_state=N,
                              init=to_np(init[:, heads]), want_final=True)
    cols = y_cols(heads, P)
    got, gfin = to_np(y), to_np(fin)
    for b in range(bsz):
        assert rel_err(got[b][..., cols], ry[b]) <= TOL[dtype], b
        assert rel_err(gfin[b][heads], rfin[b]) <= TOL[dtype], b
