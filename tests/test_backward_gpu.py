"""GPU parity of the mixer core's backward pass (bimamba_ssd_fwd_rev_backward)
against the oracle's adjoint (oracle.bimamba_mixer_backward, pinned by
central finite differences of the forward oracle).  Every gradient is
compared with the max-abs-relative metric: 1e-4 for fp32 activations, 2e-2
for bf16.  Shapes span several 64-token chunks with ragged tails, with short-
and long-memory decays, a conv bias and an initial state.  The 64-head case
checks the per-head gradients (x channels, dt, A, D, x conv taps, initial
state) of sampled heads; the B and C gradients sum over all heads and are
checked in full on the small shapes.  The bf16 shapes with headdim 64 and
d_state 128 run the tensor-core kernels (128-token chunks), the others the
CUDA-core kernels (64-token chunks)."""
import math

import numpy as np
import pytest
import torch

import oracle
from bidirectional_mamba_ssm_b200 import inputs as inp_mod
from parity_util import TOL, head_subset, rel_err, to_np

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lib():
    from bidirectional_mamba_ssm_b200 import _lib
    return _lib


CASES = [
    # dtype, batch, L, H, P, N
    ("f32", 1, 130, 2, 32, 16),
    ("f32", 2, 70, 3, 16, 32),
    ("bf16", 2, 200, 4, 64, 128),
    ("bf16", 1, 300, 2, 64, 128),
    ("bf16", 1, 64, 2, 32, 64),
    ("bf16", 2, 70, 3, 8, 8),   # 40 channels: a partial 64-channel conv tile, rows of 80 bytes
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "-".join(map(str, c)))
@pytest.mark.parametrize("memory", ["short", "long"])
def test_backward_small(lib, case, memory):
    dtype, bsz, L, H, P, N = case
    w = inp_mod.Workload("bwd", bsz, L, H, P, N, dtype=dtype,
                         bc_scale=1.0 if dtype == "f32" else 1.0 / math.sqrt(N))
    a = (1.0, 16.0) if memory == "short" else (1e-3, 1e-2)
    cpu = inp_mod.make_inputs(w, seed=L + 3 * H, a_range=a, conv_bias=True)
    init = inp_mod.make_state(bsz, H, P, N, seed=5, scale=0.3)
    g = torch.Generator().manual_seed(L)
    dy = torch.randn((bsz, L, H * P), generator=g).to(inp_mod.torch_dtype(dtype))
    d = {k: (None if v is None else v.cuda()) for k, v in cpu.items()}
    got = lib.bimamba_ssd_fwd_rev_backward(d["xbc"], d["dt"], d["A"], d["D"], d["conv_w"], d["conv_b"],
                                           init.cuda(), dy.cuda(), heads=H, headdim=P, d_state=N,
                                           want_dinit=True)
    assert lib.bimamba_get_error() == lib.BIMAMBA_OK
    n = {k: to_np(v) for k, v in cpu.items()}
    ref = oracle.bimamba_mixer_backward(n["xbc"], n["dt"], n["A"], n["D"], n["conv_w"], n["conv_b"],
                                        to_np(dy), heads=H, headdim=P, d_state=N, init=to_np(init))
    tol = TOL[dtype]
    for k in ("xbc", "dt", "A", "D", "conv_w", "conv_b", "init"):
        assert rel_err(to_np(got[k]), ref[k]) <= tol, (k, rel_err(to_np(got[k]), ref[k]))


def test_backward_64_heads_sampled(lib):
    """b2 x L1024, 64 heads x 64, d_state 128 (the 1.3B layer's head shape):
    the per-head gradients of 3 heads against the oracle on those heads."""
    bsz, L, H, P, N = 2, 1024, 64, 64, 128
    w = inp_mod.Workload("bwd64", bsz, L, H, P, N, dtype="bf16", bc_scale=1.0 / math.sqrt(N))
    cpu = inp_mod.make_inputs(w, seed=41, conv_bias=True)
    g = torch.Generator().manual_seed(42)
    dy = torch.randn((bsz, L, H * P), generator=g).to(torch.bfloat16)
    d = {k: (None if v is None else v.cuda()) for k, v in cpu.items()}
    got = lib.bimamba_ssd_fwd_rev_backward(d["xbc"], d["dt"], d["A"], d["D"], d["conv_w"], d["conv_b"],
                                           None, dy.cuda(), heads=H, headdim=P, d_state=N,
                                           want_dinit=True)
    assert lib.bimamba_get_error() == lib.BIMAMBA_OK
    heads = [0, 37, 63]
    n = {k: to_np(v) for k, v in cpu.items()}
    sub, xcols = head_subset(n, heads, H, P, N)
    ycols = np.concatenate([np.arange(h * P, (h + 1) * P) for h in heads])
    # the other heads' B/C gradients are not in the subset, so only per-head terms compare
    ref = oracle.bimamba_mixer_backward(sub["xbc"], sub["dt"], sub["A"], sub["D"], sub["conv_w"],
                                        sub["conv_b"], to_np(dy)[..., ycols], heads=len(heads),
                                        headdim=P, d_state=N)
    hp = len(heads) * P
    tol = TOL["bf16"]
    assert rel_err(to_np(got["xbc"])[..., xcols], ref["xbc"][..., :hp]) <= tol
    assert rel_err(to_np(got["dt"])[..., heads], ref["dt"]) <= tol
    assert rel_err(to_np(got["A"])[heads], ref["A"]) <= tol
    assert rel_err(to_np(got["D"])[heads], ref["D"]) <= tol
    assert rel_err(to_np(got["conv_w"])[xcols], ref["conv_w"][:hp]) <= tol
    assert rel_err(to_np(got["init"])[:, heads], ref["init"]) <= tol


TC_EDGES = [
    # batch, L, decay: shapes of the tensor-core backward (bf16, headdim 64,
    # d_state 128): one token, one full 128-token chunk, one chunk plus one
    # token, several chunks with a ragged tail, and the closed-form decays
    (1, 1, "short"),
    (1, 128, "long"),
    (1, 129, "long"),
    (3, 257, "short"),
    (2, 384, "zero"),
    (1, 200, "steep"),
]


@pytest.mark.parametrize("case", TC_EDGES, ids=lambda c: "-".join(map(str, c)))
def test_backward_tensor_core_edges(lib, case):
    """The tensor-core backward against the oracle's adjoint on its edge
    shapes: chunk boundaries at 1, 128 and 129 tokens, a ragged tail with
    batch 3, A = 0 (every decay exactly 1: the state adjoint never shrinks)
    and A = -50 (decays of ~1e-3 per step)."""
    bsz, L, decay = case
    H, P, N = 2, 64, 128
    w = inp_mod.Workload("bwdtc", bsz, L, H, P, N, dtype="bf16", bc_scale=1.0 / math.sqrt(N))
    a = {"short": (1.0, 16.0), "long": (1e-3, 1e-2), "zero": (1.0, 2.0), "steep": (1.0, 2.0)}[decay]
    cpu = inp_mod.make_inputs(w, seed=7 * L + bsz, a_range=a, conv_bias=True)
    if decay == "zero":
        cpu["A"] = torch.zeros_like(cpu["A"])
    elif decay == "steep":
        # a decay of ~e^-6.5 per step; steeper, dL/dA itself underflows (the
        # oracle's is ~1e-74 at A = -1e4) and a relative metric has nothing
        # left to compare
        cpu["A"] = torch.full_like(cpu["A"], -50.0)
    init = inp_mod.make_state(bsz, H, P, N, seed=9, scale=0.3)
    g = torch.Generator().manual_seed(L + 1)
    dy = torch.randn((bsz, L, H * P), generator=g).to(torch.bfloat16)
    d = {k: (None if v is None else v.cuda()) for k, v in cpu.items()}
    got = lib.bimamba_ssd_fwd_rev_backward(d["xbc"], d["dt"], d["A"], d["D"], d["conv_w"], d["conv_b"],
                                           init.cuda(), dy.cuda(), heads=H, headdim=P, d_state=N,
                                           want_dinit=True)
    assert lib.bimamba_get_error() == lib.BIMAMBA_OK
    n = {k: to_np(v) for k, v in cpu.items()}
    ref = oracle.bimamba_mixer_backward(n["xbc"], n["dt"], n["A"], n["D"], n["conv_w"], n["conv_b"],
                                        to_np(dy), heads=H, headdim=P, d_state=N, init=to_np(init))
    tol = TOL["bf16"]
    for k in ("xbc", "dt", "A", "D", "conv_w", "conv_b", "init"):
        assert rel_err(to_np(got[k]), ref[k]) <= tol, (k, rel_err(to_np(got[k]), ref[k]))
