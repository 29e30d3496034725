"""GPU parity of the projections around the mixer (bimamba_in_proj,
bimamba_out_proj: the tcgen05 GEMM with the mixer's own epilogues) against
the oracle's Linear maps, and of the whole mixer layer (in-projection ->
bidirectional mixer core -> out-projection) against the oracle chain.

Shapes: ragged tiles (tokens, output width and depth that are not multiples
of the 128 x 256 x 64 tile), and the 1.3B-layer shapes (d_model 2048, 64
heads x 64, d_state 128: in-projection 2048 -> 4352 + 64, out-projection
4096 -> 2048, the untied block's fusion 8192 -> 2048) on 32 768 tokens with
sampled rows checked.  Source: "DiffuMamba" blog post, network-architecture
listing (d_model 2048, expand 2, the bidirectional block's concatenation
and fusion Linear)."""
import math

import numpy as np
import pytest
import torch

import oracle
from bidirectional_mamba_ssm_b200 import inputs as inp_mod
from parity_util import TOL, rel_err, to_np

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lib():
    from bidirectional_mamba_ssm_b200 import _lib
    return _lib


def _in_proj(lib, pr, H, P, N):
    tokens = pr["u"].shape[0]
    ch = H * P + 2 * N
    xbc = torch.full((tokens, ch), float("nan"), dtype=torch.bfloat16, device="cuda")
    dt = torch.full((tokens, H), float("nan"), dtype=torch.bfloat16, device="cuda")
    lib.bimamba_in_proj(pr["u"].cuda(), pr["w_in"].cuda(), pr["dt_bias"].cuda(), xbc, dt, heads=H,
                        headdim=P, d_state=N)
    assert lib.bimamba_get_error() == lib.BIMAMBA_OK
    return xbc, dt


@pytest.mark.parametrize("tokens,d_model,H,P,N", [
    (1, 64, 2, 64, 128),       # one row; output width 386 (ragged N tile)
    (130, 72, 2, 32, 16),      # ragged M, depth 72 (K tail inside one 64 slice)
    (300, 200, 4, 64, 128),    # several tiles, depth not a multiple of 64
    (257, 2048, 3, 64, 128),   # full depth, ragged everything
])
def test_in_proj_small(lib, tokens, d_model, H, P, N):
    pr = inp_mod.make_projections(d_model, H, P, N, tokens, seed=tokens + d_model)
    xbc, dt = _in_proj(lib, pr, H, P, N)
    rx, rdt = oracle.in_proj(pr["u"], pr["w_in"], pr["dt_bias"], heads=H, headdim=P, d_state=N)
    assert rel_err(to_np(xbc), rx) <= TOL["bf16"]
    assert rel_err(to_np(dt), rdt) <= TOL["bf16"]


@pytest.mark.parametrize("tokens,d_inner,d_model", [(1, 64, 64), (130, 200, 72), (300, 4096, 300),
                                                    (513, 8192, 2048)])
def test_out_proj_small(lib, tokens, d_inner, d_model):
    pr = inp_mod.make_projections(d_model, 1, 8, 8, tokens, seed=7 + tokens, d_inner_out=d_inner)
    out = torch.full((tokens, d_model), float("nan"), dtype=torch.bfloat16, device="cuda")
    lib.bimamba_out_proj(pr["y"].cuda(), pr["w_out"].cuda(), out)
    assert lib.bimamba_get_error() == lib.BIMAMBA_OK
    assert rel_err(to_np(out), oracle.out_proj(pr["y"], pr["w_out"])) <= TOL["bf16"]


def _sampled_rows(tokens, k=48, seed=0):
    g = np.random.default_rng(seed)
    rows = set(g.choice(tokens, size=k, replace=False).tolist())
    rows.update({0, tokens - 1, 127, 128, 255, 256})
    return sorted(r for r in rows if r < tokens)


def test_in_proj_1p3b_layer_sampled_rows(lib):
    w = inp_mod.LAYER_1P3B
    tokens, H, P, N = w.batch * w.seqlen, w.heads, w.headdim, w.d_state
    pr = inp_mod.make_projections(2048, H, P, N, tokens, seed=1, device="cuda")
    xbc, dt = _in_proj(lib, pr, H, P, N)
    rows = _sampled_rows(tokens)
    rx, rdt = oracle.in_proj(pr["u"][rows].cpu(), pr["w_in"].cpu(), pr["dt_bias"].cpu(), heads=H,
                             headdim=P, d_state=N)
    assert rel_err(to_np(xbc[rows]), rx) <= TOL["bf16"]
    assert rel_err(to_np(dt[rows]), rdt) <= TOL["bf16"]
    assert not torch.isnan(xbc).any() and not torch.isnan(dt).any()


@pytest.mark.parametrize("d_inner", [4096, 8192])
def test_out_proj_1p3b_layer_sampled_rows(lib, d_inner):
    tokens = inp_mod.LAYER_1P3B.batch * inp_mod.LAYER_1P3B.seqlen
    pr = inp_mod.make_projections(2048, 1, 8, 8, tokens, seed=2, d_inner_out=d_inner, device="cuda")
    out = torch.full((tokens, 2048), float("nan"), dtype=torch.bfloat16, device="cuda")
    lib.bimamba_out_proj(pr["y"].cuda(), pr["w_out"].cuda(), out)
    assert lib.bimamba_get_error() == lib.BIMAMBA_OK
    rows = _sampled_rows(tokens, seed=3)
    assert rel_err(to_np(out[rows]), oracle.out_proj(pr["y"][rows].cpu(), pr["w_out"].cpu())) <= TOL["bf16"]
    assert not torch.isnan(out).any()


def test_mixer_layer_chain(lib):
    """in-projection -> conv + SiLU, forward and reverse SSD, summed ->
    out-projection, against the oracle's chain (inputs of each stage rounded
    to bf16 as the library stores them)."""
    bsz, L, H, P, N, d_model = 2, 300, 4, 64, 128, 256
    tokens = bsz * L
    pr = inp_mod.make_projections(d_model, H, P, N, tokens, seed=11)
    mix = inp_mod.make_inputs(inp_mod.Workload("m", bsz, L, H, P, N, dtype="bf16"), seed=12)
    xbc, dt = _in_proj(lib, pr, H, P, N)
    y = torch.empty((bsz, L, H * P), dtype=torch.bfloat16, device="cuda")
    ws = lib.new_workspace(lib.make_dims(bsz, L, H, P, N, torch.bfloat16))
    A, D, cw = mix["A"].cuda(), mix["D"].cuda(), mix["conv_w"].cuda()
    lib.bimamba_ssd_fwd_rev(xbc.view(bsz, L, -1), dt.view(bsz, L, H), A, D, cw, None, None, None, y,
                            ws, heads=H, headdim=P, d_state=N)
    out = torch.empty((tokens, d_model), dtype=torch.bfloat16, device="cuda")
    lib.bimamba_out_proj(y.view(tokens, -1), pr["w_out"].cuda(), out)
    assert lib.bimamba_get_error() == lib.BIMAMBA_OK
    rx, rdt = oracle.in_proj(pr["u"], pr["w_in"], pr["dt_bias"], heads=H, headdim=P, d_state=N)
    bf = lambda a: torch.from_numpy(a).to(torch.bfloat16).double().numpy()   # stored as bf16
    ry = oracle.bimamba(bf(rx).reshape(bsz, L, -1), bf(rdt).reshape(bsz, L, H), to_np(mix["A"]),
                        to_np(mix["D"]), to_np(mix["conv_w"]), None, heads=H, headdim=P, d_state=N)
    rout = oracle.out_proj(bf(ry).reshape(tokens, -1), pr["w_out"])
    assert rel_err(to_np(out), rout) <= TOL["bf16"]
