"""GPU parity of the pooled cached decode (bimamba_block_decode_pool): a batch
of streams whose states and conv tails live in a pool, each row reading its
own pool entry and committing its new state and tail back in place when its
block is finished ("Fixed state, long reach: constant-size caches in
large-scale block diffusion", abstract and section 1: one O(1) cache entry
per stream, many streams decoded together).  Checked against the oracle's
cached decode per row, with the untouched pool entries compared bit for bit."""
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


@pytest.mark.parametrize("blk", [64, 37, 1])
@pytest.mark.parametrize("memory", ["short", "long"])
def test_pool_decode_rows_and_commits(lib, blk, memory):
    pool, H, P, N = 8, 4, 64, 128
    slots = [6, 1, 3, 0, 7]
    commit = [1, 0, 1, 1, 0]
    rows = len(slots)
    w = inp_mod.Workload("pool", rows, blk, H, P, N, dtype="bf16", bc_scale=1.0 / math.sqrt(N))
    a = (1.0, 16.0) if memory == "short" else (1e-3, 1e-2)
    cpu = inp_mod.make_inputs(w, seed=blk + 5, a_range=a, conv_bias=True)
    states = inp_mod.make_state(pool, H, P, N, seed=21, scale=0.2)
    tails = inp_mod.make_tail(pool, 4, w.channels, "bf16", seed=22, bc_split=H * P,
                              bc_scale=w.bc_scale)
    g = {k: (None if v is None else v.cuda()) for k, v in cpu.items()}
    sp, tp = states.clone().cuda(), tails.clone().cuda()
    y = torch.full((rows, blk, H * P), float("nan"), dtype=torch.bfloat16, device="cuda")
    ws = lib.new_workspace(lib.make_dims(rows, blk, H, P, N, torch.bfloat16))
    slot_t = torch.tensor(slots, dtype=torch.int32, device="cuda")
    commit_t = torch.tensor(commit, dtype=torch.int32, device="cuda")
    lib.bimamba_block_decode_pool(g["xbc"], g["dt"], g["A"], g["D"], g["conv_w"], g["conv_b"], sp,
                                  tp, slot_t, commit_t, y, ws, heads=H, headdim=P, d_state=N)
    assert lib.bimamba_get_error() == lib.BIMAMBA_OK
    n = {k: to_np(v) for k, v in cpu.items()}
    got_y, got_s, got_t = to_np(y), to_np(sp), to_np(tp)
    for r, (slot, c) in enumerate(zip(slots, commit)):
        ry, rso, rto = oracle.block_decode(n["xbc"][r:r + 1], n["dt"][r:r + 1], n["A"], n["D"],
                                           n["conv_w"], n["conv_b"], to_np(states[slot:slot + 1]),
                                           to_np(tails[slot:slot + 1]), heads=H, headdim=P,
                                           d_state=N, want_commit=True)
        assert rel_err(got_y[r:r + 1], ry) <= TOL["bf16"], r
        if c:
            assert rel_err(got_s[slot:slot + 1], rso) <= TOL["bf16"], r
            np.testing.assert_array_equal(got_t[slot:slot + 1], rto)
        else:
            np.testing.assert_array_equal(got_s[slot], to_np(states[slot]))
            np.testing.assert_array_equal(got_t[slot], to_np(tails[slot]))
    for slot in set(range(pool)) - set(slots):
        np.testing.assert_array_equal(got_s[slot], to_np(states[slot]))
        np.testing.assert_array_equal(got_t[slot], to_np(tails[slot]))


def test_pool_decode_without_commit_flags_commits_every_row(lib):
    pool, H, P, N, blk = 3, 2, 64, 128, 64
    slots = [2, 0]
    w = inp_mod.Workload("pool", 2, blk, H, P, N, dtype="bf16", bc_scale=1.0 / math.sqrt(N))
    cpu = inp_mod.make_inputs(w, seed=3, a_range=(1e-3, 1e-2))
    states = inp_mod.make_state(pool, H, P, N, seed=4, scale=0.2)
    tails = inp_mod.make_tail(pool, 4, w.channels, "bf16", seed=5, bc_split=H * P,
                              bc_scale=w.bc_scale)
    g = {k: (None if v is None else v.cuda()) for k, v in cpu.items()}
    sp, tp = states.clone().cuda(), tails.clone().cuda()
    y = torch.empty((2, blk, H * P), dtype=torch.bfloat16, device="cuda")
    ws = lib.new_workspace(lib.make_dims(2, blk, H, P, N, torch.bfloat16))
    lib.bimamba_block_decode_pool(g["xbc"], g["dt"], g["A"], g["D"], g["conv_w"], None, sp, tp,
                                  torch.tensor(slots, dtype=torch.int32, device="cuda"), None, y, ws,
                                  heads=H, headdim=P, d_state=N)
    assert lib.bimamba_get_error() == lib.BIMAMBA_OK
    n = {k: to_np(v) for k, v in cpu.items()}
    for r, slot in enumerate(slots):
        _, rso, rto = oracle.block_decode(n["xbc"][r:r + 1], n["dt"][r:r + 1], n["A"], n["D"],
                                          n["conv_w"], None, to_np(states[slot:slot + 1]),
                                          to_np(tails[slot:slot + 1]), heads=H, headdim=P,
                                          d_state=N, want_commit=True)
        assert rel_err(to_np(sp[slot:slot + 1]), rso) <= TOL["bf16"]
        np.testing.assert_array_equal(to_np(tp[slot:slot + 1]), rto)
    np.testing.assert_array_equal(to_np(sp[1]), to_np(states[1]))


def test_pool_decode_slot_outside_the_pool_is_reported(lib):
    """A row whose slot lies outside the pool is skipped and reported as an
    invalid argument; the other rows are still decoded."""
    pool, H, P, N, blk = 2, 2, 64, 128, 16
    w = inp_mod.Workload("pool", 2, blk, H, P, N, dtype="bf16", bc_scale=1.0 / math.sqrt(N))
    cpu = inp_mod.make_inputs(w, seed=8)
    states = inp_mod.make_state(pool, H, P, N, seed=9, scale=0.2)
    tails = inp_mod.make_tail(pool, 4, w.channels, "bf16", seed=10, bc_split=H * P,
                              bc_scale=w.bc_scale)
    g = {k: (None if v is None else v.cuda()) for k, v in cpu.items()}
    sp, tp = states.clone().cuda(), tails.clone().cuda()
    y = torch.full((2, blk, H * P), float("nan"), dtype=torch.bfloat16, device="cuda")
    ws = lib.new_workspace(lib.make_dims(2, blk, H, P, N, torch.bfloat16))
    lib.bimamba_block_decode_pool(g["xbc"], g["dt"], g["A"], g["D"], g["conv_w"], None, sp, tp,
                                  torch.tensor([1, 5], dtype=torch.int32, device="cuda"), None, y,
                                  ws, heads=H, headdim=P, d_state=N)
    assert lib.bimamba_get_error() == lib.BIMAMBA_ERR_INVALID
    assert lib.bimamba_get_error() == lib.BIMAMBA_OK
    n = {k: to_np(v) for k, v in cpu.items()}
    ry, _, _ = oracle.block_decode(n["xbc"][:1], n["dt"][:1], n["A"], n["D"], n["conv_w"], None,
                                   to_np(states[1:2]), to_np(tails[1:2]), heads=H, headdim=P,
                                   d_state=N, want_commit=True)
    assert rel_err(to_np(y[:1]), ry) <= TOL["bf16"]
    np.testing.assert_array_equal(to_np(sp[0]), to_np(states[0]))
