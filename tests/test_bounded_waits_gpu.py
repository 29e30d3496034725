"""Failure detection without a GPU fault: every wait in the kernels is a
bounded spin that records BIMAMBA_ERR_TIMEOUT in the device status word and
lets the kernel finish.  This test launches a tiny grid with a dependency
that can never be met, checks the status and that the call came back
promptly, then checks that the context still computes correct results."""
import math
import time

import pytest
import torch

import oracle
from bidirectional_mamba_ssm_b200 import inputs as inp_mod
from parity_util import TOL, rel_err, to_np

pytestmark = pytest.mark.gpu


def test_unmet_partner_wait_times_out_and_the_context_stays_usable():
    from bidirectional_mamba_ssm_b200 import _lib as lib
    bsz, L, H, P, N = 1, 256, 2, 64, 128      # one head pair: one forward and one reverse CTA
    w = inp_mod.Workload("wait", bsz, L, H, P, N, dtype="bf16", bc_scale=1.0 / math.sqrt(N))
    cpu = inp_mod.make_inputs(w, seed=2)
    g = {k: (None if v is None else v.cuda()) for k, v in cpu.items()}
    dims = lib.make_dims(bsz, L, H, P, N, torch.bfloat16)
    assert lib.bimamba_launch_plan(dims)["segments"] == 1
    assert lib.bimamba_get_error() == lib.BIMAMBA_OK

    # The workspace starts with the meeting counters [batch][head pair][chunk][arrivals, ready].
    # Marking chunk 0 as already reached by someone makes both CTAs wait there for a
    # ready flag that nothing will ever set.
    ws = lib.new_workspace(dims)
    ws.view(torch.int32)[0] = 1
    y = torch.empty((bsz, L, H * P), dtype=torch.bfloat16, device="cuda")
    t0 = time.time()
    lib.bimamba_ssd_fwd_rev(g["xbc"], g["dt"], g["A"], g["D"], g["conv_w"], None, None, None, y, ws,
                            heads=H, headdim=P, d_state=N)
    torch.cuda.synchronize()
    elapsed = time.time() - t0
    assert lib.bimamba_get_error() == lib.BIMAMBA_ERR_TIMEOUT
    assert elapsed < 30.0, elapsed            # each wait gives up after about two seconds
    assert lib.bimamba_get_error() == lib.BIMAMBA_OK   # reading the status cleared it

    # the same context, a fresh call (a CTA that gave up may leave counters set
    # in the poisoned workspace, so it is not reused): correct results
    y2 = torch.full((bsz, L, H * P), float("nan"), dtype=torch.bfloat16, device="cuda")
    lib.bimamba_ssd_fwd_rev(g["xbc"], g["dt"], g["A"], g["D"], g["conv_w"], None, None, None, y2,
                            lib.new_workspace(dims), heads=H, headdim=P, d_state=N)
    assert lib.bimamba_get_error() == lib.BIMAMBA_OK
    n = {k: to_np(v) for k, v in cpu.items()}
    ry = oracle.bimamba(n["xbc"], n["dt"], n["A"], n["D"], n["conv_w"], None, heads=H, headdim=P,
                        d_state=N)
    assert rel_err(to_np(y2), ry) <= TOL["bf16"]
