"""The no-allocation decode entry point against the regular one.

bimamba_block_decode_noalloc serves callers that cannot allocate device
memory (a serving process whose pool already holds the whole device, or a
decode loop that must not allocate once it serves): it takes its scratch
from a fixed array inside the library instead of a caller workspace.  This
file checks, through the C ABI, that two calls in a row give the regular
entry point's results within the bf16 tolerance, and that a call too large
for the fixed array is refused.  It is collected last on purpose.
"""
import math

import pytest
import torch

from bidirectional_mamba_ssm_b200 import inputs as I
from parity_util import TOL, rel_err, to_np

pytestmark = pytest.mark.gpu


def _problem(seed):
    S, blk, H, P, N = 4, 64, 4, 64, 128
    w = I.Workload("noalloc", S, blk, H, P, N, dtype="bf16", bc_scale=1 / math.sqrt(N))
    g = {k: (None if v is None else v.cuda())
         for k, v in I.make_inputs(w, seed=seed, conv_bias=True, a_range=(1e-3, 1e-2)).items()}
    state = I.make_state(S, H, P, N, seed=seed + 1, scale=0.1).cuda()
    tail = I.make_tail(S, 4, w.channels, "bf16", seed=seed + 2, bc_split=H * P,
                       bc_scale=w.bc_scale).cuda()
    return w, g, state, tail


def test_noalloc_decode_matches_regular_decode_twice():
    from bidirectional_mamba_ssm_b200 import _lib as lib
    assert lib.bimamba_noalloc_scratch_bytes() >= 1 << 20
    for call in range(2):
        w, g, state, tail = _problem(seed=10 * call)
        S, blk, H, P, N = w.batch, w.seqlen, w.heads, w.headdim, w.d_state
        kw = dict(heads=H, headdim=P, d_state=N)
        y_ref = torch.full((S, blk, H * P), float("nan"), dtype=torch.bfloat16, device="cuda")
        so_ref = torch.full_like(state, float("nan"))
        lib.bimamba_block_decode(g["xbc"], g["dt"], g["A"], g["D"], g["conv_w"], g["conv_b"],
                                 state, tail, y_ref, so_ref, None,
                                 lib.new_workspace(lib.make_dims(S, blk, H, P, N, torch.bfloat16)),
                                 **kw)
        y = torch.full_like(y_ref, float("nan"))
        so = torch.full_like(so_ref, float("nan"))
        lib.bimamba_block_decode_noalloc(g["xbc"], g["dt"], g["A"], g["D"], g["conv_w"],
                                         g["conv_b"], state, tail, y, so, None, **kw)
        assert lib.bimamba_get_error() == lib.BIMAMBA_OK
        assert rel_err(to_np(y), to_np(y_ref)) <= TOL["bf16"], call
        assert rel_err(to_np(so), to_np(so_ref)) <= TOL["bf16"], call


def test_noalloc_decode_rejects_problems_beyond_the_scratch():
    from bidirectional_mamba_ssm_b200 import _lib as lib
    H, P, N = 64, 64, 128
    streams, blk = 64, 4096          # ~64 MiB of scratch, more than the fixed array
    dims = lib.make_dims(streams, blk, H, P, N, torch.bfloat16)
    assert lib.bimamba_workspace_bytes(dims) > lib.bimamba_noalloc_scratch_bytes()
    L = lib.library()
    import ctypes
    st = L.bimamba_block_decode_noalloc(ctypes.byref(dims), 16, 16, 16, 16, 16, None, 16, 16, 16,
                                        None, None, None)
    assert st == lib.BIMAMBA_ERR_WORKSPACE
