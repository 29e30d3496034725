"""Helpers shared by the GPU parity tests: error metric, head/stream sampling.

Error metric (fixed before any kernel was written):
    err = max_i |g_i - r_i| / max_i |r_i|
over one output tensor (per sampled head group / stream).  Bars: 1e-4 for
fp32 activations, 2e-2 for bf16 activations (fp32 state and accumulation).
Integer/index work (conv padding and tap order) is compared bit for bit.
"""
import numpy as np
import torch

TOL = {"f32": 1e-4, "bf16": 2e-2}


def rel_err(got, ref) -> float:
    g = np.asarray(got, dtype=np.float64)
    r = np.asarray(ref, dtype=np.float64)
    assert g.shape == r.shape, (g.shape, r.shape)
    den = float(np.max(np.abs(r))) if r.size else 1.0
    return float(np.max(np.abs(g - r))) / max(den, 1e-300) if r.size else 0.0


def to_np(t):
    if t is None:
        return None
    t = t.detach().cpu()
    if t.dtype in (torch.bfloat16, torch.float16):
        t = t.float()
    return t.double().numpy()


def head_subset(inp, heads, H, P, N):
    """Slice one input set to a subset of heads (x channels, dt, A, D, conv
    rows).  B and C are shared by all heads (one group) and kept whole.  The
    per-channel conv and the per-head scan make this slice exact."""
    heads = list(heads)
    xcols = np.concatenate([np.arange(h * P, (h + 1) * P) for h in heads])
    bc = np.arange(H * P, H * P + 2 * N)
    cols = np.concatenate([xcols, bc])
    out = {
        "xbc": inp["xbc"][..., cols],
        "dt": inp["dt"][..., heads],
        "A": inp["A"][heads],
        "D": inp["D"][heads],
        "conv_w": None if inp.get("conv_w") is None else inp["conv_w"][cols],
        "conv_b": None if inp.get("conv_b") is None else inp["conv_b"][cols],
    }
    return out, xcols


def y_cols(heads, P):
    return np.concatenate([np.arange(h * P, (h + 1) * P) for h in heads])
