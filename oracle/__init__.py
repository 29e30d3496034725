"""Double-precision CPU oracle for the bidirectional Mamba-2 mixer core.

TEST INFRASTRUCTURE ONLY.  Only the tests, ``__graft_entry__.smoke()`` and
the CPU-baseline leg of ``bench.py`` may import this package.  The product
library never loads it and shares no code with it.

The arithmetic lives in ``bimamba_oracle.c`` (plain C, double precision,
sequential recurrence, OpenMP only across independent (batch, head) pairs).
This module compiles it with gcc on first use and marshals numpy arrays.
Inputs given in a narrower type (bf16, fp32) are widened exactly to float64
first, so input quantisation never counts as error.

Parity status: every function here is pinned by the tests in
``tests/test_oracle_pins.py`` (brute-force quadratic form, closed forms,
flip identities, split/resume, hand-derived golden values).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "bimamba_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile the C oracle into oracle/liboracle.so (gcc, -O2, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp.%d" % os.getpid()
        cmd = ["gcc", "-O2", "-fPIC", "-shared", "-fopenmp", "-std=c99",
               "-o", tmp, _SRC, "-lm"]
        subprocess.check_call(cmd)
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB)
            dp = ctypes.POINTER(ctypes.c_double)
            i = ctypes.c_int
            lib.oracle_num_threads.restype = i
            lib.oracle_conv.argtypes = [dp, dp, dp, dp, i, i, i, i, i, i, dp]
            lib.oracle_scan.argtypes = [dp, dp, dp, dp, dp, dp, dp, i, i, i, i, i, i, i, dp, dp]
            lib.oracle_bimamba.argtypes = [dp, dp, dp, dp, dp, dp, dp, dp,
                                           i, i, i, i, i, i, i, dp, dp, dp, dp]
            lib.oracle_block_decode.argtypes = [dp, dp, dp, dp, dp, dp, dp, dp,
                                                i, i, i, i, i, i, i, dp, dp, dp]
            lib.oracle_bimamba_untied.argtypes = [dp] * 13 + [i] * 8 + [dp, dp]
            lib.oracle_scan_backward.argtypes = [dp] * 8 + [i] * 7 + [dp] * 7
            lib.oracle_conv_backward.argtypes = [dp] * 4 + [i] * 5 + [dp] * 3
            _lib = lib
    return _lib


def _f64(a):
    """Exact widening to a contiguous float64 numpy array (None passes through).

    torch tensors (including bfloat16) are widened through float32, which is
    exact for bf16 and fp32 values.
    """
    if a is None:
        return None
    if hasattr(a, "detach"):  # torch tensor
        import torch
        a = a.detach().to("cpu")
        if a.dtype in (torch.bfloat16, torch.float16):
            a = a.float()
        a = a.double().numpy()
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _ptr(a):
    if a is None:
        return None
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def num_threads() -> int:
    return int(_load().oracle_num_threads())


def conv(u, w, bias=None, tail=None, reverse=False, silu=True):
    """Depthwise causal (or mirrored) conv1d + optional SiLU.

    u: (batch, len, ch); w: (ch, K); bias: (ch); tail: (batch, K, ch).
    """
    lib = _load()
    u, w, bias, tail = _f64(u), _f64(w), _f64(bias), _f64(tail)
    bsz, L, ch = u.shape
    K = w.shape[1]
    out = np.empty_like(u)
    lib.oracle_conv(_ptr(u), _ptr(w), _ptr(bias), _ptr(tail), bsz, L, ch, K,
                    int(bool(reverse)), int(bool(silu)), _ptr(out))
    return out


def scan(x, B, C, dt, A, D, init=None, reverse=False, want_final=False):
    """One direction of the selective scan (sequential recurrence).

    x: (batch, len, H, P); B, C: (batch, len, G, N); dt: (batch, len, H);
    A, D: (H); init: (batch, H, P, N).  Returns y (and the final state).
    """
    lib = _load()
    x, B, C, dt, A, D, init = map(_f64, (x, B, C, dt, A, D, init))
    bsz, L, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    y = np.empty_like(x)
    fin = np.empty((bsz, H, P, N)) if want_final else None
    lib.oracle_scan(_ptr(x), _ptr(B), _ptr(C), _ptr(dt), _ptr(A), _ptr(D),
                    _ptr(init), bsz, L, H, P, N, G, int(bool(reverse)),
                    _ptr(y), _ptr(fin))
    return (y, fin) if want_final else y


def bimamba(xbc, dt, A, D, conv_w=None, conv_b=None, *, heads, headdim, d_state,
            ngroups=1, tail=None, init=None, want_final=False, want_dirs=False):
    """Full bidirectional mixer core: conv+SiLU per direction, scan both ways, sum.

    xbc: (batch, len, H*P + 2*G*N) raw; dt: (batch, len, H).
    Returns y (batch, len, H*P) [, final_state] [, (y_fwd, y_rev)].
    """
    lib = _load()
    xbc, dt, A, D, conv_w, conv_b, tail, init = map(
        _f64, (xbc, dt, A, D, conv_w, conv_b, tail, init))
    bsz, L, ch = xbc.shape
    H, P, N, G = heads, headdim, d_state, ngroups
    assert ch == H * P + 2 * G * N
    K = conv_w.shape[1] if conv_w is not None else 4
    y = np.empty((bsz, L, H * P))
    fin = np.empty((bsz, H, P, N)) if want_final else None
    yf = np.empty_like(y) if want_dirs else None
    yr = np.empty_like(y) if want_dirs else None
    lib.oracle_bimamba(_ptr(xbc), _ptr(dt), _ptr(A), _ptr(D), _ptr(conv_w),
                       _ptr(conv_b), _ptr(tail), _ptr(init), bsz, L, H, P, N, G,
                       K, _ptr(y), _ptr(fin), _ptr(yf), _ptr(yr))
    out = [y]
    if want_final:
        out.append(fin)
    if want_dirs:
        out.append((yf, yr))
    return out[0] if len(out) == 1 else tuple(out)


def scan_backward(x, B, C, dt, A, D, dy, init=None, reverse=False, grads=None):
    """Gradients of L = sum(dy * y) for one direction of the scan (no conv),
    y = scan(x, B, C, dt, A, D, init, reverse).  Returns a dict of float64
    arrays (x, B, C, dt, A, D, init); pass `grads` to accumulate into it."""
    lib = _load()
    x, B, C, dt, A, D, dy, init = map(_f64, (x, B, C, dt, A, D, dy, init))
    bsz, L, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    if grads is None:
        grads = {"x": np.zeros_like(x), "B": np.zeros_like(B), "C": np.zeros_like(C),
                 "dt": np.zeros_like(dt), "A": np.zeros_like(A), "D": np.zeros_like(D),
                 "init": np.zeros((bsz, H, P, N))}
    lib.oracle_scan_backward(_ptr(x), _ptr(B), _ptr(C), _ptr(dt), _ptr(A), _ptr(D), _ptr(init),
                             _ptr(dy), bsz, L, H, P, N, G, int(bool(reverse)), _ptr(grads["x"]),
                             _ptr(grads["B"]), _ptr(grads["C"]), _ptr(grads["dt"]),
                             _ptr(grads["A"]), _ptr(grads["D"]), _ptr(grads["init"]))
    return grads


def bimamba_backward(x, B, C, dt, A, D, dy, init=None):
    """Gradients of L = sum(dy * y) for the bidirectional scan without conv,
    y = scan(forward, from init) + scan(reverse, from zero): the two
    directions' adjoints summed (the initial state only enters forward)."""
    g = scan_backward(x, B, C, dt, A, D, dy, init=init, reverse=False)
    init_grad = g["init"].copy()
    g = scan_backward(x, B, C, dt, A, D, dy, init=None, reverse=True, grads=g)
    g["init"] = init_grad
    return g


def conv_backward(u, w, bias, dout, reverse=False):
    """Gradients of L = sum(dout * conv_silu(u)) w.r.t. u, w and bias (no
    tail): returns (du, dw, dbias)."""
    lib = _load()
    u, w, bias, dout = map(_f64, (u, w, bias, dout))
    bsz, L, ch = u.shape
    du, dw, db = np.zeros_like(u), np.zeros_like(w), np.zeros(ch)
    lib.oracle_conv_backward(_ptr(u), _ptr(w), _ptr(bias), _ptr(dout), bsz, L, ch, w.shape[1],
                             int(bool(reverse)), _ptr(du), _ptr(dw), _ptr(db))
    return du, dw, db


def bimamba_mixer_backward(xbc, dt, A, D, conv_w, conv_b, dy, *, heads, headdim, d_state,
                           init=None):
    """Gradients of L = sum(dy * y) for the whole bidirectional mixer core
    (conv+SiLU per direction, both scans, summed; one group): each
    direction's scan adjoint gives the gradient of its activated x, B and C,
    which its conv's backward carries to the raw xBC and the conv taps.
    Returns a dict: xbc, dt, A, D, conv_w, conv_b, init."""
    xbc, dt, A, D, conv_w, conv_b, dy, init = map(_f64, (xbc, dt, A, D, conv_w, conv_b, dy, init))
    bsz, L, ch = xbc.shape
    H, P, N = heads, headdim, d_state
    out = {"xbc": np.zeros_like(xbc), "dt": np.zeros_like(dt), "A": np.zeros_like(A),
           "D": np.zeros_like(D), "conv_w": np.zeros_like(conv_w), "conv_b": np.zeros(ch),
           "init": np.zeros((bsz, H, P, N))}
    for reverse in (False, True):
        act = conv(xbc, conv_w, conv_b, reverse=reverse)
        x = act[..., :H * P].reshape(bsz, L, H, P)
        Bm = act[..., H * P:H * P + N].reshape(bsz, L, 1, N)
        Cm = act[..., H * P + N:].reshape(bsz, L, 1, N)
        g = scan_backward(x, Bm, Cm, dt, A, D, dy.reshape(bsz, L, H, P),
                          init=None if reverse else init, reverse=reverse)
        dact = np.concatenate([g["x"].reshape(bsz, L, H * P), g["B"].reshape(bsz, L, N),
                               g["C"].reshape(bsz, L, N)], axis=-1)
        du, dw, db = conv_backward(xbc, conv_w, conv_b, dact, reverse=reverse)
        out["xbc"] += du
        out["conv_w"] += dw
        out["conv_b"] += db
        for k in ("dt", "A", "D"):
            out[k] += g[k]
        if not reverse:
            out["init"] += g["init"]
    return out


def bimamba_untied(xbc_f, xbc_r, dt_f, dt_r, A_f, A_r, D_f, D_r, conv_w_f=None, conv_w_r=None,
                   conv_b_f=None, conv_b_r=None, *, heads, headdim, d_state, ngroups=1,
                   init=None, concat=False, want_final=False):
    """Untied directions: each stream with its own parameters, outputs summed
    (y: (batch, len, H*P)) or concatenated per token as [forward | reverse]
    (y: (batch, len, 2*H*P)).  Returns y [, forward final state]."""
    lib = _load()
    (xbc_f, xbc_r, dt_f, dt_r, A_f, A_r, D_f, D_r, conv_w_f, conv_w_r, conv_b_f, conv_b_r,
     init) = map(_f64, (xbc_f, xbc_r, dt_f, dt_r, A_f, A_r, D_f, D_r, conv_w_f, conv_w_r,
                        conv_b_f, conv_b_r, init))
    bsz, L, ch = xbc_f.shape
    H, P, N, G = heads, headdim, d_state, ngroups
    assert ch == H * P + 2 * G * N and xbc_r.shape == xbc_f.shape
    K = 4
    for w in (conv_w_f, conv_w_r):
        if w is not None:
            K = w.shape[1]
    y = np.empty((bsz, L, (2 if concat else 1) * H * P))
    fin = np.empty((bsz, H, P, N)) if want_final else None
    lib.oracle_bimamba_untied(_ptr(xbc_f), _ptr(xbc_r), _ptr(dt_f), _ptr(dt_r), _ptr(A_f),
                              _ptr(A_r), _ptr(D_f), _ptr(D_r), _ptr(conv_w_f), _ptr(conv_w_r),
                              _ptr(conv_b_f), _ptr(conv_b_r), _ptr(init), bsz, L, H, P, N, G, K,
                              int(bool(concat)), _ptr(y), _ptr(fin))
    return (y, fin) if want_final else y


def block_decode(block, dt, A, D, conv_w, conv_b, state, tail, *, heads, headdim,
                 d_state, ngroups=1, want_commit=False):
    """Cached block decode: forward resumes from (state, tail); reverse covers
    the block only.  Returns y [, state_out, tail_out]."""
    lib = _load()
    block, dt, A, D, conv_w, conv_b, state, tail = map(
        _f64, (block, dt, A, D, conv_w, conv_b, state, tail))
    S, L, ch = block.shape
    H, P, N, G = heads, headdim, d_state, ngroups
    K = conv_w.shape[1]
    y = np.empty((S, L, H * P))
    so = np.empty((S, H, P, N)) if want_commit else None
    to = np.empty((S, K, ch)) if want_commit else None
    lib.oracle_block_decode(_ptr(block), _ptr(dt), _ptr(A), _ptr(D), _ptr(conv_w),
                            _ptr(conv_b), _ptr(state), _ptr(tail), S, L, H, P, N,
                            G, K, _ptr(y), _ptr(so), _ptr(to))
    return (y, so, to) if want_commit else y


# --------------------------------------------------------------------------
# The projections on either side of the mixer ("DiffuMamba" blog post,
# network-architecture listing: d_model = 2048, expand = 2; each mixer maps
# d_model to its inner width and back, the bidirectional block maps the
# concatenation of its two streams back to d with a Linear).  Weights are
# row-major (out_features, in_features), as a Linear layer stores them.

def softplus(x):
    """softplus(x) = log(1 + exp(x)), evaluated without overflow:
    max(x, 0) + log1p(exp(-|x|))."""
    x = _f64(x)
    return np.maximum(x, 0.0) + np.log1p(np.exp(-np.abs(x)))


def linear(x, w, bias=None):
    """A Linear layer: y[..., o] = sum_i x[..., i] w[o, i] (+ bias[o]), in
    float64 (one library matrix product)."""
    x, w, bias = _f64(x), _f64(w), _f64(bias)
    y = np.matmul(x, w.T)
    return y if bias is None else y + bias


def in_proj(u, w_in, dt_bias=None, *, heads, headdim, d_state, ngroups=1):
    """The mixer's input projection: the first ch = H*P + 2*G*N output rows of
    w_in give the raw xBC the conv reads, the last H rows the step sizes,
    dt = softplus(u . w_dt^T + dt_bias).  Returns (xbc, dt)."""
    ch = heads * headdim + 2 * ngroups * d_state
    w_in = _f64(w_in)
    assert w_in.shape[0] == ch + heads
    xbc = linear(u, w_in[:ch])
    dt = softplus(linear(u, w_in[ch:], dt_bias))
    return xbc, dt


def out_proj(y, w_out):
    """The mixer's output projection: out = y . w_out^T (w_out: (d_model,
    d_inner)); for untied directions with concatenated streams y is
    (tokens, 2*H*P) and w_out the block's fusion Linear."""
    return linear(y, w_out)
