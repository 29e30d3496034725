"""Thin ctypes binding of libbimamba.so (the C ABI in include/bimamba.h).

Argument marshalling only: tensors are passed as device pointers, the stream
is torch's current CUDA stream unless one is given, and a non-OK status is
raised as BimambaError.  All computation happens in the library's kernels;
there is no fallback of any kind -- if the shared library is missing or
cannot be loaded, importing this module raises.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libbimamba.so")

BIMAMBA_OK = 0
BIMAMBA_ERR_INVALID = 1
BIMAMBA_ERR_UNSUPPORTED = 2
BIMAMBA_ERR_CUDA = 3
BIMAMBA_ERR_TIMEOUT = 4
BIMAMBA_ERR_WORKSPACE = 5
BIMAMBA_F32 = 0
BIMAMBA_BF16 = 1
BIMAMBA_FUSE_SUM = 0
BIMAMBA_FUSE_CONCAT = 1

# every symbol include/bimamba.h declares
EXPORTED = (
    "bimamba_version",
    "bimamba_launch_count",
    "bimamba_set_timing_events",
    "bimamba_strerror",
    "bimamba_get_error",
    "bimamba_conv_silu",
    "bimamba_workspace_bytes",
    "bimamba_launch_plan",
    "bimamba_ssd_fwd_rev",
    "bimamba_ssd_fwd_rev_untied",
    "bimamba_shard_states",
    "bimamba_ssd_fwd_rev_shard",
    "bimamba_block_decode",
    "bimamba_block_decode_pool",
    "bimamba_backward_workspace_bytes",
    "bimamba_ssd_fwd_rev_backward",
    "bimamba_in_proj",
    "bimamba_out_proj",
    "bimamba_noalloc_scratch_bytes",
    "bimamba_block_decode_noalloc",
)


class BimambaError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {strerror(status)} (status {status})")


class Dims(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int), ("len", ctypes.c_int), ("heads", ctypes.c_int),
                ("headdim", ctypes.c_int), ("d_state", ctypes.c_int), ("ngroups", ctypes.c_int),
                ("d_conv", ctypes.c_int), ("dtype", ctypes.c_int)]


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing; build it with "
                          "`python -m bidirectional_mamba_ssm_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    vp, i, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
    dp = ctypes.POINTER(Dims)
    lib.bimamba_version.restype = i
    lib.bimamba_version.argtypes = []
    lib.bimamba_launch_count.restype = ctypes.c_ulonglong
    lib.bimamba_launch_count.argtypes = []
    lib.bimamba_set_timing_events.restype = i
    lib.bimamba_set_timing_events.argtypes = [vp, vp]
    lib.bimamba_strerror.restype = ctypes.c_char_p
    lib.bimamba_strerror.argtypes = [i]
    lib.bimamba_get_error.restype = i
    lib.bimamba_get_error.argtypes = [vp]
    lib.bimamba_conv_silu.restype = i
    lib.bimamba_conv_silu.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, i, i, vp]
    lib.bimamba_workspace_bytes.restype = sz
    lib.bimamba_workspace_bytes.argtypes = [dp]
    lib.bimamba_launch_plan.restype = i
    lib.bimamba_launch_plan.argtypes = [dp, ctypes.POINTER(ctypes.c_int)]
    lib.bimamba_ssd_fwd_rev.restype = i
    lib.bimamba_ssd_fwd_rev.argtypes = [dp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
    lib.bimamba_ssd_fwd_rev_untied.restype = i
    lib.bimamba_ssd_fwd_rev_untied.argtypes = [dp] + [vp] * 15 + [i, vp, sz, vp]
    lib.bimamba_shard_states.restype = i
    lib.bimamba_shard_states.argtypes = [dp] + [vp] * 10 + [sz, vp]
    lib.bimamba_ssd_fwd_rev_shard.restype = i
    lib.bimamba_ssd_fwd_rev_shard.argtypes = [dp] + [vp] * 11 + [i, i, vp, vp, vp, sz, vp]
    lib.bimamba_block_decode.restype = i
    lib.bimamba_block_decode.argtypes = [dp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
    lib.bimamba_block_decode_pool.restype = i
    lib.bimamba_block_decode_pool.argtypes = [dp, vp, vp, vp, vp, vp, vp, vp, vp, i, vp, vp, vp, vp,
                                              sz, vp]
    lib.bimamba_backward_workspace_bytes.restype = sz
    lib.bimamba_backward_workspace_bytes.argtypes = [dp]
    lib.bimamba_ssd_fwd_rev_backward.restype = i
    lib.bimamba_ssd_fwd_rev_backward.argtypes = [dp] + [vp] * 16 + [sz, vp]
    lib.bimamba_in_proj.restype = i
    lib.bimamba_in_proj.argtypes = [i, i, i, i, i, vp, vp, vp, vp, vp, vp]
    lib.bimamba_out_proj.restype = i
    lib.bimamba_out_proj.argtypes = [i, i, i, vp, vp, vp, vp]
    lib.bimamba_noalloc_scratch_bytes.restype = sz
    lib.bimamba_noalloc_scratch_bytes.argtypes = []
    lib.bimamba_block_decode_noalloc.restype = i
    lib.bimamba_block_decode_noalloc.argtypes = [dp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp]
    return lib


_lib = _load()


def library() -> ctypes.CDLL:
    return _lib


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return BIMAMBA_F32
    if t.dtype == torch.bfloat16:
        return BIMAMBA_BF16
    raise BimambaError(BIMAMBA_ERR_UNSUPPORTED, f"dtype {t.dtype}")


def _check(status: int, where: str):
    if status != BIMAMBA_OK:
        raise BimambaError(status, where)


def bimamba_version() -> int:
    return _lib.bimamba_version()


def bimamba_launch_count() -> int:
    """Kernels this library has launched in this process so far."""
    return int(_lib.bimamba_launch_count())


def bimamba_set_timing_events(start=None, stop=None):
    """Record torch.cuda.Event `start`/`stop` around the main scan kernel of
    every later call on this thread (None, None switches it off)."""
    st = _lib.bimamba_set_timing_events(None if start is None else start.cuda_event,
                                        None if stop is None else stop.cuda_event)
    _check(st, "bimamba_set_timing_events")


def strerror(status: int) -> str:
    return _lib.bimamba_strerror(status).decode()


bimamba_strerror = strerror


def bimamba_get_error(stream=None) -> int:
    """Synchronise `stream`, then read and clear the device status word."""
    return _lib.bimamba_get_error(_stream(stream))


def make_dims(batch, seqlen, heads, headdim, d_state, dtype, ngroups=1, d_conv=4) -> Dims:
    code = dtype if isinstance(dtype, int) else (
        BIMAMBA_F32 if dtype in (torch.float32, "f32") else BIMAMBA_BF16)
    return Dims(batch, seqlen, heads, headdim, d_state, ngroups, d_conv, code)


def bimamba_workspace_bytes(dims: Dims) -> int:
    return int(_lib.bimamba_workspace_bytes(ctypes.byref(dims)))


def bimamba_launch_plan(dims: Dims) -> dict:
    """How a call with these dims is launched (host only): tensor-core path
    or not, segments per direction, chunks per segment, state-only items."""
    out = (ctypes.c_int * 4)()
    _check(_lib.bimamba_launch_plan(ctypes.byref(dims), out), "bimamba_launch_plan")
    return {"tensor_core": bool(out[0]), "segments": out[1], "seg_chunks": out[2],
            "items": out[3]}


def new_workspace(dims: Dims, device=None) -> torch.Tensor:
    """Zero-filled workspace of the size the library asks for (>= 256 bytes)."""
    n = max(256, bimamba_workspace_bytes(dims))
    return torch.zeros(n, dtype=torch.uint8, device=device or "cuda")


def bimamba_conv_silu(u, out, w, bias=None, tail=None, reverse=False, silu=True, stream=None):
    """out = SiLU(depthwise conv(u)) (or the pre-activation with silu=False)."""
    bsz, L, ch = u.shape
    st = _lib.bimamba_conv_silu(_ptr(u), _ptr(out), _ptr(w), _ptr(bias), _ptr(tail), bsz, L, ch,
                                w.shape[1], int(bool(reverse)), int(bool(silu)), _dtype_code(u),
                                _stream(stream))
    _check(st, "bimamba_conv_silu")
    return out


def bimamba_ssd_fwd_rev(xbc, dt, A, D, conv_w, conv_b, init_state, final_state, y, workspace,
                        *, heads, headdim, d_state, ngroups=1, stream=None, dims=None):
    """y = forward stream + reverse stream of the conv+SiLU'd selective scan."""
    if dims is None:
        bsz, L, _ = xbc.shape
        dims = make_dims(bsz, L, heads, headdim, d_state, _dtype_code(xbc), ngroups)
    wsz = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = _lib.bimamba_ssd_fwd_rev(ctypes.byref(dims), _ptr(xbc), _ptr(dt), _ptr(A), _ptr(D),
                                  _ptr(conv_w), _ptr(conv_b), _ptr(init_state), _ptr(final_state),
                                  _ptr(y), _ptr(workspace), wsz, _stream(stream))
    _check(st, "bimamba_ssd_fwd_rev")
    return y


def bimamba_ssd_fwd_rev_untied(fwd, rev, init_state, final_state, y, workspace, *, heads,
                               headdim, d_state, concat=False, ngroups=1, stream=None):
    """Untied directions: `fwd` and `rev` are dicts with keys xbc, dt, A, D,
    conv_w, conv_b (conv_w/conv_b may be None) holding each stream's own
    inputs.  y = forward + reverse (concat=False, (batch, len, H*P)) or
    per token [forward | reverse] (concat=True, (batch, len, 2*H*P))."""
    bsz, L, _ = fwd["xbc"].shape
    dims = make_dims(bsz, L, heads, headdim, d_state, _dtype_code(fwd["xbc"]), ngroups)
    wsz = 0 if workspace is None else workspace.numel() * workspace.element_size()
    g = lambda d, k: _ptr(d.get(k))
    st = _lib.bimamba_ssd_fwd_rev_untied(
        ctypes.byref(dims), g(fwd, "xbc"), g(rev, "xbc"), g(fwd, "dt"), g(rev, "dt"), g(fwd, "A"),
        g(rev, "A"), g(fwd, "D"), g(rev, "D"), g(fwd, "conv_w"), g(rev, "conv_w"), g(fwd, "conv_b"),
        g(rev, "conv_b"), _ptr(init_state), _ptr(final_state), _ptr(y),
        BIMAMBA_FUSE_CONCAT if concat else BIMAMBA_FUSE_SUM, _ptr(workspace), wsz, _stream(stream))
    _check(st, "bimamba_ssd_fwd_rev_untied")
    return y


def bimamba_shard_states(xbc, dt, A, conv_w, conv_b, tail, head, states, decays, workspace, *,
                         heads, headdim, d_state, ngroups=1, stream=None):
    """One sequence shard's end states from zero, (2, batch, H, P, N) [forward,
    reverse], and log2 decays (2, batch, H).  tail/head: (batch, 4, ch) raw
    tokens before/after the shard, or None (zeros)."""
    bsz, L, _ = xbc.shape
    dims = make_dims(bsz, L, heads, headdim, d_state, _dtype_code(xbc), ngroups)
    wsz = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = _lib.bimamba_shard_states(ctypes.byref(dims), _ptr(xbc), _ptr(dt), _ptr(A), _ptr(conv_w),
                                   _ptr(conv_b), _ptr(tail), _ptr(head), _ptr(states),
                                   _ptr(decays), _ptr(workspace), wsz, _stream(stream))
    _check(st, "bimamba_shard_states")
    return states, decays


def bimamba_ssd_fwd_rev_shard(xbc, dt, A, D, conv_w, conv_b, tail, head, init_state, all_states,
                              all_decays, rank, nranks, final_state, y, workspace, *, heads,
                              headdim, d_state, ngroups=1, stream=None):
    """One sequence shard's outputs, entering with the states the other
    shards hand on (all_states / all_decays: every rank's shard states)."""
    bsz, L, _ = xbc.shape
    dims = make_dims(bsz, L, heads, headdim, d_state, _dtype_code(xbc), ngroups)
    wsz = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = _lib.bimamba_ssd_fwd_rev_shard(
        ctypes.byref(dims), _ptr(xbc), _ptr(dt), _ptr(A), _ptr(D), _ptr(conv_w), _ptr(conv_b),
        _ptr(tail), _ptr(head), _ptr(init_state), _ptr(all_states), _ptr(all_decays), int(rank),
        int(nranks), _ptr(final_state), _ptr(y), _ptr(workspace), wsz, _stream(stream))
    _check(st, "bimamba_ssd_fwd_rev_shard")
    return y


def bimamba_block_decode(xbc_block, dt_block, A, D, conv_w, conv_b, state, tail, y, state_out,
                         tail_out, workspace, *, heads, headdim, d_state, ngroups=1, stream=None):
    """Cached block decode: forward resumes from (state, tail); reverse covers the block."""
    S, L, _ = xbc_block.shape
    dims = make_dims(S, L, heads, headdim, d_state, _dtype_code(xbc_block), ngroups)
    wsz = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = _lib.bimamba_block_decode(ctypes.byref(dims), _ptr(xbc_block), _ptr(dt_block), _ptr(A),
                                   _ptr(D), _ptr(conv_w), _ptr(conv_b), _ptr(state), _ptr(tail),
                                   _ptr(y), _ptr(state_out), _ptr(tail_out), _ptr(workspace), wsz,
                                   _stream(stream))
    _check(st, "bimamba_block_decode")
    return y


def bimamba_block_decode_pool(xbc_block, dt_block, A, D, conv_w, conv_b, state_pool, tail_pool,
                              slots, commit, y, workspace, *, heads, headdim, d_state, ngroups=1,
                              stream=None):
    """Cached block decode of a batch of streams held in a pool: row s uses
    pool entry slots[s] (int32 device tensor) and, where commit[s] != 0 (all
    rows when commit is None), writes its new state and conv tail back there."""
    S, L, _ = xbc_block.shape
    dims = make_dims(S, L, heads, headdim, d_state, _dtype_code(xbc_block), ngroups)
    wsz = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = _lib.bimamba_block_decode_pool(ctypes.byref(dims), _ptr(xbc_block), _ptr(dt_block), _ptr(A),
                                        _ptr(D), _ptr(conv_w), _ptr(conv_b), _ptr(state_pool),
                                        _ptr(tail_pool), int(state_pool.shape[0]), _ptr(slots),
                                        _ptr(commit), _ptr(y), _ptr(workspace), wsz, _stream(stream))
    _check(st, "bimamba_block_decode_pool")
    return y


def bimamba_backward_workspace_bytes(dims: Dims) -> int:
    return int(_lib.bimamba_backward_workspace_bytes(ctypes.byref(dims)))


def bimamba_ssd_fwd_rev_backward(xbc, dt, A, D, conv_w, conv_b, init_state, dy, *, heads, headdim,
                                 d_state, want_dinit=False, workspace=None, stream=None):
    """Gradients of sum(dy * y) for y = bimamba_ssd_fwd_rev(...): returns a dict
    of fp32 tensors xbc, dt, A, D, conv_w, conv_b (None without a bias) and
    init (None unless want_dinit)."""
    bsz, L, ch = xbc.shape
    dims = make_dims(bsz, L, heads, headdim, d_state, _dtype_code(xbc))
    dev = xbc.device
    f32 = torch.float32
    g = {"xbc": torch.empty((bsz, L, ch), dtype=f32, device=dev),
         "dt": torch.empty((bsz, L, heads), dtype=f32, device=dev),
         "A": torch.empty((heads,), dtype=f32, device=dev),
         "D": torch.empty((heads,), dtype=f32, device=dev),
         "conv_w": torch.empty((ch, 4), dtype=f32, device=dev),
         "conv_b": None if conv_b is None else torch.empty((ch,), dtype=f32, device=dev),
         "init": torch.empty((bsz, heads, headdim, d_state), dtype=f32, device=dev)
         if want_dinit else None}
    if workspace is None:
        workspace = torch.empty(max(256, bimamba_backward_workspace_bytes(dims)), dtype=torch.uint8,
                                device=dev)
    wsz = workspace.numel() * workspace.element_size()
    st = _lib.bimamba_ssd_fwd_rev_backward(
        ctypes.byref(dims), _ptr(xbc), _ptr(dt), _ptr(A), _ptr(D), _ptr(conv_w), _ptr(conv_b),
        _ptr(init_state), _ptr(dy), _ptr(g["xbc"]), _ptr(g["dt"]), _ptr(g["A"]), _ptr(g["D"]),
        _ptr(g["conv_w"]), _ptr(g["conv_b"]), _ptr(g["init"]), _ptr(workspace), wsz, _stream(stream))
    _check(st, "bimamba_ssd_fwd_rev_backward")
    return g


def bimamba_in_proj(u, w_in, dt_bias, xbc, dt, *, heads, headdim, d_state, stream=None):
    """[xbc | dt] = u . W_in^T with dt = softplus(. + dt_bias); u (tokens,
    d_model) bf16, w_in (ch + H, d_model) bf16, xbc (tokens, ch), dt (tokens, H)."""
    tokens, d_model = u.shape[-2] if u.dim() == 2 else u.shape[0] * u.shape[1], u.shape[-1]
    st = _lib.bimamba_in_proj(int(tokens), int(d_model), heads, headdim, d_state, _ptr(u), _ptr(w_in),
                              _ptr(dt_bias), _ptr(xbc), _ptr(dt), _stream(stream))
    _check(st, "bimamba_in_proj")
    return xbc, dt


def bimamba_out_proj(y, w_out, out, stream=None):
    """out = y . W_out^T; y (tokens, d_inner) bf16, w_out (d_model, d_inner) bf16."""
    d_inner = y.shape[-1]
    tokens = y.numel() // d_inner
    st = _lib.bimamba_out_proj(int(tokens), int(d_inner), int(w_out.shape[0]), _ptr(y), _ptr(w_out),
                               _ptr(out), _stream(stream))
    _check(st, "bimamba_out_proj")
    return out


def bimamba_noalloc_scratch_bytes() -> int:
    """Size of the fixed scratch array bimamba_block_decode_noalloc uses."""
    return int(_lib.bimamba_noalloc_scratch_bytes())


def bimamba_block_decode_noalloc(xbc_block, dt_block, A, D, conv_w, conv_b, state, tail, y,
                                 state_out, tail_out, *, heads, headdim, d_state, ngroups=1,
                                 stream=None):
    """Cached block decode for callers that cannot allocate device memory:
    same as bimamba_block_decode, but the scratch is the library's own fixed
    array (no workspace argument).  Calls sharing that array must not
    overlap on the GPU."""
    S, L, _ = xbc_block.shape
    dims = make_dims(S, L, heads, headdim, d_state, _dtype_code(xbc_block), ngroups)
    st = _lib.bimamba_block_decode_noalloc(ctypes.byref(dims), _ptr(xbc_block), _ptr(dt_block),
                                           _ptr(A), _ptr(D), _ptr(conv_w), _ptr(conv_b),
                                           _ptr(state), _ptr(tail), _ptr(y), _ptr(state_out),
                                           _ptr(tail_out), _stream(stream))
    _check(st, "bimamba_block_decode_noalloc")
    return y
