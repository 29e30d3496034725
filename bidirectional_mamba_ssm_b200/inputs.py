"""Seeded synthetic inputs shaped like the DiffuMamba mixer workloads.

This module is the one piece shared by the CUDA path's tests/benchmark and
by the oracle's tests.  It holds no arithmetic of the method itself: it only
draws random numbers and casts them.

Recipe (all draws from one ``torch.Generator`` seeded with ``seed``, in this
order; a normal is written N(mean, variance)):

  xbc     (batch, len, H*P + 2*G*N)  N(0, 1); the B and C channels are then
                                     multiplied by ``bc_scale``
  dt_raw  (batch, len, H)            N(-2, 0.5);  dt = softplus(dt_raw)
  A_u     (H)                        U[log a_lo, log a_hi];  A = -exp(A_u)
  D       (H)                        N(0, 1)
  conv_w  (ch, K)                    N(0, 1/4)
  conv_b  (ch)                       zero unless ``conv_bias`` is set, then N(0, 0.01)

Shapes follow the model configuration on the pages (d_model 2048, expand 2,
d_state 128, d_conv 4; "DiffuMamba" blog post, network-architecture listing).
The raw xBC, dt and output tensors are stored in ``dtype`` (fp32 or bf16);
A, D and the conv parameters stay fp32.
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    seqlen: int
    heads: int
    headdim: int
    d_state: int
    ngroups: int = 1
    d_conv: int = 4
    dtype: str = "bf16"          # "bf16" or "f32"
    bc_scale: float = 1.0

    @property
    def channels(self) -> int:
        return self.heads * self.headdim + 2 * self.ngroups * self.d_state

    @property
    def tokens(self) -> int:
        return self.batch * self.seqlen


# The workloads the benchmark and the parity tests use.
TINY_F32 = Workload("tiny-f32 b1 L256 H4x32 N16", 1, 256, 4, 32, 16, dtype="f32")
LAYER_1P3B = Workload("1.3B-layer b8 L4096 H64x64 N128 bf16", 8, 4096, 64, 64, 128,
                      dtype="bf16", bc_scale=1.0 / math.sqrt(128))
LONG_131K = Workload("long b1 L131072 H64x64 N128 bf16", 1, 131072, 64, 64, 128,
                     dtype="bf16", bc_scale=1.0 / math.sqrt(128))
# cached block decode: 32 streams, 64-token active block, 65536-token prefix
DECODE_STREAMS = 32
DECODE_BLOCK = 64
DECODE_PREFIX = 65536
SWEEP_LENGTHS = (1024, 4096, 16384, 65536, 262144)


def torch_dtype(name: str) -> torch.dtype:
    return {"bf16": torch.bfloat16, "f32": torch.float32}[name]


def make_inputs(w: Workload, seed: int = 0, *, a_range=(1.0, 16.0),
                conv_bias: bool = False, device="cpu", seqlen: int | None = None,
                batch: int | None = None):
    """Draw one seeded input set for workload ``w``.

    ``seqlen``/``batch`` override the workload's sizes (same recipe).
    ``a_range`` = (a_lo, a_hi) gives A in [-a_hi, -a_lo]; pass e.g.
    (1e-3, 1e-2) for long-memory decays.
    Returns a dict of tensors on ``device``.
    """
    L = w.seqlen if seqlen is None else seqlen
    bsz = w.batch if batch is None else batch
    H, P, N, G, K = w.heads, w.headdim, w.d_state, w.ngroups, w.d_conv
    ch = H * P + 2 * G * N
    dev = torch.device(device)
    g = torch.Generator(device=dev)
    g.manual_seed(seed)
    xbc = torch.randn((bsz, L, ch), generator=g, device=dev, dtype=torch.float32)
    if w.bc_scale != 1.0:
        xbc[..., H * P:] *= w.bc_scale
    dt_raw = torch.randn((bsz, L, H), generator=g, device=dev) * math.sqrt(0.5) - 2.0
    dt = torch.nn.functional.softplus(dt_raw)
    lo, hi = math.log(a_range[0]), math.log(a_range[1])
    A = -torch.exp(torch.rand((H,), generator=g, device=dev) * (hi - lo) + lo)
    D = torch.randn((H,), generator=g, device=dev)
    conv_w = torch.randn((ch, K), generator=g, device=dev) * 0.5
    conv_b = (torch.randn((ch,), generator=g, device=dev) * 0.1) if conv_bias else None
    td = torch_dtype(w.dtype)
    return {
        "xbc": xbc.to(td).contiguous(),
        "dt": dt.to(td).contiguous(),
        "A": A.float().contiguous(),
        "D": D.float().contiguous(),
        "conv_w": conv_w.float().contiguous(),
        "conv_b": None if conv_b is None else conv_b.float().contiguous(),
    }


def make_state(batch: int, heads: int, headdim: int, d_state: int, seed: int = 1,
               scale: float = 1.0, device="cpu"):
    """A seeded fp32 SSM state (batch, H, P, N), N(0, scale^2)."""
    g = torch.Generator(device=torch.device(device))
    g.manual_seed(seed)
    return (torch.randn((batch, heads, headdim, d_state), generator=g,
                        device=torch.device(device)) * scale).contiguous()


def make_tail(batch: int, d_conv: int, channels: int, dtype: str, seed: int = 2,
              bc_split: int | None = None, bc_scale: float = 1.0, device="cpu"):
    """A seeded raw conv tail (batch, d_conv, ch), same distribution as xbc."""
    g = torch.Generator(device=torch.device(device))
    g.manual_seed(seed)
    t = torch.randn((batch, d_conv, channels), generator=g, device=torch.device(device))
    if bc_split is not None and bc_scale != 1.0:
        t[..., bc_split:] *= bc_scale
    return t.to(torch_dtype(dtype)).contiguous()


def make_projections(d_model: int, heads: int, headdim: int, d_state: int, tokens: int,
                     seed: int = 0, *, d_inner_out: int | None = None, device="cpu"):
    """Seeded inputs and weights of the mixer's projections (bf16 storage;
    draws in fp32 from one torch.Generator, in this order):

      u       (tokens, d_model)          N(0, 1)
      w_in    (ch + H, d_model)          N(0, 1/d_model)   (rows: xBC, then dt)
      dt_bias (H)                        N(-2, 0.5)        (dt = softplus(u.w + b))
      w_out   (d_model, d_inner_out)     N(0, 1/d_inner_out), d_inner_out = H*P
                                         unless given (2*H*P for concatenated
                                         untied streams)
      y       (tokens, d_inner_out)      N(0, 1)           (a mixer output)
    """
    ch = heads * headdim + 2 * d_state
    k_out = heads * headdim if d_inner_out is None else d_inner_out
    dev = torch.device(device)
    g = torch.Generator(device=dev)
    g.manual_seed(seed)
    u = torch.randn((tokens, d_model), generator=g, device=dev)
    w_in = torch.randn((ch + heads, d_model), generator=g, device=dev) / math.sqrt(d_model)
    dt_bias = torch.randn((heads,), generator=g, device=dev) * math.sqrt(0.5) - 2.0
    w_out = torch.randn((d_model, k_out), generator=g, device=dev) / math.sqrt(k_out)
    y = torch.randn((tokens, k_out), generator=g, device=dev)
    bf = torch.bfloat16
    return {"u": u.to(bf).contiguous(), "w_in": w_in.to(bf).contiguous(),
            "dt_bias": dt_bias.float().contiguous(), "w_out": w_out.to(bf).contiguous(),
            "y": y.to(bf).contiguous()}
