"""The chunked form the tensor-core kernel computes, restated in float64
numpy (test code only) and checked against the oracle's plain recurrence.

The kernel's algebra, per head, for chunks of Q = 128 walk steps with
c = inclusive prefix sums of dt*A*log2(e) inside the chunk:
    M[t,s] = (C_t . B_s) 2^(c_t - c_s) dt_s  for s <= t   (+ D on the diagonal)
    y_t    = (M X)_t + 2^(c_t) (S_in C_t)
    S_out  = 2^(c_last) S_in + sum_s 2^(c_last - c_s) dt_s x_s B_s^T
with 2^(c_t - c_s) evaluated the kernel's way:
  * s in a 32-slot block below t's: 2^(c_t - c_R) 2^(c_R - c_s), R = that block's last slot;
  * s in t's own 32-slot block whose whole decay is at most 2^60: through 4-slot sub-blocks,
    2^(c_t - c_R4) 2^(c_R4 - c_s), R4 = s | 3;
  * otherwise one exponential per element, 2^min(c_t - c_s, 0).
Pinning this model to the oracle checks the decomposition (and both
branches of the diagonal blocks) independently of the GPU."""
import math

import numpy as np
import pytest

import oracle

Q = 128
LOG2E = 1.4426950408889634


def _decay_factors(c, d):
    """F[t, s] = 2^(c_t - c_s) dt_s for s <= t (0 above), the kernel's way."""
    n = len(c)
    F = np.zeros((n, n))
    for t in range(n):
        bt = t // 32
        for s in range(t + 1):
            bs = s // 32
            if bs < bt:
                R = 32 * bs + 31
                f = 2.0 ** (c[t] - c[R]) * 2.0 ** (c[R] - c[s])
            elif c[32 * bt] - c[32 * bt + 31] <= 60.0:
                R4 = s | 3
                f = 2.0 ** (c[t] - c[R4]) * 2.0 ** (c[R4] - c[s])
            else:
                f = 2.0 ** min(c[t] - c[s], 0.0)
            F[t, s] = f * d[s]
    return F


def chunked_scan(x, B, C, dt, A, D, init=None):
    """One forward direction, (batch, len, H, P) etc. as oracle.scan, one group."""
    bsz, L, H, P = x.shape
    N = B.shape[-1]
    y = np.zeros_like(x)
    fin = np.zeros((bsz, H, P, N))
    for b in range(bsz):
        for h in range(H):
            S = np.zeros((P, N)) if init is None else init[b, h].copy()
            for t0 in range(0, L, Q):
                cnt = min(Q, L - t0)
                d = np.zeros(Q)
                d[:cnt] = dt[b, t0:t0 + cnt, h]
                c = np.cumsum(d * A[h] * LOG2E)
                Bc = np.zeros((Q, N))
                Cc = np.zeros((Q, N))
                Xc = np.zeros((Q, P))
                Bc[:cnt] = B[b, t0:t0 + cnt, 0]
                Cc[:cnt] = C[b, t0:t0 + cnt, 0]
                Xc[:cnt] = x[b, t0:t0 + cnt, h]
                M = (Cc @ Bc.T) * _decay_factors(c, d) + np.diag(np.full(Q, D[h]))
                Y = M @ Xc + (2.0 ** c)[:, None] * (Cc @ S.T)
                w = 2.0 ** (c[-1] - c) * d
                S = 2.0 ** c[-1] * S + (Xc * w[:, None]).T @ Bc
                y[b, t0:t0 + cnt, h] = Y[:cnt]
            fin[b, h] = S
    return y, fin


def _inputs(rng, bsz, L, H, P, N, a_lo, a_hi, dt_mu):
    x = rng.normal(size=(bsz, L, H, P))
    B = rng.normal(size=(bsz, L, 1, N)) / math.sqrt(N)
    C = rng.normal(size=(bsz, L, 1, N)) / math.sqrt(N)
    dt = np.log1p(np.exp(rng.normal(dt_mu, 0.5, (bsz, L, H))))
    A = -np.exp(rng.uniform(math.log(a_lo), math.log(a_hi), H))
    D = rng.normal(size=H)
    return x, B, C, dt, A, D


@pytest.mark.parametrize("case", [
    # L, a range, dt mean (pre-softplus): the workloads' decays, long memory, and
    # decays steep enough that one head's diagonal blocks take the per-element branch
    (300, (1.0, 16.0), -2.0),
    (257, (1e-3, 1e-2), -2.0),
    (200, (2.0, 16.0), -1.0),
])
def test_chunked_form_equals_the_recurrence(case):
    L, (a_lo, a_hi), dt_mu = case
    rng = np.random.default_rng(L)
    H, P, N = 2, 4, 8
    x, B, C, dt, A, D = _inputs(rng, 1, L, H, P, N, a_lo, a_hi, dt_mu)
    init = rng.normal(0, 0.5, (1, H, P, N))
    y, fin = chunked_scan(x, B, C, dt, A, D, init)
    ry, rfin = oracle.scan(x, B, C, dt, A, D, init=init, want_final=True)
    scale = max(1.0, np.max(np.abs(ry)))
    assert np.max(np.abs(y - ry)) <= 1e-10 * scale
    assert np.max(np.abs(fin - rfin)) <= 1e-10 * max(1.0, np.max(np.abs(rfin)))


def test_steep_case_uses_both_diagonal_branches():
    """In the steep case one head's diagonal blocks decay by at most 2^60
    (sub-block branch) and the other's by more (per-element branch), so the
    test above covers both."""
    rng = np.random.default_rng(200)
    x, B, C, dt, A, D = _inputs(rng, 1, 200, 2, 4, 8, 2.0, 16.0, -1.0)
    spans = []
    for h in range(2):
        c = np.cumsum(dt[0, :128, h] * A[h] * LOG2E)
        spans += [c[32 * k] - c[32 * k + 31] for k in range(4)]
    assert min(spans) <= 60.0 < max(spans)
