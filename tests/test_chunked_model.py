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


# ------------------------------------------------------------------ backward
def chunked_scan_backward(x, B, C, dt, A, D, dy, init=None):
    """Gradients of L = sum(dy * y) for one forward direction in the chunked
    form (natural units, decay factors evaluated directly), chunk by chunk
    from the last: a blueprint of the backward kernel.  Per chunk, with
    W[t,s] = (C_t . B_s) e^(c_t - c_s) dt_s and T[t,s] = (dY_t . x_s)
    e^(c_t - c_s) dt_s for s <= t (T is the Q x Q product dY X^T masked by
    the same decays), w_s = e^(c_last - c_s) dt_s, S_in the state entering
    the chunk and dS the adjoint of the state leaving it:
        dX    = W^T dY + D dY + w * (B dS^T)
        dB    = T^T C + w * (X dS)
        dC    = T B + e^c * (dY S_in)
        dS_in = e^(c_last) dS + (e^c * dY)^T C
    The prefix sums c collect dL/dc from W, the off-diagonal term and the
    state; dt receives them through suffix sums (c_j = A sum_{i <= j} dt_i)
    plus its direct terms, and A through sum_j dL/dc_j sum_{i <= j} dt_i."""
    bsz, L, H, P = x.shape
    N = B.shape[-1]
    g = {k: np.zeros_like(v) for k, v in (("x", x), ("B", B), ("C", C), ("dt", dt), ("A", A),
                                          ("D", D))}
    g["init"] = np.zeros((bsz, H, P, N))
    for b in range(bsz):
        for h in range(H):
            a_h = A[h]
            # forward, keeping the state entering every chunk
            S = np.zeros((P, N)) if init is None else init[b, h].copy()
            starts = list(range(0, L, Q))
            S_in = []
            for t0 in starts:
                S_in.append(S.copy())
                cnt = min(Q, L - t0)
                d = dt[b, t0:t0 + cnt, h]
                c = np.cumsum(d * a_h)
                Xc, Bc = x[b, t0:t0 + cnt, h], B[b, t0:t0 + cnt, 0]
                S = np.exp(c[-1]) * S + (Xc * (np.exp(c[-1] - c) * d)[:, None]).T @ Bc
            # backward, last chunk first
            dS = np.zeros((P, N))
            for k in range(len(starts) - 1, -1, -1):
                t0 = starts[k]
                cnt = min(Q, L - t0)
                d = dt[b, t0:t0 + cnt, h]
                c = np.cumsum(d * a_h)
                Xc, Bc, Cc = x[b, t0:t0 + cnt, h], B[b, t0:t0 + cnt, 0], C[b, t0:t0 + cnt, 0]
                dY = dy[b, t0:t0 + cnt, h]
                Sk = S_in[k]
                mask = np.tril(np.ones((cnt, cnt)))
                E = np.exp(np.minimum(c[:, None] - c[None, :], 0.0)) * mask   # e^(c_t - c_s), s <= t
                CB = Cc @ Bc.T
                W = CB * E * d[None, :]
                DYX = dY @ Xc.T                                  # (dY_t . x_s)
                T = DYX * E * d[None, :]                         # shares W's mask and decays
                wl = np.exp(c[-1] - c) * d                       # e^(c_last - c_s) dt_s
                ec = np.exp(c)
                SC = Cc @ Sk.T                                   # (S_in C_t), rows t
                # x, B, C, D
                g["x"][b, t0:t0 + cnt, h] += W.T @ dY + D[h] * dY + wl[:, None] * (Bc @ dS.T)
                g["B"][b, t0:t0 + cnt, 0] += T.T @ Cc + wl[:, None] * (Xc @ dS)
                g["C"][b, t0:t0 + cnt, 0] += T @ Bc + ec[:, None] * (dY @ Sk)
                g["D"][h] += np.sum(dY * Xc)
                # dL/dc_j and the direct dt_s terms
                dc = np.zeros(cnt)
                TW = DYX * W                                     # d/dc of the intra-chunk term
                dc += TW.sum(axis=1)
                dc -= TW.sum(axis=0)
                dc += ec * np.sum(dY * SC, axis=1)               # off-diagonal term e^(c_t) S_in C_t
                U = wl * np.einsum("pn,sp,sn->s", dS, Xc, Bc)    # state input, per source slot
                dc[-1] += np.exp(c[-1]) * np.sum(dS * Sk) + U.sum()
                dc -= U
                ddt = (DYX * CB * E).sum(axis=0) + np.exp(c[-1] - c) * np.einsum("pn,sp,sn->s", dS, Xc, Bc)
                # c_j = a_h * sum_{i <= j} dt_i
                suffix = np.cumsum(dc[::-1])[::-1]               # sum_{j >= i} dL/dc_j
                g["dt"][b, t0:t0 + cnt, h] += ddt + a_h * suffix
                g["A"][h] += np.sum(dc * np.cumsum(d))
                # the adjoint of the state entering this chunk
                dS = np.exp(c[-1]) * dS + (ec[:, None] * dY).T @ Cc
            g["init"][b, h] += dS
    return g


@pytest.mark.parametrize("case", [
    (300, (1.0, 16.0), -2.0),
    (257, (1e-3, 1e-2), -2.0),
    (130, (2.0, 16.0), -1.0),
])
def test_chunked_backward_equals_the_adjoint_recurrence(case):
    L, (a_lo, a_hi), dt_mu = case
    rng = np.random.default_rng(L + 1)
    H, P, N = 2, 3, 4
    x, B, C, dt, A, D = _inputs(rng, 1, L, H, P, N, a_lo, a_hi, dt_mu)
    init = rng.normal(0, 0.5, (1, H, P, N))
    dy = rng.normal(size=x.shape)
    got = chunked_scan_backward(x, B, C, dt, A, D, dy, init)
    ref = oracle.scan_backward(x, B, C, dt, A, D, dy, init=init)
    for k in ("x", "B", "C", "dt", "A", "D", "init"):
        scale = max(1.0, np.max(np.abs(ref[k])))
        assert np.max(np.abs(got[k] - ref[k])) <= 1e-9 * scale, k
