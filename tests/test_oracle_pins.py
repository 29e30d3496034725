"""Pins for the CPU oracle: each check compares it with something other than
itself -- a brute-force materialised quadratic form, closed forms, library
routines (numpy cumsum / convolve), hand-derived values under tests/golden,
and invariants (flip identity, split/resume, decode == recompute).

Each pin is chosen so that a plausible mistake in the oracle (a dropped term,
a wrong sign or index, a transposed operand, an off-by-one in the decay
window or the conv taps) fails at least one of them.
"""
import math
import os

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    vals = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            k, *v = line.split()
            vals[k] = np.array([float(t) for t in v])
    return vals


def _rand(rng, bsz, L, H, P, N, G=1, a_lo=1.0, a_hi=16.0):
    x = rng.standard_normal((bsz, L, H, P))
    B = rng.standard_normal((bsz, L, G, N))
    C = rng.standard_normal((bsz, L, G, N))
    dt = np.log1p(np.exp(rng.normal(-2.0, math.sqrt(0.5), (bsz, L, H))))
    A = -np.exp(rng.uniform(math.log(a_lo), math.log(a_hi), H))
    D = rng.standard_normal(H)
    return x, B, C, dt, A, D


def _xbc(x, B, C):
    bsz, L, H, P = x.shape
    return np.concatenate([x.reshape(bsz, L, H * P), B.reshape(bsz, L, -1),
                           C.reshape(bsz, L, -1)], axis=-1)


def _brute_force(x, B, C, dt, A, D):
    """Materialised quadratic (semiseparable) form of both directions.

    M_f[t,s] = (C_t . B_s) exp(A sum_{r=s+1..t} dt_r) dt_s      (s <= t)
    M_r[t,s] = (C_t . B_s) exp(A sum_{r=t..s-1} dt_r) dt_s      (s >= t)
    y = (M_f + M_r) x + 2 D x
    Built with explicit double loops over (t, s); independent of the
    sequential recurrence.
    """
    bsz, L, H, P = x.shape
    G = B.shape[2]
    hpg = H // G
    y = np.zeros_like(x)
    for b in range(bsz):
        for h in range(H):
            g = h // hpg
            CB = C[b, :, g, :] @ B[b, :, g, :].T          # (t, s)
            M = np.zeros((L, L))
            for t in range(L):
                for s in range(L):
                    if s <= t:
                        seg = dt[b, s + 1:t + 1, h].sum()
                        M[t, s] += CB[t, s] * math.exp(A[h] * seg) * dt[b, s, h]
                    if s >= t:
                        seg = dt[b, t:s, h].sum()
                        M[t, s] += CB[t, s] * math.exp(A[h] * seg) * dt[b, s, h]
            y[b, :, h, :] = M @ x[b, :, h, :] + 2.0 * D[h] * x[b, :, h, :]
    return y


@pytest.mark.parametrize("L,H,P,N,G", [(1, 1, 1, 1, 1), (7, 2, 3, 4, 1),
                                       (33, 4, 2, 5, 2), (64, 2, 4, 8, 1)])
@pytest.mark.parametrize("memory", ["short", "long"])
def test_bidirectional_equals_quadratic_form(L, H, P, N, G, memory):
    rng = np.random.default_rng(L * 1000 + H * 10 + N)
    a = (1.0, 16.0) if memory == "short" else (1e-3, 1e-2)
    x, B, C, dt, A, D = _rand(rng, 2, L, H, P, N, G, *a)
    y = oracle.bimamba(_xbc(x, B, C), dt, A, D, heads=H, headdim=P, d_state=N, ngroups=G)
    ref = _brute_force(x, B, C, dt, A, D).reshape(2, L, H * P)
    assert np.max(np.abs(y - ref)) <= 1e-12 * max(1.0, np.max(np.abs(ref)))


def test_golden_hand_scalar():
    g = _golden("scan_hand.txt")
    x = np.array([1.0, 2.0, 3.0]).reshape(1, 3, 1, 1)
    one = np.ones((1, 3, 1, 1))
    dt = np.ones((1, 3, 1))
    A = np.array([-math.log(2.0)])
    for D, key in ((0.0, "case1_y_D0"), (0.5, "case1_y_D05")):
        y, fin = oracle.bimamba(_xbc(x, one, one), dt, A, np.array([D]), heads=1,
                                headdim=1, d_state=1, want_final=True)
        np.testing.assert_allclose(y.ravel(), g[key], rtol=0, atol=1e-14)
        np.testing.assert_allclose(fin.ravel(), g["case1_final"], rtol=0, atol=1e-14)


def test_golden_hand_matrix_orientation():
    g = _golden("scan_hand.txt")
    x = np.array([[1.0, 0.0], [0.0, 1.0]]).reshape(1, 2, 1, 2)
    B = np.array([[1.0, 0.0], [0.0, 2.0]]).reshape(1, 2, 1, 2)
    C = np.array([[1.0, 1.0], [3.0, 0.0]]).reshape(1, 2, 1, 2)
    dt = np.ones((1, 2, 1))
    y, fin = oracle.bimamba(_xbc(x, B, C), dt, np.array([-math.log(2.0)]),
                            np.array([0.0]), heads=1, headdim=2, d_state=2,
                            want_final=True)
    np.testing.assert_allclose(y.ravel(), g["case2_y"], rtol=0, atol=1e-14)
    np.testing.assert_allclose(fin.ravel(), g["case2_final"], rtol=0, atol=1e-14)


def test_golden_hand_conv():
    g = _golden("conv_hand.txt")
    u = g["u"].reshape(1, 4, 1)
    cases = [((1, 0, 0, 0), "w_shift_fwd", "w_shift_rev"),
             ((1, 2, 3, 4), "w_1234_fwd", "w_1234_rev")]
    for w, kf, kr in cases:
        w = np.array(w, dtype=float).reshape(1, 4)
        f = oracle.conv(u, w, reverse=False, silu=False).ravel()
        r = oracle.conv(u, w, reverse=True, silu=False).ravel()
        np.testing.assert_array_equal(f, g[kf])
        np.testing.assert_array_equal(r, g[kr])
    ident = oracle.conv(u, np.array([[0, 0, 0, 1.0]]), silu=False).ravel()
    np.testing.assert_array_equal(ident, g["u"])
    tail = g["tail"].reshape(1, 4, 1)
    f = oracle.conv(u, np.array([[1, 2, 3, 4.0]]), tail=tail, silu=False).ravel()
    np.testing.assert_array_equal(f, g["w_1234_fwd_tail"])


def test_conv_matches_numpy_convolve_and_silu():
    rng = np.random.default_rng(5)
    bsz, L, ch, K = 2, 37, 6, 4
    u = rng.standard_normal((bsz, L, ch))
    w = rng.standard_normal((ch, K))
    bias = rng.standard_normal(ch)
    tail = rng.standard_normal((bsz, K, ch))
    f = oracle.conv(u, w, bias, tail=tail, reverse=False, silu=True)
    r = oracle.conv(u, w, bias, reverse=True, silu=True)
    for b in range(bsz):
        for c in range(ch):
            full = np.concatenate([tail[b, :, c], u[b, :, c]])
            pre_f = np.convolve(full, w[c, ::-1])[K:K + L] + bias[c]
            pre_r = np.convolve(u[b, ::-1, c], w[c, ::-1])[:L][::-1] + bias[c]
            np.testing.assert_allclose(f[b, :, c], pre_f / (1 + np.exp(-pre_f)), rtol=1e-13, atol=1e-13)
            np.testing.assert_allclose(r[b, :, c], pre_r / (1 + np.exp(-pre_r)), rtol=1e-13, atol=1e-13)


def test_a_zero_is_prefix_sum():
    """A = 0: every decay is 1; with B = C = e_0 the forward stream is the
    running sum of dt*x (numpy cumsum), the reverse stream the suffix sum."""
    rng = np.random.default_rng(7)
    bsz, L, H, P, N = 2, 50, 3, 4, 5
    x = rng.standard_normal((bsz, L, H, P))
    dt = rng.uniform(0.01, 1.0, (bsz, L, H))
    B = np.zeros((bsz, L, 1, N)); B[..., 0] = 1.0
    C = B.copy()
    A = np.zeros(H)
    D = rng.standard_normal(H)
    y, (yf, yr) = oracle.bimamba(_xbc(x, B, C), dt, A, D, heads=H, headdim=P,
                                 d_state=N, want_dirs=True)
    dx = dt[..., None] * x
    pre = np.cumsum(dx, axis=1) + D[None, None, :, None] * x
    suf = np.cumsum(dx[:, ::-1], axis=1)[:, ::-1] + D[None, None, :, None] * x
    np.testing.assert_allclose(yf, pre.reshape(yf.shape), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(yr, suf.reshape(yr.shape), rtol=1e-12, atol=1e-12)


def test_length_one_closed_form():
    rng = np.random.default_rng(11)
    H, P, N = 3, 4, 6
    x, B, C, dt, A, D = _rand(rng, 1, 1, H, P, N)
    h0 = rng.standard_normal((1, H, P, N))
    y = oracle.bimamba(_xbc(x, B, C), dt, A, D, heads=H, headdim=P, d_state=N, init=h0)
    cb = float(C[0, 0, 0] @ B[0, 0, 0])
    for h in range(H):
        d = dt[0, 0, h]
        xv = x[0, 0, h]
        fwd = math.exp(d * A[h]) * (h0[0, h] @ C[0, 0, 0]) + cb * d * xv + D[h] * xv
        rev = cb * d * xv + D[h] * xv
        np.testing.assert_allclose(y[0, 0, h * P:(h + 1) * P], fwd + rev, rtol=1e-13, atol=1e-13)


def test_scalar_geometric_closed_form():
    """P = N = 1, constant dt, A, x and B = C = 1: the forward stream is a
    geometric series dt*x*(1-a^(t+1))/(1-a) + D x, the reverse one mirrors it."""
    L = 40
    dt, A, xv, D = 0.3, -0.7, 1.25, 0.4
    a = math.exp(dt * A)
    x = np.full((1, L, 1, 1), xv)
    one = np.ones((1, L, 1, 1))
    y = oracle.bimamba(_xbc(x, one, one), np.full((1, L, 1), dt), np.array([A]),
                       np.array([D]), heads=1, headdim=1, d_state=1).ravel()
    t = np.arange(L)
    fwd = dt * xv * (1 - a ** (t + 1)) / (1 - a) + D * xv
    rev = dt * xv * (1 - a ** (L - t)) / (1 - a) + D * xv
    np.testing.assert_allclose(y, fwd + rev, rtol=1e-13)


def test_infinite_decay_keeps_only_the_diagonal():
    rng = np.random.default_rng(13)
    H, P, N, L = 2, 3, 4, 9
    x, B, C, dt, _, D = _rand(rng, 1, L, H, P, N)
    A = np.full(H, -1e30)
    y = oracle.bimamba(_xbc(x, B, C), dt, A, D, heads=H, headdim=P, d_state=N)
    cb = np.einsum("tn,tn->t", C[0, :, 0], B[0, :, 0])
    want = 2 * (cb[:, None, None] * dt[0, :, :, None] * x[0] + D[None, :, None] * x[0])
    np.testing.assert_allclose(y[0], want.reshape(L, H * P), rtol=1e-13, atol=1e-13)


def test_flip_identities():
    """reverse stream == flip(forward(flip(input))), for the conv and the
    scan separately, and the tied bidirectional output is flip-equivariant."""
    rng = np.random.default_rng(17)
    bsz, L, H, P, N = 2, 29, 2, 3, 4
    x, B, C, dt, A, D = _rand(rng, bsz, L, H, P, N)
    ch = H * P + 2 * N
    u = rng.standard_normal((bsz, L, ch))
    w = rng.standard_normal((ch, 4))
    r = oracle.conv(u, w, reverse=True)
    f = oracle.conv(u[:, ::-1], w, reverse=False)[:, ::-1]
    np.testing.assert_allclose(r, f, rtol=0, atol=1e-14)
    yr = oracle.scan(x, B, C, dt, A, D, reverse=True)
    yf = oracle.scan(x[:, ::-1], B[:, ::-1], C[:, ::-1], dt[:, ::-1], A, D)[:, ::-1]
    np.testing.assert_allclose(yr, yf, rtol=1e-13, atol=1e-13)
    y = oracle.bimamba(u, dt, A, D, w, heads=H, headdim=P, d_state=N)
    yflip = oracle.bimamba(u[:, ::-1], dt[:, ::-1], A, D, w, heads=H, headdim=P, d_state=N)
    np.testing.assert_allclose(y, yflip[:, ::-1], rtol=1e-12, atol=1e-12)


def test_linearity_in_x():
    rng = np.random.default_rng(19)
    x, B, C, dt, A, D = _rand(rng, 1, 21, 2, 3, 4)
    x2 = rng.standard_normal(x.shape)
    y1 = oracle.scan(x, B, C, dt, A, D)
    y2 = oracle.scan(x2, B, C, dt, A, D)
    y12 = oracle.scan(2.0 * x - 3.0 * x2, B, C, dt, A, D)
    np.testing.assert_allclose(y12, 2.0 * y1 - 3.0 * y2, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("split", [1, 5, 16, 30])
def test_split_resume(split):
    """scan(0..L) == scan(l..L | final_state(0..l)) for the forward stream."""
    rng = np.random.default_rng(23)
    x, B, C, dt, A, D = _rand(rng, 2, 31, 2, 3, 5, 1, 1e-3, 1e-2)
    y, fin = oracle.scan(x, B, C, dt, A, D, want_final=True)
    y1, s1 = oracle.scan(x[:, :split], B[:, :split], C[:, :split], dt[:, :split], A, D, want_final=True)
    y2, s2 = oracle.scan(x[:, split:], B[:, split:], C[:, split:], dt[:, split:], A, D, init=s1, want_final=True)
    np.testing.assert_allclose(np.concatenate([y1, y2], axis=1), y, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(s2, fin, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("prefix", [0, 2, 3, 17])
def test_block_decode_equals_recompute(prefix):
    """Cached decode of a block == the forward stream of a full recompute over
    prefix + block at the block positions, plus the reverse stream of the
    block alone (block-causal reading of the cached-decode pages)."""
    rng = np.random.default_rng(29 + prefix)
    S, blk, H, P, N, K = 2, 11, 2, 3, 4, 4
    ch = H * P + 2 * N
    u = rng.standard_normal((S, prefix + blk, ch))
    dt = np.log1p(np.exp(rng.normal(-2.0, 0.7, (S, prefix + blk, H))))
    A = -np.exp(rng.uniform(math.log(1e-3), math.log(1.0), H))
    D = rng.standard_normal(H)
    w = rng.standard_normal((ch, K)) * 0.5
    bias = rng.standard_normal(ch) * 0.1
    # prefix summary produced by the oracle itself: state after the prefix and
    # its last K raw tokens (zeros where the prefix is shorter than K)
    if prefix:
        _, state = oracle.bimamba(u[:, :prefix], dt[:, :prefix], A, D, w, bias,
                                  heads=H, headdim=P, d_state=N, want_final=True)
    else:
        state = np.zeros((S, H, P, N))
    tail = np.zeros((S, K, ch))
    take = min(prefix, K)
    if take:
        tail[:, K - take:] = u[:, prefix - take:prefix]
    y, so, to = oracle.block_decode(u[:, prefix:], dt[:, prefix:], A, D, w, bias,
                                    state, tail, heads=H, headdim=P, d_state=N,
                                    want_commit=True)
    _, fin, (yf_full, _) = oracle.bimamba(u, dt, A, D, w, bias, heads=H, headdim=P,
                                          d_state=N, want_final=True, want_dirs=True)
    _, (_, yr_blk) = oracle.bimamba(u[:, prefix:], dt[:, prefix:], A, D, w, bias,
                                    heads=H, headdim=P, d_state=N, want_dirs=True)
    np.testing.assert_allclose(y, yf_full[:, prefix:] + yr_blk, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(so, fin, rtol=1e-12, atol=1e-12)
    full_tail = np.concatenate([np.zeros((S, K, ch)), u], axis=1)[:, -K:]
    np.testing.assert_array_equal(to, full_tail)


def test_decode_golden_scalar():
    """Case 1 of scan_hand.txt split as prefix (1,2) + block (3): the forward
    state after the prefix is 2.5; the block output is 0.5*2.5+3 (forward,
    resumed) + 3 (reverse over the block alone) = 7.25, which equals the full
    bidirectional output at the last position."""
    one = np.ones((1, 1, 1))
    u = np.array([[[3.0, 1.0, 1.0]]])          # x=3, B=1, C=1, no conv
    y = oracle.bimamba(u, one, np.array([-math.log(2.0)]), np.array([0.0]),
                       heads=1, headdim=1, d_state=1, init=np.full((1, 1, 1, 1), 2.5))
    assert abs(y.ravel()[0] - 7.25) < 1e-14


# ------------------------------------------------------- untied directions
def _brute_force_dir(x, B, C, dt, A, D, reverse):
    """One direction of the materialised quadratic form (no conv):
    forward  M[t,s] = (C_t . B_s) exp(A sum_{r=s+1..t} dt_r) dt_s   (s <= t)
    reverse  M[t,s] = (C_t . B_s) exp(A sum_{r=t..s-1} dt_r) dt_s   (s >= t)
    y = M x + D x.  Explicit double loops, independent of the recurrence."""
    bsz, L, H, P = x.shape
    G = B.shape[2]
    hpg = H // G
    y = np.zeros_like(x)
    for b in range(bsz):
        for h in range(H):
            g = h // hpg
            CB = C[b, :, g, :] @ B[b, :, g, :].T
            M = np.zeros((L, L))
            for t in range(L):
                for s in range(L):
                    if not reverse and s <= t:
                        M[t, s] = CB[t, s] * math.exp(A[h] * dt[b, s + 1:t + 1, h].sum()) * dt[b, s, h]
                    if reverse and s >= t:
                        M[t, s] = CB[t, s] * math.exp(A[h] * dt[b, t:s, h].sum()) * dt[b, s, h]
            y[b, :, h, :] = M @ x[b, :, h, :] + D[h] * x[b, :, h, :]
    return y


@pytest.mark.parametrize("L,H,P,N,G", [(1, 1, 1, 1, 1), (9, 2, 3, 4, 1), (40, 4, 2, 5, 2)])
@pytest.mark.parametrize("memory", ["short", "long"])
@pytest.mark.parametrize("concat", [False, True])
def test_untied_equals_quadratic_forms(L, H, P, N, G, memory, concat):
    """Untied directions (separate x, B, C, dt, A, D per stream, as in the
    blog's two-module listing): the sum, or the per-token concatenation
    [forward | reverse], of two independently parameterised quadratic forms."""
    rng = np.random.default_rng(L * 7 + H + 100 * concat)
    a = (1.0, 16.0) if memory == "short" else (1e-3, 1e-2)
    xf, Bf, Cf, dtf, Af, Df = _rand(rng, 2, L, H, P, N, G, *a)
    xr, Br, Cr, dtr, Ar, Dr = _rand(rng, 2, L, H, P, N, G, *a)
    y = oracle.bimamba_untied(_xbc(xf, Bf, Cf), _xbc(xr, Br, Cr), dtf, dtr, Af, Ar, Df, Dr,
                              heads=H, headdim=P, d_state=N, ngroups=G, concat=concat)
    yf = _brute_force_dir(xf, Bf, Cf, dtf, Af, Df, False).reshape(2, L, H * P)
    yr = _brute_force_dir(xr, Br, Cr, dtr, Ar, Dr, True).reshape(2, L, H * P)
    ref = np.concatenate([yf, yr], axis=-1) if concat else yf + yr
    assert y.shape == ref.shape
    assert np.max(np.abs(y - ref)) <= 1e-12 * max(1.0, np.max(np.abs(ref)))


def test_untied_with_equal_parameters_is_the_tied_mixer():
    rng = np.random.default_rng(5)
    L, H, P, N = 30, 2, 4, 8
    x, B, C, dt, A, D = _rand(rng, 2, L, H, P, N)
    u = _xbc(x, B, C)
    ch = u.shape[-1]
    w = rng.normal(0, 0.5, (ch, 4))
    bias = rng.normal(0, 0.1, ch)
    init = rng.normal(0, 0.3, (2, H, P, N))
    ref, rfin = oracle.bimamba(u, dt, A, D, w, bias, heads=H, headdim=P, d_state=N, init=init,
                               want_final=True, want_dirs=False)
    y, fin = oracle.bimamba_untied(u, u, dt, dt, A, A, D, D, w, w, bias, bias, heads=H, headdim=P,
                                   d_state=N, init=init, want_final=True)
    np.testing.assert_allclose(y, ref, rtol=0, atol=1e-13)
    np.testing.assert_allclose(fin, rfin, rtol=0, atol=1e-13)


def test_untied_streams_read_only_their_own_parameters():
    """Changing every reverse-stream input leaves the forward half of the
    concatenation (and the forward final state) bit-identical, and the other
    way round."""
    rng = np.random.default_rng(8)
    L, H, P, N = 25, 2, 3, 4
    f = _rand(rng, 1, L, H, P, N)
    r1 = _rand(rng, 1, L, H, P, N)
    r2 = _rand(rng, 1, L, H, P, N)
    ch = H * P + 2 * N
    wf, w1, w2 = (rng.normal(0, 0.5, (ch, 4)) for _ in range(3))

    def run(fp, rp, wr):
        xf, Bf, Cf, dtf, Af, Df = fp
        xr, Br, Cr, dtr, Ar, Dr = rp
        return oracle.bimamba_untied(_xbc(xf, Bf, Cf), _xbc(xr, Br, Cr), dtf, dtr, Af, Ar, Df, Dr,
                                     wf, wr, heads=H, headdim=P, d_state=N, concat=True,
                                     want_final=True)
    y1, fin1 = run(f, r1, w1)
    y2, fin2 = run(f, r2, w2)
    np.testing.assert_array_equal(y1[..., :H * P], y2[..., :H * P])
    np.testing.assert_array_equal(fin1, fin2)
    assert np.max(np.abs(y1[..., H * P:] - y2[..., H * P:])) > 1e-3
    y3, _ = run(r1, r1, w1)
    np.testing.assert_array_equal(y3[..., H * P:], y1[..., H * P:])


# ------------------------------------------------------- backward (adjoint)
def _loss(x, B, C, dt, A, D, dy, init, reverse):
    y = oracle.scan(x, B, C, dt, A, D, init=init, reverse=reverse)
    return float(np.sum(y * dy))


def _fd_grad(f, arr, eps=1e-6):
    """Central finite differences of the scalar f() w.r.t. every element of
    arr (perturbed in place)."""
    out = np.zeros_like(arr)
    it = np.nditer(arr, flags=["multi_index"])
    for _ in it:
        i = it.multi_index
        v = arr[i]
        arr[i] = v + eps
        hi = f()
        arr[i] = v - eps
        lo = f()
        arr[i] = v
        out[i] = (hi - lo) / (2 * eps)
    return out


@pytest.mark.parametrize("reverse", [False, True])
@pytest.mark.parametrize("memory", ["short", "long"])
def test_scan_backward_matches_finite_differences(reverse, memory):
    """The adjoint recurrence against central differences of the forward
    recurrence, for every element of every input (x, B, C, dt, A, D and the
    initial state), one direction at a time, with two heads sharing a group."""
    rng = np.random.default_rng(11 + reverse)
    L, H, P, N, G = 6, 2, 2, 3, 1
    a = (1.0, 4.0) if memory == "short" else (1e-3, 1e-2)
    x, B, C, dt, A, D = _rand(rng, 1, L, H, P, N, G, *a)
    dy = rng.normal(size=x.shape)
    init = rng.normal(0, 0.5, (1, H, P, N)) if not reverse else None
    g = oracle.scan_backward(x, B, C, dt, A, D, dy, init=init, reverse=reverse)
    inputs = {"x": x, "B": B, "C": C, "dt": dt, "A": A, "D": D}
    if init is not None:
        inputs["init"] = init
    for name, arr in inputs.items():
        fd = _fd_grad(lambda: _loss(x, B, C, dt, A, D, dy, init, reverse), arr)
        scale = max(1.0, np.max(np.abs(fd)))
        assert np.max(np.abs(g[name] - fd)) <= 1e-6 * scale, name


def test_bidirectional_backward_matches_finite_differences():
    """Both directions' adjoints summed, against central differences of
    y = forward(init) + reverse(0)."""
    rng = np.random.default_rng(21)
    L, H, P, N, G = 5, 2, 2, 2, 1
    x, B, C, dt, A, D = _rand(rng, 2, L, H, P, N, G, 1.0, 8.0)
    dy = rng.normal(size=x.shape)
    init = rng.normal(0, 0.5, (2, H, P, N))

    def loss():
        yf = oracle.scan(x, B, C, dt, A, D, init=init)
        yr = oracle.scan(x, B, C, dt, A, D, reverse=True)
        return float(np.sum((yf + yr) * dy))
    g = oracle.bimamba_backward(x, B, C, dt, A, D, dy, init=init)
    for name, arr in {"x": x, "B": B, "C": C, "dt": dt, "A": A, "D": D, "init": init}.items():
        fd = _fd_grad(loss, arr)
        scale = max(1.0, np.max(np.abs(fd)))
        assert np.max(np.abs(g[name] - fd)) <= 1e-6 * scale, name
    # D enters each direction once per token: dL/dD_h = 2 sum_t dy_t . x_t
    np.testing.assert_allclose(g["D"], 2 * np.einsum("blhp,blhp->h", dy, x), rtol=1e-12)


@pytest.mark.parametrize("reverse", [False, True])
def test_conv_backward_matches_finite_differences(reverse):
    rng = np.random.default_rng(31 + reverse)
    u = rng.normal(size=(2, 7, 5))
    w = rng.normal(0, 0.5, (5, 4))
    bias = rng.normal(0, 0.3, 5)
    dout = rng.normal(size=u.shape)
    du, dw, db = oracle.conv_backward(u, w, bias, dout, reverse=reverse)

    def loss():
        return float(np.sum(oracle.conv(u, w, bias, reverse=reverse) * dout))
    for got, arr in ((du, u), (dw, w), (db, bias)):
        fd = _fd_grad(loss, arr)
        assert np.max(np.abs(got - fd)) <= 1e-7 * max(1.0, np.max(np.abs(fd)))


def test_mixer_backward_matches_finite_differences():
    """The whole bidirectional mixer core (conv+SiLU per direction, both
    scans, summed): every element of the raw xBC, dt, A, D, conv taps, conv
    bias and initial state against central differences of the forward
    oracle."""
    rng = np.random.default_rng(41)
    bsz, L, H, P, N = 1, 6, 2, 2, 2
    ch = H * P + 2 * N
    xbc = rng.normal(size=(bsz, L, ch))
    dt = np.log1p(np.exp(rng.normal(-1.0, 0.5, (bsz, L, H))))
    A = -np.exp(rng.uniform(0.0, np.log(8.0), H))
    D = rng.normal(size=H)
    w = rng.normal(0, 0.5, (ch, 4))
    bias = rng.normal(0, 0.3, ch)
    init = rng.normal(0, 0.5, (bsz, H, P, N))
    dy = rng.normal(size=(bsz, L, H * P))
    kw = dict(heads=H, headdim=P, d_state=N)
    g = oracle.bimamba_mixer_backward(xbc, dt, A, D, w, bias, dy, init=init, **kw)

    def loss():
        return float(np.sum(oracle.bimamba(xbc, dt, A, D, w, bias, init=init, **kw) * dy))
    for name, arr in {"xbc": xbc, "dt": dt, "A": A, "D": D, "conv_w": w, "conv_b": bias,
                      "init": init}.items():
        fd = _fd_grad(loss, arr)
        assert np.max(np.abs(g[name] - fd)) <= 1e-6 * max(1.0, np.max(np.abs(fd))), name
