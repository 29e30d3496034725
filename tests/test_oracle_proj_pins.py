"""Pins of the projection oracle (oracle.linear / in_proj / out_proj /
softplus) against what does not depend on it: hand-derived values
(tests/golden/proj_hand.txt), brute-force loops on tiny inputs, exact
identities, and softplus's closed forms.  A mistake such as a transposed
weight, swapped xBC/dt rows, a missing bias or a wrong softplus branch fails
one of these."""
import math
import os

import numpy as np

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "proj_hand.txt")


def _golden():
    vals = {}
    for line in open(GOLDEN):
        if line.startswith("#") or not line.strip():
            continue
        k, *v = line.split()
        vals[k] = np.array([float(x) for x in v])
    return vals


def test_hand_derived_projection_values():
    g = _golden()
    u = np.array([[1.0, 2.0], [-1.0, 0.5]])
    w_in = np.array([[1.0, 0.0], [0.0, 1.0], [1.0, 1.0], [2.0, -1.0]])
    xbc, dt = oracle.in_proj(u, w_in, np.array([-1.0]), heads=1, headdim=1, d_state=1)
    np.testing.assert_allclose(xbc.ravel(), g["in_xbc"], rtol=0, atol=1e-15)
    np.testing.assert_allclose(dt.ravel(), g["in_dt"], rtol=1e-14)
    out = oracle.out_proj(np.array([[1.0, -2.0, 0.5]]), np.array([[1.0, 1.0, 1.0], [0.0, 2.0, -4.0]]))
    np.testing.assert_allclose(out.ravel(), g["out"], rtol=0, atol=1e-15)


def test_linear_against_brute_force_loops():
    rng = np.random.default_rng(0)
    x = rng.standard_normal((3, 4, 5))
    w = rng.standard_normal((6, 5))
    b = rng.standard_normal(6)
    want = np.zeros((3, 4, 6))
    for i in range(3):
        for j in range(4):
            for o in range(6):
                acc = b[o]
                for k in range(5):
                    acc += x[i, j, k] * w[o, k]
                want[i, j, o] = acc
    np.testing.assert_allclose(oracle.linear(x, w, b), want, rtol=1e-13, atol=1e-13)


def test_identity_weights_copy_the_input():
    rng = np.random.default_rng(1)
    H, P, N = 2, 3, 2
    ch = H * P + 2 * N
    u = rng.standard_normal((5, ch))
    w_in = np.concatenate([np.eye(ch), np.zeros((H, ch))])
    bias = np.array([0.0, 2.0])
    xbc, dt = oracle.in_proj(u, w_in, bias, heads=H, headdim=P, d_state=N)
    np.testing.assert_array_equal(xbc, u)
    np.testing.assert_allclose(dt, np.broadcast_to([math.log(2.0), math.log1p(math.exp(2.0))], (5, 2)),
                               rtol=1e-15)


def test_softplus_closed_forms():
    assert oracle.softplus(0.0) == math.log(2.0)
    np.testing.assert_allclose(oracle.softplus(math.log(math.e - 1.0)), 1.0, rtol=1e-15)
    np.testing.assert_allclose(oracle.softplus(40.0), 40.0 + math.exp(-40.0), rtol=1e-15)
    np.testing.assert_allclose(oracle.softplus(-40.0), math.exp(-40.0), rtol=1e-12)
    np.testing.assert_allclose(oracle.softplus(1000.0), 1000.0, rtol=1e-15)   # no overflow
    x = np.linspace(-10, 10, 101)
    # softplus(x) - softplus(-x) = x
    np.testing.assert_allclose(oracle.softplus(x) - oracle.softplus(-x), x, atol=1e-14)


def test_out_projection_of_concatenated_streams_composes_two_linears():
    """The untied block maps each stream with its own Linear, concatenates
    and fuses with a Linear(2d -> d); composed, that is one Linear of the
    concatenation with W = [F_f W_f | F_r W_r]."""
    rng = np.random.default_rng(2)
    yf, yr = rng.standard_normal((4, 6)), rng.standard_normal((4, 6))
    wf, wr = rng.standard_normal((3, 6)), rng.standard_normal((3, 6))
    fuse = rng.standard_normal((3, 6))
    two_step = oracle.linear(np.concatenate([oracle.linear(yf, wf), oracle.linear(yr, wr)], -1), fuse)
    w = np.concatenate([fuse[:, :3] @ wf, fuse[:, 3:] @ wr], axis=1)
    np.testing.assert_allclose(oracle.out_proj(np.concatenate([yf, yr], -1), w), two_step, rtol=1e-12,
                               atol=1e-12)
