"""Pins of the fp64 oracle's HC variant and Amax Gain diagnostic.

"mHC page" is "mHC: Manifold-Constrained Hyper-Connections" (paper notes):
section 3 Eq.(5) gives the HC coefficients (RMSNorm on the last dimension,
tanh of linear projections, gate factors alpha, static biases b); section 3
Eq.(4) the composite residual map across layers; section 3.1 the Amax Gain
Magnitude (largest absolute row / column sum of that map).  The cases are
chosen so that a dropped term (tanh, alpha, b, the norm), a wrong index (the
stream against the H_res row), a global instead of a per-stream norm, or a
reversed product order each fails at least one of them.
"""
from __future__ import annotations

import math
import os

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand_hc(T, n, C, seed=0, alpha=0.7):
    rng = np.random.default_rng(seed)
    X = rng.normal(size=(T, n, C)) * rng.uniform(0.5, 2.0, size=(T, n, 1))
    theta = rng.normal(size=(n + 2, C)) / math.sqrt(C)
    b = rng.normal(size=n * n + 2 * n) * 0.3
    b[2 * n:] += np.eye(n).reshape(-1)
    a = np.array([alpha, alpha * 1.3, alpha * 0.6])
    return X, theta, a, b


@pytest.mark.parametrize("n", [1, 3, 4])
def test_hc_zero_gates_leave_the_static_map(n):
    """Eq.(5) with alpha = 0: every map equals its bias, for any input.  The bias
    of H_res is row-major (entry [a][b] at 2n + a*n + b)."""
    X, theta, _, b = _rand_hc(5, n, 16, seed=n)
    co = oracle.hc_coeffs(X, theta, np.zeros(3), b)
    np.testing.assert_array_equal(co["H_pre"], np.broadcast_to(b[:n], (5, n)))
    np.testing.assert_array_equal(co["H_post"], np.broadcast_to(b[n:2 * n], (5, n)))
    np.testing.assert_array_equal(co["H_res"], np.broadcast_to(b[2 * n:].reshape(n, n), (5, n, n)))


def test_hc_closed_form_on_constant_streams():
    """Stream s of X is the constant v_s and projection row q the constant w_q.
    With eps = 0 the per-stream RMSNorm gives x~_s = sign(v_s) (all entries), so
    theta_q . x~_s = C w_q sign(v_s).  Taking w_q = atanh(k_q) / C makes the tanh
    exactly +-k_q: H_pre[s] = a_pre k_0 sign(v_s) + b_pre[s],
    H_post[s] = a_post k_1 sign(v_s) + b_post[s],
    H_res[a][s] = a_res k_(2+a) sign(v_s) + b_res[a][s].  The streams have
    different magnitudes (a global norm would not give +-1) and the res rows
    different k (a transposed H_res would not match)."""
    n, C = 3, 8
    v = np.array([0.5, -2.0, 3.0])
    X = np.broadcast_to(v[None, :, None], (1, n, C)).copy()
    k = np.array([0.2, -0.4, 0.1, 0.6, -0.3])
    theta = np.broadcast_to((np.arctanh(k) / C)[:, None], (n + 2, C)).copy()
    alpha = np.array([0.5, 0.25, 2.0])
    b = np.arange(n * n + 2 * n, dtype=np.float64) * 0.01
    co = oracle.hc_coeffs(X, theta, alpha, b, eps=0.0)
    sg = np.sign(v)
    np.testing.assert_allclose(co["H_pre"][0], alpha[0] * k[0] * sg + b[:n], rtol=0, atol=1e-15)
    np.testing.assert_allclose(co["H_post"][0], alpha[1] * k[1] * sg + b[n:2 * n], rtol=0, atol=1e-15)
    want = alpha[2] * k[2:, None] * sg[None, :] + b[2 * n:].reshape(n, n)
    np.testing.assert_allclose(co["H_res"][0], want, rtol=0, atol=1e-15)


def test_hc_per_stream_norm_invariance_and_odd_symmetry():
    """RMSNorm acts on each stream alone (the last dimension): with eps = 0,
    scaling one stream by k > 0 changes nothing; k < 0 flips the sign of that
    stream's tanh terms (tanh is odd), i.e. H - b changes sign in the entries
    of that stream (H_pre[s], H_post[s], column s of H_res) and no others."""
    X, theta, a, b = _rand_hc(4, 4, 32, seed=7)
    base = oracle.hc_coeffs(X, theta, a, b, eps=0.0)
    Xs = X.copy()
    Xs[:, 2] *= 7.5
    Xs[:, 0] *= 0.01
    sc = oracle.hc_coeffs(Xs, theta, a, b, eps=0.0)
    for key in ("H_pre", "H_post", "H_res"):
        np.testing.assert_allclose(sc[key], base[key], rtol=0, atol=1e-13)
    Xf = X.copy()
    Xf[:, 1] *= -3.0
    fl = oracle.hc_coeffs(Xf, theta, a, b, eps=0.0)
    n = 4
    sgn = np.ones(n)
    sgn[1] = -1.0
    np.testing.assert_allclose(fl["H_pre"] - b[:n], (base["H_pre"] - b[:n]) * sgn, atol=1e-13)
    np.testing.assert_allclose(fl["H_post"] - b[n:2 * n], (base["H_post"] - b[n:2 * n]) * sgn, atol=1e-13)
    br = b[2 * n:].reshape(n, n)
    np.testing.assert_allclose(fl["H_res"] - br, (base["H_res"] - br) * sgn[None, None, :], atol=1e-13)


def test_hc_stream_permutation_moves_the_stream_index_only():
    """Permuting the streams of X (with zero biases) permutes H_pre and H_post and
    the COLUMNS of H_res (the source stream); the rows of H_res belong to the
    projection rows theta_res[a] and stay."""
    X, theta, a, _ = _rand_hc(3, 4, 24, seed=3)
    b = np.zeros(24)
    perm = np.array([2, 0, 3, 1])
    base = oracle.hc_coeffs(X, theta, a, b)
    pm = oracle.hc_coeffs(X[:, perm], theta, a, b)
    np.testing.assert_allclose(pm["H_pre"], base["H_pre"][:, perm], rtol=0, atol=1e-14)
    np.testing.assert_allclose(pm["H_post"], base["H_post"][:, perm], rtol=0, atol=1e-14)
    np.testing.assert_allclose(pm["H_res"], base["H_res"][:, :, perm], rtol=0, atol=1e-14)


def test_hc_eps_enters_inside_the_root():
    """r_s = sqrt(mean(x_s^2) + eps): with a stream of all ones and a single
    nonzero projection entry, theta . x~ = w / sqrt(1 + eps) exactly."""
    C = 4
    X = np.ones((1, 1, C))
    theta = np.zeros((3, C))
    theta[0, 0] = 0.9
    eps = 0.25
    co = oracle.hc_coeffs(X, theta, np.array([1.0, 1.0, 1.0]), np.zeros(3), eps=eps)
    assert co["H_pre"][0, 0] == pytest.approx(math.tanh(0.9 / math.sqrt(1.25)), abs=1e-15)
    assert co["H_post"][0, 0] == 0.0 and co["H_res"][0, 0, 0] == 0.0


def _golden_amax():
    rows = []
    with open(os.path.join(GOLDEN, "amax_gain_hand.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            name, n, L, H, fw, bw = [x.strip() for x in line.split("|")]
            n, L = int(n), int(L)
            H = np.array([float(x) for x in H.split()]).reshape(L, 1, n, n)
            rows.append((name, H, [float(x) for x in fw.split()], [float(x) for x in bw.split()]))
    return rows


@pytest.mark.parametrize("case", _golden_amax(), ids=lambda c: c[0])
def test_amax_gain_hand_worked(case):
    """Values worked by hand (tests/golden/amax_gain_hand.txt): the product order
    of Eq.(4) and the absolute row / column sums of section 3.1."""
    _, H, fw, bw = case
    g = oracle.amax_gain(H)
    np.testing.assert_array_equal(g[:, 0, 0], fw)
    np.testing.assert_array_equal(g[:, 0, 1], bw)


def test_amax_gain_of_row_stochastic_layers_is_one():
    """Section 4.1 (compositional closure): products of matrices whose rows sum to
    1 have rows summing to 1, so the forward gain of a stack of Sinkhorn outputs
    (the last step normalises rows) is 1 at every depth; its backward gain stays
    within the column residual of the iterations."""
    rng = np.random.default_rng(11)
    L, T, n = 12, 6, 4
    H = np.stack([[oracle.sinkhorn(rng.normal(size=(n, n)) * 1.5, 20) for _ in range(T)] for _ in range(L)])
    g = oracle.amax_gain(H)
    np.testing.assert_allclose(g[..., 0], 1.0, rtol=0, atol=1e-12)
    np.testing.assert_allclose(g[..., 1], 1.0, rtol=0, atol=1e-3)


def test_amax_gain_constant_layer_is_a_matrix_power():
    """The same map at every layer: M_d = H^d (numpy.linalg.matrix_power)."""
    rng = np.random.default_rng(5)
    n, L = 5, 7
    H1 = np.eye(n) + rng.normal(size=(n, n)) * 0.3
    H = np.broadcast_to(H1, (L, 1, n, n)).copy()
    g = oracle.amax_gain(H)
    for d in range(1, L + 1):
        M = np.linalg.matrix_power(H1, d)
        assert g[d - 1, 0, 0] == pytest.approx(np.abs(M.sum(1)).max(), rel=1e-12)
        assert g[d - 1, 0, 1] == pytest.approx(np.abs(M.sum(0)).max(), rel=1e-12)


def test_amax_gain_scalar_stream_and_sign():
    """n = 1: the composite map is the product of the scalars and both gains are
    its absolute value; H = -1 at every layer keeps the gain at 1 (the absolute
    value of the sum, not the signed sum)."""
    h = np.array([1.5, -2.0, 0.5, -1.0])
    g = oracle.amax_gain(h.reshape(4, 1, 1, 1))
    np.testing.assert_allclose(g[:, 0, 0], np.abs(np.cumprod(h)), rtol=1e-15)
    np.testing.assert_array_equal(g[:, 0, 0], g[:, 0, 1])
    g2 = oracle.amax_gain(-np.ones((5, 1, 1, 1)))
    np.testing.assert_array_equal(g2[..., 0], 1.0)
