"""Pins of the fp64 oracle against what the pages and the mathematics fix.

Each test names the passage it follows.  "mHC page" is "mHC:
Manifold-Constrained Hyper-Connections" (paper notes); "xHC page" is the xHC
summary ("xHC: Expanded Hyper-Connections").  Together these are chosen so
that a dropped term, a wrong sign or index, or a transposed operand anywhere
in the oracle fails at least one of them.
"""
from __future__ import annotations

import itertools
import math
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle
from tests import brute_mhc

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rng(seed=0):
    return np.random.default_rng(seed)


def _rand_mhc(T, n, C, seed=0, alpha=0.5, bres_diag=2.0):
    rng = _rng(seed)
    P = n * n + 2 * n
    X = rng.normal(size=(T, n, C))
    F = rng.normal(size=(T, C))
    phi = rng.normal(size=(n * C, P)) / math.sqrt(n * C)
    b = rng.normal(size=P) * 0.3
    b[2 * n:] += (bres_diag * np.eye(n)).reshape(-1)
    a = np.array([alpha, alpha * 1.3, alpha * 0.7])
    return X, F, phi, a, b


# ----------------------------------------------------------------- Sinkhorn
def _golden_sinkhorn():
    cases = []
    with open(os.path.join(GOLDEN, "sinkhorn_hand.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            name, n, t, m0, mt = [s.strip() for s in line.split("|")]
            n, t = int(n), int(t)
            M0 = np.array([float(v) for v in m0.split()]).reshape(n, n)
            Mt = np.array([float(Fraction(v)) for v in mt.split()]).reshape(n, n)
            cases.append((name, t, M0, Mt))
    return cases


@pytest.mark.parametrize("case", _golden_sinkhorn(), ids=lambda c: c[0])
def test_sinkhorn_hand_worked(case):
    """mHC page Eq.(9): column normalisation, then row normalisation, per iteration
    (hand-derived exact fractions in tests/golden/sinkhorn_hand.txt)."""
    _, t, M0, Mt = case
    H = oracle.sinkhorn(np.log(M0), t)
    np.testing.assert_allclose(H, Mt, rtol=0, atol=1e-15)


def test_sinkhorn_rows_exact_columns_converge_monotone():
    """mHC page Eq.(6),(9): the last step of each iteration is a row normalisation,
    so rows sum to 1 after every iteration; the L1 column-sum error never grows."""
    rng = _rng(1)
    for n in range(2, 9):
        L = rng.normal(0, 2, (n, n))
        _, tr = oracle.sinkhorn(L, 20, trace=True)
        prev = np.inf
        for t in range(1, 21):
            np.testing.assert_allclose(tr[t].sum(1), 1.0, atol=1e-14)
            assert (tr[t] >= 0).all()
            err = np.abs(tr[t].sum(0) - 1).sum()
            assert err <= prev * (1 + 1e-12) + 1e-15
            prev = err
        # t=1 with random logits is far from doubly stochastic: the column error is real
        assert np.abs(tr[1].sum(0) - 1).sum() > 1e-6


def test_sinkhorn_cross_ratios_preserved():
    """Diagonal scalings D1 M D2 keep every cross-ratio m_ij m_kl / (m_il m_kj)."""
    rng = _rng(2)
    n = 4
    L = rng.normal(0, 1.5, (n, n))
    _, tr = oracle.sinkhorn(L, 20, trace=True)
    for t in range(21):
        M = tr[t]
        for i, j, k, l in itertools.product(range(n), repeat=4):
            cr = M[i, j] * M[k, l] / (M[i, l] * M[k, j])
            cr0 = math.exp(L[i, j] + L[k, l] - L[i, l] - L[k, j])
            assert abs(cr / cr0 - 1) < 1e-12


def test_sinkhorn_rank1_logits_give_uniform_after_one_iteration():
    """exp(a_i + b_j) = u v^T: T_c gives u_i / sum(u) in every column, T_r gives J/n."""
    rng = _rng(3)
    for n in (2, 3, 5, 8):
        a, b = rng.normal(size=n), rng.normal(size=n)
        H = oracle.sinkhorn(a[:, None] + b[None, :], 1)
        np.testing.assert_allclose(H, np.full((n, n), 1.0 / n), atol=1e-15)


def test_sinkhorn_circulant_fixed_after_one_iteration():
    """A circulant positive matrix has equal row and column sums s: after the first
    T_c it is already doubly stochastic (exp(L)/s) and stays there."""
    n = 5
    c = np.array([0.3, -1.0, 2.0, 0.1, -0.4])
    L = np.array([[c[(j - i) % n] for j in range(n)] for i in range(n)])
    E = np.exp(L)
    for t in (1, 2, 20):
        np.testing.assert_allclose(oracle.sinkhorn(L, t), E / E[0].sum(), atol=1e-15)


def test_sinkhorn_2x2_limit_closed_form():
    """The doubly stochastic 2x2 limit with the same cross-ratio kappa is
    [[p, 1-p], [1-p, p]], p = sqrt(kappa) / (1 + sqrt(kappa))."""
    rng = _rng(4)
    for _ in range(5):
        L = rng.normal(0, 1, (2, 2))
        kap = math.exp(L[0, 0] + L[1, 1] - L[0, 1] - L[1, 0])
        p = math.sqrt(kap) / (1 + math.sqrt(kap))
        np.testing.assert_allclose(oracle.sinkhorn(L, 200), [[p, 1 - p], [1 - p, p]], atol=1e-12)


def test_sinkhorn_n1_is_identity():
    """mHC page section 4.1: with n = 1 the doubly stochastic condition is the scalar 1."""
    for v in (-30.0, 0.0, 3.7, 50.0):
        assert oracle.sinkhorn(np.array([[v]]), 20)[0, 0] == 1.0


def test_sinkhorn_column_shift_invariance():
    """Adding a constant to a column of the logits scales that column of exp(L);
    the first T_c removes it, so every iterate is unchanged."""
    rng = _rng(5)
    L = rng.normal(0, 1, (4, 4))
    shift = rng.normal(0, 5, 4)
    np.testing.assert_allclose(oracle.sinkhorn(L + shift[None, :], 20), oracle.sinkhorn(L, 20),
                               atol=1e-14)


# --------------------------------------------------------------- mHC forward
def test_mhc_constant_input_closed_form():
    """X = c * ones and phi = 1/(nC) everywhere: r = sqrt(c^2 + eps), every
    projected logit is c / r, so H_pre = sigma(a_pre c/r + b), H_post =
    2 sigma(a_post c/r + b), and H_res is Sinkhorn of a rank-1 matrix = J/n.
    Pins the nC normalisation, eps inside the square root, and the gates."""
    T, n, C, c, eps = 2, 3, 5, 1.7, 0.25
    P = n * n + 2 * n
    X = np.full((T, n, C), c)
    phi = np.full((n * C, P), 1.0 / (n * C))
    a = np.array([0.9, -1.3, 0.4])
    b = np.zeros(P)
    co = oracle.mhc_coeffs(X, phi, a, b, 20, eps)
    u = c / math.sqrt(c * c + eps)
    np.testing.assert_allclose(co["r"], math.sqrt(c * c + eps), rtol=1e-15)
    np.testing.assert_allclose(co["H_pre"], 1 / (1 + math.exp(-a[0] * u)), rtol=1e-14)
    np.testing.assert_allclose(co["H_post"], 2 / (1 + math.exp(-a[1] * u)), rtol=1e-14)
    np.testing.assert_allclose(co["H_res"], np.full((T, n, n), 1.0 / n), atol=1e-15)


@pytest.mark.parametrize("col", range(4 * 4 + 8))
def test_mhc_phi_column_order(col):
    """phi columns are [pre n | post n | res n*n], res row-major (mat: z[2n + i n + j]
    is H_res[i][j]).  Only column `col` of phi is non-zero: exactly one logit moves."""
    n, C = 4, 6
    P = n * n + 2 * n
    rng = _rng(6)
    X = np.abs(rng.normal(size=(1, n, C))) + 0.5
    phi = np.zeros((n * C, P))
    phi[:, col] = 1.0
    a = np.array([1.0, 1.0, 1.0])
    co = oracle.mhc_coeffs(X, phi, a, np.zeros(P), 20, 0.0)
    zc = X.sum() / math.sqrt((X ** 2).mean())
    ez = np.zeros(P); ez[col] = zc
    np.testing.assert_allclose(co["z"][0], ez, atol=1e-12)
    if col < n:
        exp_pre = np.full(n, 0.5); exp_pre[col] = 1 / (1 + math.exp(-zc))
        np.testing.assert_allclose(co["H_pre"][0], exp_pre, atol=1e-15)
    else:
        np.testing.assert_allclose(co["H_pre"][0], 0.5, atol=1e-15)
    if n <= col < 2 * n:
        exp_post = np.ones(n); exp_post[col - n] = 2 / (1 + math.exp(-zc))
        np.testing.assert_allclose(co["H_post"][0], exp_post, atol=1e-15)
    else:
        np.testing.assert_allclose(co["H_post"][0], 1.0, atol=1e-15)
    if col >= 2 * n:
        i, j = divmod(col - 2 * n, n)
        H = co["H_res"][0]
        off = [H[i2, j2] for i2 in range(n) for j2 in range(n) if (i2, j2) != (i, j)]
        assert H[i, j] > max(off)          # the raised entry is (i, j), not (j, i)
    else:
        np.testing.assert_allclose(co["H_res"][0], 1.0 / n, atol=1e-15)


def test_mhc_alpha_segments():
    """alpha_pre / alpha_post / alpha_res scale only their own segment (Eq.(7), (16))."""
    X, F, phi, a, b = _rand_mhc(3, 4, 8, seed=7)
    base = oracle.mhc_coeffs(X, phi, a, b)
    for s, key in enumerate(("H_pre", "H_post", "H_res")):
        a2 = a.copy(); a2[s] = 0.0
        co = oracle.mhc_coeffs(X, phi, a2, b)
        n = 4
        seg = [slice(0, n), slice(n, 2 * n), slice(2 * n, None)][s]
        np.testing.assert_allclose(co["z"][:, seg], np.broadcast_to(b[seg], co["z"][:, seg].shape),
                                   atol=1e-15)
        for other in ("H_pre", "H_post", "H_res"):
            if other != key:
                np.testing.assert_array_equal(co[other], base[other])


def test_mhc_permutation_reduction():
    """mHC page Eq.(3) with H_res a permutation: bias +-40 makes H_res = P_sigma
    (H_res[i][sigma(i)] = 1), so X_next[i] = X[sigma(i)] + H_post[i] F; a 3-cycle
    catches a transposed H_res.  One-hot H_pre picks x_in = X[2]."""
    T, n, C = 3, 4, 7
    X, F, phi, _, _ = _rand_mhc(T, n, C, seed=8)
    P = n * n + 2 * n
    sig = [1, 2, 0, 3]
    b = np.zeros(P)
    b[:n] = -40.0; b[2] = 40.0
    res = np.full((n, n), -40.0)
    for i in range(n):
        res[i, sig[i]] = 40.0
    b[2 * n:] = res.reshape(-1)
    co = oracle.mhc_forward(X, F, phi, np.zeros(3), b)
    np.testing.assert_allclose(co["H_res"], np.broadcast_to(np.eye(n)[sig], (T, n, n)), atol=1e-15)
    np.testing.assert_allclose(co["H_post"], 1.0, atol=0)
    np.testing.assert_allclose(co["x_in"], X[:, 2], atol=1e-14)
    np.testing.assert_allclose(co["X_next"], X[:, sig] + F[:, None, :], atol=1e-14)


def test_mhc_reduces_to_plain_residual():
    """mHC page Eq.(1) vs Eq.(3): H_res = I, H_pre = e_0, H_post = 1 turn stream 0
    into x + F(x) with x_in = x, and leave the other streams unchanged plus F."""
    T, n, C = 2, 4, 9
    X, F, phi, _, _ = _rand_mhc(T, n, C, seed=9)
    P = n * n + 2 * n
    b = np.zeros(P)
    b[:n] = -40.0; b[0] = 40.0
    b[2 * n:] = np.where(np.eye(n) > 0, 40.0, -40.0).reshape(-1)
    co = oracle.mhc_forward(X, F, phi, np.zeros(3), b)
    np.testing.assert_allclose(co["x_in"], X[:, 0], atol=1e-14)
    np.testing.assert_allclose(co["X_next"][:, 0], X[:, 0] + F, atol=1e-14)
    np.testing.assert_allclose(co["X_next"], X + F[:, None, :], atol=1e-14)


def test_mhc_n1_path():
    """n = 1: H_res = 1 exactly, X_next = X + H_post F, x_in = H_pre X (section 4.1)."""
    X, F, phi, a, b = _rand_mhc(4, 1, 16, seed=10)
    co = oracle.mhc_forward(X, F, phi, a, b)
    assert (co["H_res"] == 1.0).all()
    np.testing.assert_allclose(co["X_next"][:, 0], X[:, 0] + co["H_post"][:, :1] * F, atol=1e-14)
    np.testing.assert_allclose(co["x_in"], co["H_pre"][:, :1] * X[:, 0], atol=1e-15)


def test_mhc_stream_mean_preserved():
    """mHC page section 1/4.1: with doubly stochastic H_res the stream sum is kept:
    sum_i X_next[i] = sum_j colsum_j X[j] + (sum_i H_post[i]) F, and colsum -> 1."""
    X, F, phi, a, b = _rand_mhc(5, 4, 32, seed=11)
    co = oracle.mhc_forward(X, F, phi, a, b, t_iters=200)
    lhs = co["X_next"].sum(1)
    rhs = X.sum(1) + co["H_post"].sum(1)[:, None] * F
    np.testing.assert_allclose(lhs, rhs, atol=1e-12)
    co20 = oracle.mhc_forward(X, F, phi, a, b, t_iters=20)
    colres = np.abs(co20["H_res"].sum(1) - 1).max()
    lhs20 = co20["X_next"].sum(1)
    rhs20 = X.sum(1) + co20["H_post"].sum(1)[:, None] * F
    assert np.abs(lhs20 - rhs20).max() <= colres * np.abs(X).sum(1).max() + 1e-12


def test_mhc_closure_and_spectral_bound():
    """mHC page section 4.1: products of doubly stochastic matrices stay doubly
    stochastic (Amax gain = 1) and the spectral norm is at most 1."""
    X, F, phi, a, b = _rand_mhc(8, 4, 16, seed=12, alpha=3.0, bres_diag=0.5)
    H = oracle.mhc_coeffs(X, phi, a, b, t_iters=300)["H_res"]
    Pm = np.eye(4)
    for t in range(8):
        assert np.linalg.norm(H[t], 2) <= 1 + 1e-9
        Pm = H[t] @ Pm
    np.testing.assert_allclose(Pm.sum(0), 1, atol=1e-9)
    np.testing.assert_allclose(Pm.sum(1), 1, atol=1e-9)
    assert (Pm >= 0).all()
    assert abs(np.abs(Pm.sum(1)).max() - 1) < 1e-9 and abs(np.abs(Pm.sum(0)).max() - 1) < 1e-9


def test_mhc_scale_invariance_of_coefficients():
    """RMSNorm makes the coefficients invariant to X -> s X (eps = 0); x_in and
    the H_res X part scale by s."""
    X, F, phi, a, b = _rand_mhc(3, 4, 8, seed=13)
    c1 = oracle.mhc_forward(X, F, phi, a, b, eps=0.0)
    c2 = oracle.mhc_forward(3.0 * X, 3.0 * F, phi, a, b, eps=0.0)
    for key in ("H_pre", "H_post", "H_res"):
        np.testing.assert_allclose(c2[key], c1[key], rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(c2["x_in"], 3 * c1["x_in"], rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(c2["X_next"], 3 * c1["X_next"], rtol=1e-12, atol=1e-13)


def test_mhc_norm_after_matmul_equivalent():
    """mHC page section 4.3.1, Eq.(14)-(16): projecting the raw x and dividing
    by r = ||x|| / sqrt(nC) afterwards gives the Eq.(7) logits (eps = 0)."""
    X, F, phi, a, b = _rand_mhc(4, 4, 16, seed=14)
    co = oracle.mhc_coeffs(X, phi, a, b, eps=0.0)
    T, n, C = X.shape
    x = X.reshape(T, -1)
    d = x @ phi                                                 # Eq.(14)
    r = np.linalg.norm(x, axis=1) / math.sqrt(n * C)            # Eq.(15)
    aseg = np.concatenate([np.full(n, a[0]), np.full(n, a[1]), np.full(n * n, a[2])])
    z = d * aseg[None, :] / r[:, None] + b[None, :]             # Eq.(16)
    np.testing.assert_allclose(co["z"], z, atol=1e-12)


@pytest.mark.parametrize("n,C", [(2, 8), (3, 4), (4, 3)])
def test_mhc_brute_force_tiny(n, C):
    """An independent pure-Python float64 statement (tests/brute_mhc.py)."""
    X, F, phi, a, b = _rand_mhc(2, n, C, seed=15 + n)
    co = oracle.mhc_forward(X, F, phi, a, b)
    for t in range(2):
        x_in, hp, ho, hr, xn = brute_mhc.sublayer(X[t].tolist(), F[t].tolist(), phi.tolist(),
                                                  a.tolist(), b.tolist())
        np.testing.assert_allclose(co["x_in"][t], x_in, atol=1e-12)
        np.testing.assert_allclose(co["H_pre"][t], hp, atol=1e-13)
        np.testing.assert_allclose(co["H_post"][t], ho, atol=1e-13)
        np.testing.assert_allclose(co["H_res"][t], hr, atol=1e-13)
        np.testing.assert_allclose(co["X_next"][t], xn, atol=1e-12)


def test_oracle_reads_bf16_bits_exactly():
    """The oracle widens the stored bf16 bit patterns exactly."""
    bits = np.array([0x3F80, 0xBF40, 0x0001, 0x7F7F], dtype=np.uint16)
    vals = oracle.widen(bits)
    assert vals[0] == 1.0 and vals[1] == -0.75
    assert vals[2] == 2.0 ** -133 and vals[3] == (2 - 2 ** -7) * 2.0 ** 127
