"""Pins of the oracle's xHC steps (xHC summary page: "stream routing", "dense
read", "sparse residual update", "temporal feature augmentation"; project page
"default xHC configuration").  The router / update parameter shapes are this
project's reading (parity unpinned beyond these internal-consistency checks)."""
from __future__ import annotations

import itertools
import math

import numpy as np

import oracle


def _route_case(T=6, N=8, C=6, m=2, seed=40, alpha=2.0):
    rng = np.random.default_rng(seed)
    R = 2 * N - m
    X = rng.normal(size=(T, N, C))
    phi = rng.normal(size=(N * C, R)) / math.sqrt(N * C)
    b = rng.normal(size=R) * 0.3
    return X, phi, np.array([alpha, alpha]), b


def test_route_topk_matches_subset_brute_force():
    """Fixed streams 0..m-1 are always active with weight 1; the k-m routed streams
    are the subset of m..N-1 with the largest scores (checked over every subset)."""
    N, k, m = 8, 4, 2
    X, phi, a, b = _route_case(T=20, N=N, m=m)
    out = oracle.xhc_route(X, phi, a, b, k, m)
    for t in range(X.shape[0]):
        sc = out["score"][t]
        best = max(itertools.combinations(range(N - m), k - m), key=lambda s: sum(sc[q] for q in s))
        expect = list(range(m)) + sorted(m + q for q in best)
        assert out["idx"][t].tolist() == expect
        np.testing.assert_array_equal(out["w"][t][:m], 1.0)
        np.testing.assert_allclose(out["w"][t][m:], [sc[q - m] for q in expect[m:]], rtol=0, atol=0)


def test_route_topk_ties_go_to_lower_index():
    N, k, m, C = 6, 3, 1, 4
    X = np.ones((1, N, C))
    phi = np.zeros((N * C, 2 * N - m))
    b = np.zeros(2 * N - m)
    out = oracle.xhc_route(X, phi, np.zeros(2), b, k, m)
    assert out["idx"][0].tolist() == [0, 1, 2]


def test_route_scores_and_dense_read():
    """H_pre = sigma of the first N logits; x_in = sum over ALL N streams (dense read);
    with alpha = 0 and one-hot b_pre the read is a single stream."""
    N, k, m, C = 8, 4, 2, 6
    X, phi, a, b = _route_case(N=N, C=C)
    out = oracle.xhc_route(X, phi, a, b, k, m)
    np.testing.assert_allclose(out["x_in"], np.einsum("ti,tic->tc", out["H_pre"], X), atol=1e-13)
    b2 = b.copy(); b2[:N] = -40.0; b2[5] = 40.0
    out2 = oracle.xhc_route(X, phi, np.zeros(2), b2, k, m)
    np.testing.assert_allclose(out2["x_in"], X[:, 5], atol=1e-14)
    np.testing.assert_allclose(out2["score"], 1 / (1 + np.exp(-b2[N:])).reshape(1, -1).repeat(X.shape[0], 0),
                               atol=1e-15)


def test_conv_matches_numpy_convolve():
    """Causal depthwise conv: per channel, numpy.convolve truncated to the first T
    outputs; sequences restart the window."""
    rng = np.random.default_rng(41)
    T, C = 30, 5
    F = rng.normal(size=(T, C))
    ws = [rng.normal(size=(kk, C)) for kk in (4, 8, 12)]
    G = oracle.xhc_conv(F, ws)
    for j, w in enumerate(ws):
        for c in range(C):
            np.testing.assert_allclose(G[:, j, c], np.convolve(F[:, c], w[:, c])[:T], atol=1e-13)
    G2 = oracle.xhc_conv(F, ws, seq_len=10)
    for s0 in (0, 10, 20):
        Gs = oracle.xhc_conv(F[s0:s0 + 10], ws)
        np.testing.assert_allclose(G2[s0:s0 + 10], Gs, atol=0)


def test_mgs_orthogonal_span_and_classical_agree():
    rng = np.random.default_rng(42)
    T, C = 5, 64
    F = rng.normal(size=(T, C))
    G = rng.normal(size=(T, 3, C)) + 0.5 * F[:, None, :]
    V = oracle.xhc_gs(F, G)
    Vc = oracle.xhc_gs(F, G, classical=True)
    np.testing.assert_allclose(V, Vc, rtol=1e-10, atol=1e-12)
    np.testing.assert_array_equal(V[:, 0], F)
    for t in range(T):
        for i in range(4):
            for j in range(i):
                cos = V[t, i] @ V[t, j] / (np.linalg.norm(V[t, i]) * np.linalg.norm(V[t, j]))
                assert abs(cos) <= 1e-12
        A = np.stack([F[t], *G[t]], 1)
        # v_{j+1} = g_j - (combination of earlier v's): triangular change of basis
        coef, *_ = np.linalg.lstsq(V[t].T, A, rcond=None)
        np.testing.assert_allclose(V[t].T @ coef, A, atol=1e-12)
        np.testing.assert_allclose(np.tril(coef, -1), 0, atol=1e-12)
        np.testing.assert_allclose(np.diag(coef), 1, atol=1e-12)


def test_mgs_zero_component_contributes_nothing():
    T, C = 2, 8
    F = np.zeros((T, C))
    G = np.random.default_rng(43).normal(size=(T, 3, C))
    V = oracle.xhc_gs(F, G)
    assert (V[:, 0] == 0).all()
    np.testing.assert_allclose(V[:, 1], G[:, 0], atol=0)


def _upd_case(T=4, N=8, k=4, C=6, Kr=4, seed=44):
    rng = np.random.default_rng(seed)
    X = rng.normal(size=(T, N, C))
    V = rng.normal(size=(T, Kr, C))
    idx = np.stack([np.sort(np.concatenate([[0, 1], rng.choice(np.arange(2, N), k - 2, replace=False)]))
                    for _ in range(T)]).astype(np.int32)
    w = np.concatenate([np.ones((T, 2)), rng.uniform(0.2, 0.9, (T, k - 2))], 1)
    Pa = k * k + k * Kr
    phi = rng.normal(size=(k * C, Pa)) / math.sqrt(k * C)
    b = rng.normal(size=Pa) * 0.3
    b[:k * k] += (2 * np.eye(k)).reshape(-1)
    return X, V, idx, w, phi, np.array([1.5, 0.8]), b


def test_sparse_update_inactive_streams_untouched():
    X, V, idx, w, phi, a, b = _upd_case()
    Xn, Hr, Ho = oracle.xhc_sparse_update(X, V, idx, w, phi, a, b)
    for t in range(X.shape[0]):
        inactive = sorted(set(range(X.shape[1])) - set(idx[t].tolist()))
        np.testing.assert_array_equal(Xn[t, inactive], X[t, inactive])
        np.testing.assert_allclose(Hr[t].sum(1), 1, atol=1e-14)     # Sinkhorn on the active mix
        assert (Ho[t] > 0).all() and (Ho[t] < 2).all()               # 2 sigma


def test_sparse_update_permutation_and_writeback():
    """alpha = 0, H_res = P_sigma (bias +-40), H_post one-hot on component c0 (2 sigma(40) = 2):
    X_new[idx[j]] = X[idx[sigma(j)]] + 2 w_j V[c0]."""
    T, N, k, C, Kr = 3, 8, 4, 5, 4
    X, V, idx, w, phi, _, _ = _upd_case(T, N, k, C, Kr, seed=45)
    sig = [2, 0, 3, 1]
    res = np.full((k, k), -40.0)
    for j in range(k):
        res[j, sig[j]] = 40.0
    post = np.full((k, Kr), -40.0)
    post[:, 1] = 40.0
    b = np.concatenate([res.reshape(-1), post.reshape(-1)])
    Xn, Hr, Ho = oracle.xhc_sparse_update(X, V, idx, w, phi, np.zeros(2), b)
    for t in range(T):
        for j in range(k):
            exp = X[t, idx[t, sig[j]]] + 2.0 * w[t, j] * V[t, 1]
            np.testing.assert_allclose(Xn[t, idx[t, j]], exp, atol=1e-13)


def test_sparse_update_k_equals_n_matches_dense_mix():
    """With every stream active (k = N, idx = 0..N-1, w = 1) and one write-back
    component the update is the dense Eq.(3) post step with H_post = 2 sigma."""
    T, N, C = 3, 4, 6
    rng = np.random.default_rng(46)
    X = rng.normal(size=(T, N, C))
    F = rng.normal(size=(T, C))
    idx = np.tile(np.arange(N, dtype=np.int32), (T, 1))
    w = np.ones((T, N))
    Pa = N * N + N
    phi = rng.normal(size=(N * C, Pa)) / math.sqrt(N * C)
    b = rng.normal(size=Pa) * 0.3
    Xn, Hr, Ho = oracle.xhc_sparse_update(X, F[:, None, :], idx, w, phi, np.array([0.9, 0.6]), b)
    ref = oracle.mhc_post(X, F, Ho[:, :, 0], Hr)
    np.testing.assert_allclose(Xn, ref, atol=1e-13)
