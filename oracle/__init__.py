"""fp64 CPU oracle for the mHC / xHC residual-stream mixing.

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, by ``__graft_entry__.smoke()``
and by the CPU-baseline leg of ``bench.py``.  The CUDA library and its Python
binding never import it, and it shares no code with them (only the seeded
input generators in ``synth`` serve both sides).

The arithmetic lives in ``oracle.c`` (plain C, double precision, OpenMP over
tokens); this module widens the stored bit patterns (bf16 as uint16, or fp32)
exactly to float64 and marshals numpy arrays through ctypes.  Every function
cites the passage of the pages it follows in ``oracle.c``.
"""
from __future__ import annotations

import ctypes as ct
import os

import numpy as np

from . import build as _build

_lib = None


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = ct.CDLL(path)
        D = ct.POINTER(ct.c_double)
        I32 = ct.POINTER(ct.c_int32)
        i64, i32, dbl = ct.c_int64, ct.c_int, ct.c_double
        L.orc_sinkhorn.argtypes = [D, i32, i32, D, D]
        L.orc_mhc_coeffs.argtypes = [D, D, D, D, i64, i32, i32, i32, dbl, D, D, D, D, D]
        L.orc_mhc_apply_pre.argtypes = [D, D, i64, i32, i32, D]
        L.orc_mhc_post.argtypes = [D, D, D, D, i64, i32, i32, D]
        L.orc_mhc_backward.argtypes = [D, D, D, D, D, D, D, i64, i32, i32, i32, dbl,
                                       D, D, D, D, D]
        L.orc_xhc_route.argtypes = [D, D, D, D, i64, i32, i32, i32, i32, dbl, D, D, D, I32, D]
        L.orc_xhc_conv.argtypes = [D, D, ct.POINTER(ct.c_int), i32, i64, i32, i64, D]
        L.orc_xhc_gs.argtypes = [D, D, i64, i32, i32, i32, D]
        L.orc_xhc_sparse_update.argtypes = [D, D, i32, I32, D, D, D, D, i64, i32, i32, i32,
                                            i32, dbl, D, D]
        L.orc_hc_coeffs.argtypes = [D, D, D, D, i64, i32, i32, dbl, D, D, D]
        L.orc_amax_gain.argtypes = [D, i32, i64, i32, D]
        for f in ("orc_sinkhorn", "orc_mhc_coeffs", "orc_mhc_apply_pre", "orc_mhc_post",
                  "orc_mhc_backward", "orc_xhc_route", "orc_xhc_conv", "orc_xhc_gs",
                  "orc_xhc_sparse_update", "orc_hc_coeffs", "orc_amax_gain"):
            getattr(L, f).restype = None
        _lib = L
    return _lib


def widen(a) -> np.ndarray:
    """Exact widening of stored values to float64: uint16 arrays are bf16 bit
    patterns; float arrays are taken as they are."""
    a = np.asarray(a)
    if a.dtype == np.uint16:
        return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return np.ascontiguousarray(a, dtype=np.float64)


def _p(a):
    if a is None:
        return None
    return a.ctypes.data_as(ct.POINTER(ct.c_double))


def _c(a):
    return np.ascontiguousarray(widen(a))


def threads(n: int | None) -> None:
    """Set the OpenMP thread count for subsequent calls (None: library default)."""
    if n is not None:
        os.environ["OMP_NUM_THREADS"] = str(n)


# ------------------------------------------------------------------- Sinkhorn
def sinkhorn(L, t_iters: int = 20, trace: bool = False):
    """Eq.(8)-(9) of the mHC paper: exp, then t_iters x (column-, row-normalise)."""
    L = _c(L)
    n = L.shape[-1]
    assert L.shape == (n, n)
    H = np.empty((n, n))
    tr = np.empty((t_iters + 1, n, n)) if trace else None
    lib().orc_sinkhorn(_p(L), n, t_iters, _p(H), _p(tr))
    return (H, tr) if trace else H


# ---------------------------------------------------------------------- mHC
def mhc_coeffs(X, phi, alpha, b, t_iters=20, eps=1e-6):
    """Eq.(7)-(9): returns dict z [T][P], r [T], H_pre [T][n], H_post [T][n], H_res [T][n][n]."""
    X, phi, alpha, b = _c(X), _c(phi), _c(alpha), _c(b)
    T, n, C = X.shape
    P = n * n + 2 * n
    assert phi.shape == (n * C, P) and b.shape == (P,) and alpha.shape == (3,)
    z = np.empty((T, P)); r = np.empty(T)
    Hp = np.empty((T, n)); Ho = np.empty((T, n)); Hr = np.empty((T, n, n))
    lib().orc_mhc_coeffs(_p(X), _p(phi), _p(alpha), _p(b), T, n, C, t_iters, eps,
                         _p(z), _p(r), _p(Hp), _p(Ho), _p(Hr))
    return dict(z=z, r=r, H_pre=Hp, H_post=Ho, H_res=Hr)


def mhc_apply_pre(X, H_pre):
    X, H_pre = _c(X), _c(H_pre)
    T, n, C = X.shape
    out = np.empty((T, C))
    lib().orc_mhc_apply_pre(_p(X), _p(H_pre), T, n, C, _p(out))
    return out


def mhc_pre(X, phi, alpha, b, t_iters=20, eps=1e-6):
    """The pre half: coefficients (Eq.7-9) and x_in = H_pre X (F_pre)."""
    co = mhc_coeffs(X, phi, alpha, b, t_iters, eps)
    co["x_in"] = mhc_apply_pre(X, co["H_pre"])
    return co


def mhc_post(X, F, H_post, H_res):
    """F_post,res: X_next = H_res X + H_post^T F (Eq.3)."""
    X, F, H_post, H_res = _c(X), _c(F), _c(H_post), _c(H_res)
    T, n, C = X.shape
    out = np.empty((T, n, C))
    lib().orc_mhc_post(_p(X), _p(F), _p(H_post), _p(H_res), T, n, C, _p(out))
    return out


def mhc_forward(X, F, phi, alpha, b, t_iters=20, eps=1e-6):
    co = mhc_pre(X, phi, alpha, b, t_iters, eps)
    co["X_next"] = mhc_post(X, F, co["H_post"], co["H_res"])
    return co


def mhc_backward(X, F, phi, alpha, b, dX_next, dx_in, t_iters=20, eps=1e-6):
    """Reverse mode through mhc_pre + mhc_post (all Sinkhorn iterations unrolled)."""
    X, F, phi, alpha, b = _c(X), _c(F), _c(phi), _c(alpha), _c(b)
    dXn, dxi = _c(dX_next), _c(dx_in)
    T, n, C = X.shape
    P = n * n + 2 * n
    dX = np.empty_like(X); dF = np.empty((T, C)); dphi = np.empty((n * C, P))
    da = np.empty(3); db = np.empty(P)
    lib().orc_mhc_backward(_p(X), _p(F), _p(phi), _p(alpha), _p(b), _p(dXn), _p(dxi),
                           T, n, C, t_iters, eps, _p(dX), _p(dF), _p(dphi), _p(da), _p(db))
    return dict(dX=dX, dF=dF, dphi=dphi, dalpha=da, db=db)


# ---------------------------------------------------------------------- xHC
def xhc_route(X, phi_read, alpha_read, b_read, k, m, eps=1e-6):
    X, phi_read, alpha_read, b_read = _c(X), _c(phi_read), _c(alpha_read), _c(b_read)
    T, N, C = X.shape
    R = 2 * N - m
    assert phi_read.shape == (N * C, R) and b_read.shape == (R,)
    x_in = np.empty((T, C)); Hp = np.empty((T, N)); sc = np.empty((T, N - m))
    idx = np.empty((T, k), dtype=np.int32); w = np.empty((T, k))
    lib().orc_xhc_route(_p(X), _p(phi_read), _p(alpha_read), _p(b_read), T, N, C, k, m, eps,
                        _p(x_in), _p(Hp), _p(sc), idx.ctypes.data_as(ct.POINTER(ct.c_int32)),
                        _p(w))
    return dict(x_in=x_in, H_pre=Hp, score=sc, idx=idx, w=w)


def xhc_conv(F, conv_w, seq_len=None):
    F = _c(F)
    T, C = F.shape
    kappa = [int(np.asarray(w).shape[0]) for w in conv_w]
    wcat = np.ascontiguousarray(np.concatenate([widen(w).reshape(-1) for w in conv_w]))
    r = len(kappa)
    G = np.empty((T, r, C))
    ka = (ct.c_int * r)(*kappa)
    lib().orc_xhc_conv(_p(F), _p(wcat), ka, r, T, C, int(seq_len or T), _p(G))
    return G


def xhc_gs(F, G, classical=False):
    F, G = _c(F), _c(G)
    T, r, C = G.shape
    V = np.empty((T, r + 1, C))
    lib().orc_xhc_gs(_p(F), _p(G), T, C, r, 1 if classical else 0, _p(V))
    return V


def xhc_conv_gs(F, conv_w, seq_len=None):
    return xhc_gs(F, xhc_conv(F, conv_w, seq_len))


def xhc_sparse_update(X, V, idx, w, phi_act, alpha_act, b_act, t_iters=20, eps=1e-6):
    """Returns (X_new, H_res [T][k][k], H_post [T][k][Kr]); X is not modified."""
    Xd = _c(X).copy()
    V, w, phi_act, alpha_act, b_act = _c(V), _c(w), _c(phi_act), _c(alpha_act), _c(b_act)
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    T, N, C = Xd.shape
    k = idx.shape[1]
    Kr = V.shape[1]
    assert phi_act.shape == (k * C, k * k + k * Kr)
    Hr = np.empty((T, k, k)); Ho = np.empty((T, k, Kr))
    lib().orc_xhc_sparse_update(_p(Xd), _p(V), Kr, idx.ctypes.data_as(ct.POINTER(ct.c_int32)),
                                _p(w), _p(phi_act), _p(alpha_act), _p(b_act), T, N, C, k,
                                t_iters, eps, _p(Hr), _p(Ho))
    return Xd, Hr, Ho


# ----------------------------------------------------------------- HC (tanh)
def hc_coeffs(X, theta, alpha, b, eps=1e-6):
    """Eq.(5) of the mHC paper (the HC parameterisation): per-stream RMSNorm,
    tanh of the projections, gate factor, static bias.  theta [n+2][C] (rows pre,
    post, res_0..res_{n-1}); b [n*n+2n].  Returns dict H_pre [T][n], H_post [T][n],
    H_res [T][n][n]."""
    X, theta, alpha, b = _c(X), _c(theta), _c(alpha), _c(b)
    T, n, C = X.shape
    assert theta.shape == (n + 2, C) and b.shape == (n * n + 2 * n,) and alpha.shape == (3,)
    Hp = np.empty((T, n)); Ho = np.empty((T, n)); Hr = np.empty((T, n, n))
    lib().orc_hc_coeffs(_p(X), _p(theta), _p(alpha), _p(b), T, n, C, eps, _p(Hp), _p(Ho), _p(Hr))
    return dict(H_pre=Hp, H_post=Ho, H_res=Hr)


def hc_pre(X, theta, alpha, b, eps=1e-6):
    """HC coefficients (Eq.5) and x_in = H_pre X (the F_pre input of Eq.3)."""
    co = hc_coeffs(X, theta, alpha, b, eps)
    co["x_in"] = mhc_apply_pre(X, co["H_pre"])
    return co


def amax_gain(H_res):
    """Amax Gain Magnitude (mHC paper section 3.1) of the composite maps
    M_d = H_res[d-1] ... H_res[0], d = 1..L, per token: H_res [L][T][n][n] ->
    gain [L][T][2] = (max_i |row sum i|, max_j |column sum j|)."""
    H = _c(H_res)
    Lz, T, n, n2 = H.shape
    assert n == n2 and n <= 8
    g = np.empty((Lz, T, 2))
    lib().orc_amax_gain(_p(H), Lz, T, n, _p(g))
    return g
