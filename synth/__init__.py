"""Seeded synthetic inputs for the mHC / xHC residual-stream mixing workloads.

This module is shared by the CUDA path's tests and benchmark and by the fp64
oracle's tests.  It only draws random numbers and rounds them to the storage
dtype; it holds none of the method's arithmetic.

Conventions
-----------
* One ``numpy.random.Generator(PCG64(seed))`` per workload; arrays are drawn in
  the fixed order documented on each function.
* ``N(mu, v)`` means mean ``mu`` and VARIANCE ``v`` (so the projection
  ``phi ~ N(0, 1/(nC))`` has standard deviation ``1/sqrt(nC)``); every draw is
  float32 and, for bf16 workloads, rounded to bfloat16 with round-to-nearest-even.
* bf16 arrays are returned as their raw ``uint16`` bit patterns; fp32 arrays as
  ``float32``.  Both sides widen the very same bits.
* Layouts: X ``[T][n][C]``, F_out ``[T][C]``, phi ``[n*C][n*n+2n]`` (columns
  ``pre | post | res``), b ``[n*n+2n]``, alpha ``[3]`` = (pre, post, res).
"""
from __future__ import annotations

import numpy as np

_CHUNK = 1 << 24  # draw long arrays in chunks; the stream is identical to one draw


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round float32 to bfloat16 (round-to-nearest-even); returns uint16 bits."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    u = a.view(np.uint32)
    bias = ((u >> 16) & np.uint32(1)) + np.uint32(0x7FFF)
    return ((u + bias) >> 16).astype(np.uint16)


def f32_to_tf32(a: np.ndarray) -> np.ndarray:
    """Round float32 to tf32 (10 explicit mantissa bits, round-to-nearest-even on the
    13 dropped bits); returns float32 values whose low 13 bits are zero."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    u = a.view(np.uint32)
    finite = (u & np.uint32(0x7F800000)) != np.uint32(0x7F800000)
    bias = ((u >> 13) & np.uint32(1)) + np.uint32(0xFFF)
    r = np.where(finite, (u + bias) & np.uint32(0xFFFFE000), u)
    return r.astype(np.uint32).view(np.float32)


def _normal(rng: np.random.Generator, shape, std: float, dtype: str) -> np.ndarray:
    """float32 N(0, std^2) draws, stored as fp32 or as bf16 bits."""
    count = int(np.prod(shape)) if len(shape) else 1
    out = np.empty(count, dtype=np.uint16 if dtype == "bf16" else np.float32)
    s = np.float32(std)
    for lo in range(0, count, _CHUNK):
        hi = min(count, lo + _CHUNK)
        v = rng.standard_normal(hi - lo, dtype=np.float32)
        if std != 1.0:
            v *= s
        out[lo:hi] = f32_to_bf16_bits(v) if dtype == "bf16" else v
    return out.reshape(shape)


def mhc_inputs(T: int, n: int, C: int, dtype: str = "bf16", seed: int = 1,
               alpha: float = 0.01, phi_dtype: str | None = None) -> dict:
    """Inputs of one mHC sublayer (the mHC paper's Eq. 3 and Eq. 7-9 workload).

    Draw order: X ~ N(0,1) [T][n][C]; F_out ~ N(0,1) [T][C];
    phi ~ N(0, 1/(nC)) [nC][P]; b_pre ~ N(0, 0.1) [n]; b_post ~ N(0, 0.1) [n];
    the noise of b_res = 2*I_n + N(0, 0.1) [n][n].  X, F_out and phi take the
    storage dtype (phi_dtype="tf32": phi is the same float32 draw rounded to tf32
    instead, stored as float32); alpha (all three = ``alpha``) and b are float32.
    """
    assert dtype in ("bf16", "f32") and phi_dtype in (None, "bf16", "f32", "tf32")
    P = n * n + 2 * n
    rng = np.random.Generator(np.random.PCG64(seed))
    X = _normal(rng, (T, n, C), 1.0, dtype)
    F = _normal(rng, (T, C), 1.0, dtype)
    pd = phi_dtype or dtype
    phi = _normal(rng, (n * C, P), float(1.0 / np.sqrt(n * C)), "f32" if pd == "tf32" else pd)
    if pd == "tf32":
        phi = f32_to_tf32(phi)
    sd = float(np.sqrt(0.1))
    b_pre = rng.standard_normal(n, dtype=np.float32) * np.float32(sd)
    b_post = rng.standard_normal(n, dtype=np.float32) * np.float32(sd)
    b_res = (rng.standard_normal((n, n), dtype=np.float32) * np.float32(sd)
             + np.float32(2.0) * np.eye(n, dtype=np.float32))
    b = np.concatenate([b_pre, b_post, b_res.reshape(-1)]).astype(np.float32)
    a = np.full(3, alpha, dtype=np.float32)
    return dict(X=X, F=F, phi=phi, alpha=a, b=b, T=T, n=n, C=C, dtype=dtype, phi_dtype=pd,
                t_iters=20, eps=1e-6, seed=seed)


def mhc_grad_inputs(T: int, n: int, C: int, dtype: str = "bf16", seed: int = 4) -> dict:
    """mhc_inputs(...) followed, on the same stream, by the upstream gradients
    dX_next ~ N(0,1) [T][n][C] and dx_in ~ N(0,1) [T][C]."""
    P = n * n + 2 * n
    rng = np.random.Generator(np.random.PCG64(seed))
    X = _normal(rng, (T, n, C), 1.0, dtype)
    F = _normal(rng, (T, C), 1.0, dtype)
    phi = _normal(rng, (n * C, P), float(1.0 / np.sqrt(n * C)), dtype)
    sd = float(np.sqrt(0.1))
    b_pre = rng.standard_normal(n, dtype=np.float32) * np.float32(sd)
    b_post = rng.standard_normal(n, dtype=np.float32) * np.float32(sd)
    b_res = (rng.standard_normal((n, n), dtype=np.float32) * np.float32(sd)
             + np.float32(2.0) * np.eye(n, dtype=np.float32))
    b = np.concatenate([b_pre, b_post, b_res.reshape(-1)]).astype(np.float32)
    dXn = _normal(rng, (T, n, C), 1.0, dtype)
    dxin = _normal(rng, (T, C), 1.0, dtype)
    return dict(X=X, F=F, phi=phi, alpha=np.full(3, 0.01, dtype=np.float32), b=b,
                dX_next=dXn, dx_in=dxin, T=T, n=n, C=C, dtype=dtype, t_iters=20,
                eps=1e-6, seed=seed)


def xhc_inputs(T: int, N: int = 16, k: int = 4, m: int = 2, C: int = 2048,
               kappa=(4, 8, 12), dtype: str = "bf16", seed: int = 3,
               alpha: float = 0.01) -> dict:
    """Inputs of one xHC sublayer (xHC summary: stream routing, dense read,
    sparse residual update, temporal augmentation).

    Draw order: X ~ N(0,1) [T][N][C]; F_out ~ N(0,1) [T][C];
    phi_read ~ N(0, 1/(NC)) [N*C][2N-m]; b_read ~ N(0, 0.1) [2N-m];
    one conv weight per kernel size, w_j ~ N(0, 1/kappa_j) [kappa_j][C] (fp32);
    phi_act ~ N(0, 1/(kC)) [k*C][k*k + k*Kr]; b_act: res part 2*I_k + N(0, 0.1),
    post part N(0, 0.1) [k*Kr].  alpha_read = (pre, route), alpha_act = (res, post),
    all ``alpha``.
    """
    assert dtype in ("bf16", "f32")
    r = len(kappa)
    Kr = r + 1
    R = 2 * N - m
    Pa = k * k + k * Kr
    rng = np.random.Generator(np.random.PCG64(seed))
    X = _normal(rng, (T, N, C), 1.0, dtype)
    F = _normal(rng, (T, C), 1.0, dtype)
    phi_read = _normal(rng, (N * C, R), float(1.0 / np.sqrt(N * C)), dtype)
    sd = np.float32(np.sqrt(0.1))
    b_read = rng.standard_normal(R, dtype=np.float32) * sd
    conv_w = [rng.standard_normal((kj, C), dtype=np.float32) * np.float32(1.0 / np.sqrt(kj))
              for kj in kappa]
    phi_act = _normal(rng, (k * C, Pa), float(1.0 / np.sqrt(k * C)), dtype)
    b_res = rng.standard_normal((k, k), dtype=np.float32) * sd + np.float32(2.0) * np.eye(k, dtype=np.float32)
    b_post = rng.standard_normal(k * Kr, dtype=np.float32) * sd
    b_act = np.concatenate([b_res.reshape(-1), b_post]).astype(np.float32)
    return dict(X=X, F=F, phi_read=phi_read, b_read=b_read.astype(np.float32),
                alpha_read=np.full(2, alpha, dtype=np.float32), conv_w=conv_w,
                kappa=tuple(int(x) for x in kappa), phi_act=phi_act, b_act=b_act,
                alpha_act=np.full(2, alpha, dtype=np.float32), T=T, N=N, k=k, m=m, C=C,
                Kr=Kr, dtype=dtype, t_iters=20, eps=1e-6, seed=seed)


def hc_inputs(T: int, n: int, C: int, dtype: str = "bf16", seed: int = 5,
              alpha: float = 0.01) -> dict:
    """Inputs of one HC sublayer (the tanh parameterisation, the mHC paper's Eq. 5,
    applied by Eq. 3).

    Draw order: X ~ N(0,1) [T][n][C]; F_out ~ N(0,1) [T][C];
    theta ~ N(0, 1/C) [n+2][C] (rows pre, post, res_0..res_{n-1});
    b_pre ~ N(0, 0.1) [n]; b_post ~ N(0, 0.1) [n]; the noise of b_res = I_n + N(0, 0.1)
    [n][n] (the static residual map starts near the identity).  X, F_out and theta
    take the storage dtype; alpha (all three = ``alpha``) and b are float32.
    """
    assert dtype in ("bf16", "f32")
    rng = np.random.Generator(np.random.PCG64(seed))
    X = _normal(rng, (T, n, C), 1.0, dtype)
    F = _normal(rng, (T, C), 1.0, dtype)
    theta = _normal(rng, (n + 2, C), float(1.0 / np.sqrt(C)), dtype)
    sd = np.float32(np.sqrt(0.1))
    b_pre = rng.standard_normal(n, dtype=np.float32) * sd
    b_post = rng.standard_normal(n, dtype=np.float32) * sd
    b_res = rng.standard_normal((n, n), dtype=np.float32) * sd + np.eye(n, dtype=np.float32)
    b = np.concatenate([b_pre, b_post, b_res.reshape(-1)]).astype(np.float32)
    return dict(X=X, F=F, theta=theta, alpha=np.full(3, alpha, dtype=np.float32), b=b,
                T=T, n=n, C=C, dtype=dtype, eps=1e-6, seed=seed)


def redraw_rows(X: np.ndarray, rows, seed: int, attempt: int, dtype: str) -> None:
    """Replace token rows ``rows`` of a state X [T][N][C] with fresh N(0,1)
    draws from the derived seed (seed, attempt, row) -- used to move routed
    tokens away from TopK score ties."""
    for t in rows:
        rng = np.random.Generator(np.random.PCG64([seed, 1000 + attempt, int(t)]))
        X[t] = _normal(rng, X.shape[1:], 1.0, dtype)


# Named workloads: the per-sublayer problem shapes used by the tests and the benchmark.
WORKLOADS = {
    "mhc_tiny": dict(T=64, n=4, C=256, dtype="f32", seed=0),
    "mhc_llm": dict(T=8192, n=4, C=4096, dtype="bf16", seed=1),
    "mhc_wide": dict(T=32768, n=4, C=7168, dtype="bf16", seed=2),
    "mhc_sweep_n2": dict(T=8192, n=2, C=4096, dtype="bf16", seed=2),
    "mhc_sweep_n8": dict(T=8192, n=8, C=4096, dtype="bf16", seed=2),
    "xhc": dict(T=8192, N=16, k=4, m=2, C=2048, dtype="bf16", seed=3),
    "mhc_bwd": dict(T=8192, n=4, C=4096, dtype="bf16", seed=4),
    "hc_llm": dict(T=8192, n=4, C=4096, dtype="bf16", seed=5),
}
