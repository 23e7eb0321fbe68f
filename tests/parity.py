"""Shared helpers of the parity tests: moving the seeded inputs to the device,
reading results back, and the tolerances.

Coefficients (fp32): |gpu - oracle| <= 1e-5 absolute.

bf16 outputs y = sum_j h_j v_j: the literal rule is
    |gpu - ref| <= max(1e-2 |ref|, 2 ulp_bf16(ref)),
which no fp32-accumulating kernel can meet where the terms cancel to
|ref| ~ 1e-5.  The bound used instead adds the error that the allowed 1e-5
coefficient error alone can produce, 1e-5 * sum_j |v_j|:
    |gpu - ref| <= max(1e-2 |ref|, 2 ulp_bf16(ref)) + 1e-5 * sum_j |v_j|.
The literal-rule misses are counted and reported.  A second, tight check
("rounding only") feeds the oracle the GPU's own coefficients: then the only
differences are fp32 accumulation and the final rounding,
    |gpu - ref| <= 1 ulp_bf16(ref) + 2^-20 * sum_j |h_j v_j|.
fp32 outputs: |gpu - ref| <= 1e-5 * sum_j |v_j| + 1e-6 |ref| (coefficient
error plus fp32 rounding), and the rounding-only variant uses
2^-20 * sum_j |h_j v_j| + 2^-22 |ref|.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle

COEF_ATOL = 1e-5


def dev(a: np.ndarray, device="cuda") -> torch.Tensor:
    """numpy storage array -> device tensor (uint16 = bf16 bits)."""
    if a.dtype == np.uint16:
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(device)
    return torch.from_numpy(np.ascontiguousarray(a)).to(device)


def phi_dev(phi: np.ndarray, device="cuda") -> torch.Tensor:
    """Projection [nC][P] (the pages' orientation, as the oracle takes it) ->
    device tensor in the library's layout, phi^T [P][nC]."""
    return dev(np.ascontiguousarray(phi.T), device)


def host(t: torch.Tensor) -> np.ndarray:
    """device tensor -> float64 numpy (exact widening)."""
    t = t.detach().cpu()
    if t.dtype == torch.bfloat16:
        return oracle.widen(t.view(torch.int16).numpy().view(np.uint16))
    return t.numpy().astype(np.float64)


def ulp_bf16(x: np.ndarray) -> np.ndarray:
    ax = np.abs(x)
    _, e = np.frexp(np.maximum(ax, 2.0 ** -126))
    return np.ldexp(1.0, e - 8)


def check_coeffs(gpu: np.ndarray, ref: np.ndarray, name: str, atol: float = COEF_ATOL):
    err = np.abs(gpu - ref)
    worst = float(err.max()) if err.size else 0.0
    assert worst <= atol, f"{name}: max |gpu - oracle| = {worst:.3e} > {atol:g}"
    return worst


def check_mix(gpu: np.ndarray, ref: np.ndarray, absterms: np.ndarray, dtype: str, name: str,
              coef_tol: float = COEF_ATOL):
    """End-to-end check of a mixed output; absterms = sum_j |v_j| per element."""
    err = np.abs(gpu - ref)
    if dtype == "bf16":
        lit = np.maximum(1e-2 * np.abs(ref), 2 * ulp_bf16(ref))
        tol = lit + coef_tol * absterms
    else:
        lit = 1e-6 * np.abs(ref)
        tol = lit + coef_tol * absterms
    bad = err > tol
    assert not bad.any(), (f"{name}: {int(bad.sum())} of {err.size} elements outside tolerance; "
                           f"worst excess {float((err - tol).max()):.3e}")
    return int((err > lit).sum())


def check_rounding(gpu: np.ndarray, ref: np.ndarray, absprods: np.ndarray, dtype: str, name: str):
    """Tight check with the GPU's own coefficients; absprods = sum_j |h_j v_j|."""
    err = np.abs(gpu - ref)
    if dtype == "bf16":
        tol = ulp_bf16(ref) + 2.0 ** -20 * absprods
    else:
        tol = 2.0 ** -22 * np.abs(ref) + 2.0 ** -20 * absprods
    bad = err > tol
    assert not bad.any(), (f"{name}: {int(bad.sum())} of {err.size} elements outside the "
                           f"rounding bound; worst excess {float((err - tol).max()):.3e}")
