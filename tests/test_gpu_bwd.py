"""GPU parity of mhc_backward against the fp64 oracle's reverse mode (itself
pinned by central finite differences and torch float64 autograd), through the
C ABI.  [mHC] section 4.3.1: backward through the projection and through all
Sinkhorn iterations.

Tolerances: dX and dF_out are bf16/fp32 outputs checked like the forward's
mixes, with the coefficient-gradient error allowance raised to 1e-4 (the
gradient coefficients come out of fp32 dot products over C and a 20-step
Sinkhorn reverse).  dphi, db and dalpha are fp32 sums over tokens: each
element within 1e-3 of the tensor's largest magnitude (plus 1e-6)."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import stream_residual_connections_b200 as M
import synth
from tests.parity import check_mix, dev, host, phi_dev

pytestmark = pytest.mark.gpu

GRAD_COEF_TOL = 1e-4
SUM_REL = 1e-3


def _check_sum(gpu, ref, name):
    scale = float(np.abs(ref).max()) if ref.size else 0.0
    err = float(np.abs(gpu - ref).max()) if ref.size else 0.0
    assert err <= SUM_REL * scale + 1e-6, f"{name}: max error {err:.3e} vs scale {scale:.3e}"


def _run(inp, t_iters=20):
    T, n, C = inp["T"], inp["n"], inp["C"]
    X, F = dev(inp["X"]), dev(inp["F"])
    dXn, dxi = dev(inp["dX_next"]), dev(inp["dx_in"])
    b = torch.from_numpy(inp["b"]).cuda()
    out = M.mhc_backward(X, F, phi_dev(inp["phi"]), inp["alpha"], b, dXn, dxi, t_iters, inp["eps"])
    M.mhc_sync_status()
    return [host(o) for o in out]


def _compare(inp, got, t_iters=20, tokens=None):
    dX, dF, dphiT, dalpha, db = got
    X, F = oracle.widen(inp["X"]), oracle.widen(inp["F"])
    dXn, dxi = oracle.widen(inp["dX_next"]), oracle.widen(inp["dx_in"])
    ref = oracle.mhc_backward(X, F, inp["phi"], inp["alpha"], inp["b"], dXn, dxi, t_iters, inp["eps"])
    _check_sum(dphiT.T, ref["dphi"], "dphi")
    _check_sum(db, ref["db"], "db")
    _check_sum(dalpha, ref["dalpha"], "dalpha")
    sel = slice(None) if tokens is None else tokens
    dt = inp["dtype"]
    phi = oracle.widen(inp["phi"])                     # [nC][P]
    n, C = inp["n"], inp["C"]
    # size of the terms of dX_j: the mixes of the upstream gradients, the projection
    # term phi dd and the RMS term (bounded by the row's own magnitude)
    absphi = np.abs(phi).sum(1).reshape(n, C)        # sum_p |phi[k][p]|
    gsum = np.abs(dXn[sel]).sum(1)
    terms = (gsum[:, None, :] + np.abs(dxi[sel])[:, None, :] + absphi[None] + np.abs(X[sel]))
    check_mix(dX[sel], ref["dX"][sel], terms, dt, "dX", coef_tol=GRAD_COEF_TOL)
    check_mix(dF[sel], ref["dF"][sel], gsum, dt, "dF", coef_tol=GRAD_COEF_TOL)


@pytest.mark.parametrize("T,n,C,dtype", [(37, 4, 64, "f32"), (50, 2, 128, "bf16"), (100, 4, 512, "bf16"),
                                         (20, 3, 192, "bf16"), (16, 1, 64, "f32"), (33, 4, 1024, "f32")])
def test_backward_matches_oracle(T, n, C, dtype):
    inp = synth.mhc_grad_inputs(T, n, C, dtype, seed=800 + T + n + C)
    _compare(inp, _run(inp))


@pytest.mark.parametrize("T,n,C", [(1500, 4, 256), (8200, 2, 128), (64, 1, 128), (77, 3, 512)])
def test_backward_dphi_tensor_core_shapes(T, n, C):
    """bf16 with nC % 128 == 0 takes the tensor-core dphi product (dd^T pair x X over
    token segments): three segments with a ragged last one (T=1500), 16 segments of 576
    tokens of which the last is empty and must contribute zeros (T=8200), n = 1 and 3."""
    inp = synth.mhc_grad_inputs(T, n, C, "bf16", seed=830 + T + n + C)
    _compare(inp, _run(inp))


def test_backward_dphi_paths_agree():
    """The tensor-core dphi product against the CUDA-core one on the same inputs."""
    inp = synth.mhc_grad_inputs(1000, 4, 512, "bf16", seed=840)
    try:
        M.mhc_set_path(M.MHC_PATH_FMA)
        a = _run(inp)
    finally:
        M.mhc_set_path(M.MHC_PATH_AUTO)
    c = _run(inp)
    scale = float(np.abs(a[2]).max())
    assert np.abs(a[2] - c[2]).max() <= 1e-4 * scale
    np.testing.assert_allclose(c[4], a[4], rtol=0, atol=1e-4 * float(np.abs(a[4]).max()))


@pytest.mark.parametrize("t_iters", [0, 1, 5])
def test_backward_short_sinkhorn(t_iters):
    inp = synth.mhc_grad_inputs(24, 4, 128, "f32", seed=810 + t_iters)
    _compare(inp, _run(inp, t_iters), t_iters)


def test_backward_is_bitwise_reproducible():
    inp = synth.mhc_grad_inputs(300, 4, 512, "bf16", seed=820)
    a, b = _run(inp), _run(inp)
    for x, y in zip(a, b):
        np.testing.assert_array_equal(x, y)


def test_backward_empty_batch_zeroes_sums():
    X = torch.zeros((0, 4, 64), dtype=torch.bfloat16, device="cuda")
    F = torch.zeros((0, 64), dtype=torch.bfloat16, device="cuda")
    phi = torch.zeros((24, 256), dtype=torch.bfloat16, device="cuda")
    b = torch.zeros(24, device="cuda")
    dphi = torch.full((24, 256), 7.0, device="cuda")
    _, _, dphi, da, db = M.mhc_backward(X, F, phi, [0.01] * 3, b, X, F, dphi=dphi,
                                        workspace=torch.empty(256, dtype=torch.uint8, device="cuda"))
    torch.cuda.synchronize()
    assert (dphi == 0).all() and (da == 0).all() and (db == 0).all()


def test_backward_llm_workload():
    """n=4, C=4096, T=8192, bf16: dphi, db, dalpha over all tokens; dX, dF on 48 sampled tokens."""
    inp = synth.mhc_grad_inputs(**synth.WORKLOADS["mhc_bwd"])
    got = _run(inp)
    rng = np.random.default_rng(4)
    toks = np.unique(np.concatenate([[0, 8191], rng.choice(8192, 46, replace=False)]))
    _compare(inp, got, tokens=toks)
