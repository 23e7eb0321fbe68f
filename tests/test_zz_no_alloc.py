"""mhc_backward_noalloc: the backward for callers that cannot allocate device
memory (for instance code running while a CUDA graph is captured, or a runtime
that owns every allocation).  It uses a scratch array built into the library
instead of a caller workspace.

This file is collected last so that, if it fails, a run stopping at the first
failure has already run every other test; it does not depend on them and also
passes alone in a fresh process (the first call sets up the scratch address).
"""
from __future__ import annotations

import ctypes as ct

import numpy as np
import pytest
import torch

import stream_residual_connections_b200 as M
import synth
from tests.parity import check_mix, dev, host, phi_dev

pytestmark = pytest.mark.gpu

SUM_REL = 1e-3            # as tests/test_gpu_bwd.py for the token sums
GRAD_COEF_TOL = 1e-4      # as tests/test_gpu_bwd.py for dX and dF_out


def _inputs():
    inp = synth.mhc_grad_inputs(300, 4, 512, "bf16", seed=900)
    return dict(X=dev(inp["X"]), F=dev(inp["F"]), phi=phi_dev(inp["phi"]),
                b=torch.from_numpy(inp["b"]).cuda(), dXn=dev(inp["dX_next"]), dxi=dev(inp["dx_in"]),
                alpha=inp["alpha"], eps=inp["eps"])


def _noalloc(d, outs):
    """One call through the C ABI, outputs written into `outs` (filled with NaN first)."""
    for o in outs:
        o.fill_(float("nan"))
    T, n, C = d["X"].shape
    lib = M.native()
    alpha = (ct.c_float * 3)(*[float(a) for a in d["alpha"]])
    p = lambda t: ct.c_void_p(t.data_ptr())
    st = lib.mhc_backward_noalloc(p(d["X"]), p(d["F"]), p(d["phi"]), M.MHC_BF16, alpha, p(d["b"]),
                                  p(d["dXn"]), p(d["dxi"]), T, n, C, 20, d["eps"], p(outs[0]), p(outs[1]),
                                  p(outs[2]), p(outs[3]), p(outs[4]),
                                  ct.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == M.MHC_OK, lib.mhc_last_error().decode()
    torch.cuda.synchronize()
    return [host(o) for o in outs]


def test_noalloc_backward_matches_the_workspace_backward_on_two_calls():
    d = _inputs()
    ref = [host(o) for o in M.mhc_backward(d["X"], d["F"], d["phi"], d["alpha"], d["b"], d["dXn"],
                                            d["dxi"], 20, d["eps"])]
    torch.cuda.synchronize()
    T, n, C = d["X"].shape
    P = n * n + 2 * n
    outs = [torch.empty_like(d["X"]), torch.empty_like(d["F"]),
            torch.empty((P, n * C), dtype=torch.float32, device="cuda"),
            torch.empty(3, dtype=torch.float32, device="cuda"), torch.empty(P, dtype=torch.float32, device="cuda")]
    Xh = host(d["X"])
    terms_dX = np.abs(host(d["dXn"])).sum(1)[:, None, :] + np.abs(host(d["dxi"]))[:, None, :] + np.abs(Xh) + 1.0
    for _ in range(2):                      # the scratch keeps the first call's leftovers
        got = _noalloc(d, outs)
        check_mix(got[0], ref[0], terms_dX, "bf16", "dX", coef_tol=GRAD_COEF_TOL)
        check_mix(got[1], ref[1], np.abs(host(d["dXn"])).sum(1), "bf16", "dF", coef_tol=GRAD_COEF_TOL)
        for g, r, name in zip(got[2:], ref[2:], ("dphi", "dalpha", "db")):
            assert np.isfinite(g).all(), name
            assert np.abs(g - r).max() <= SUM_REL * np.abs(r).max() + 1e-6, name


def test_noalloc_backward_rejects_batches_beyond_its_scratch():
    lib = M.native()
    need = M.mhc_backward_workspace_bytes(200000, 4, 512)
    assert need > (4 << 20)
    alpha = (ct.c_float * 3)(0.01, 0.01, 0.01)
    fake = ct.c_void_p(1 << 20)
    st = lib.mhc_backward_noalloc(fake, fake, fake, M.MHC_BF16, alpha, fake, fake, fake, 200000, 4, 512, 20,
                                  1e-6, fake, fake, fake, fake, fake, None)
    assert st == M.MHC_ERR_UNSUPPORTED
    assert "scratch" in lib.mhc_last_error().decode()
