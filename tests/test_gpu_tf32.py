"""GPU parity of mhc_pre with the projection in tf32 (the mHC page's section 4.3.1,
Eq.(10): phi tfloat32, x bfloat16), through the C ABI.

The library takes a tf32 phi as its exact pair of bf16 rows (mhc_phi_tf32_pair);
the tensor-core kernel (n <= 7) and the CUDA-core kernel (every n) form x . hi +
x . lo = x . phi_tf32.  The oracle is the same fp64 mHC oracle given the tf32
values of phi."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import stream_residual_connections_b200 as M
import synth
from tests.parity import check_coeffs, dev, host, phi_dev
from tests.test_gpu_mhc import _compare

pytestmark = pytest.mark.gpu


def _bf16_value(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << 16).view(np.float32)


@pytest.mark.parametrize("n,C", [(1, 8), (4, 512), (7, 64), (8, 520)])
def test_pair_packing_is_exact(n, C):
    """Every element is rounded to tf32 (round to nearest even), hi = bf16(t),
    lo = bf16(t - hi); hi + lo == t exactly; the padding rows are zero."""
    P = n * n + 2 * n
    RH = (P + 15) // 16 * 16
    rng = np.random.default_rng(n * 1000 + C)
    phi = (rng.normal(size=(P, n * C)) * np.exp(rng.uniform(-20, 20, size=(P, n * C)))).astype(np.float32)
    pair = M.mhc_phi_tf32_pair(torch.from_numpy(phi).cuda(), n)
    torch.cuda.synchronize()
    assert pair.shape == (2 * RH, n * C)
    assert M.native().mhc_phi_tf32_pair_bytes(n, C) == 2 * RH * n * C * 2
    bits = pair.cpu().view(torch.int16).numpy().view(np.uint16)
    t = synth.f32_to_tf32(phi)
    hi_bits = synth.f32_to_bf16_bits(t)
    lo = t - _bf16_value(hi_bits)
    lo_bits = synth.f32_to_bf16_bits(lo)
    np.testing.assert_array_equal(bits[:P], hi_bits)
    np.testing.assert_array_equal(bits[RH:RH + P], lo_bits)
    assert (bits[P:RH] == 0).all() and (bits[RH + P:] == 0).all()
    np.testing.assert_array_equal(_bf16_value(hi_bits) + _bf16_value(lo_bits), t)


def _run_tf32(inp):
    X, F = dev(inp["X"]), dev(inp["F"])
    n = inp["n"]
    pair = M.mhc_phi_tf32_pair(phi_dev(inp["phi"]), n)
    b = torch.from_numpy(inp["b"]).cuda()
    x_in, Hp, Ho, Hr = M.mhc_pre(X, pair, inp["alpha"], b, inp["t_iters"], inp["eps"], phi_tf32_pair=True)
    Xn = M.mhc_post(X, F, Ho, Hr)
    torch.cuda.synchronize()
    M.mhc_sync_status()
    return dict(x_in=host(x_in), H_pre=host(Hp), H_post=host(Ho), H_res=host(Hr), X_next=host(Xn))


@pytest.fixture
def restore_path():
    yield
    M.mhc_set_path(M.MHC_PATH_AUTO)


@pytest.mark.parametrize("T,n,C", [(300, 4, 512), (129, 1, 512), (1000, 7, 1024), (77, 5, 2048), (64, 8, 512),
                                   (513, 3, 512), (200, 2, 4096), (1, 6, 512), (50, 4, 264)])
def test_tf32_phi_matches_oracle(T, n, C):
    """n <= 7 with C % 512 == 0 on tensor cores, n = 8 and C = 264 on CUDA cores;
    every coefficient and output against the oracle given phi's tf32 values."""
    inp = synth.mhc_inputs(T, n, C, "bf16", seed=800 + T + n + C, alpha=0.5, phi_dtype="tf32")
    _compare(inp, _run_tf32(inp))


def test_tf32_tensor_and_fma_paths_agree(restore_path):
    inp = synth.mhc_inputs(700, 4, 1024, "bf16", seed=811, alpha=0.5, phi_dtype="tf32")
    M.mhc_set_path(M.MHC_PATH_FMA)
    a = _run_tf32(inp)
    M.mhc_set_path(M.MHC_PATH_TENSOR)
    c = _run_tf32(inp)
    for key in ("H_pre", "H_post", "H_res"):
        check_coeffs(c[key], a[key], key, atol=2e-6)
    _compare(inp, c)


def test_tf32_is_the_precision_the_test_sees():
    """The bar separates the two precisions: the oracle with phi rounded to bf16
    instead of tf32 misses the tf32 GPU result by more than the 1e-5 tolerance,
    while the oracle with the tf32 phi meets it."""
    inp = synth.mhc_inputs(256, 4, 1024, "bf16", seed=812, alpha=1.0, phi_dtype="tf32")
    got = _run_tf32(inp)
    X = oracle.widen(inp["X"])
    ref = oracle.mhc_coeffs(X, inp["phi"], inp["alpha"], inp["b"])
    phi_b = oracle.widen(synth.f32_to_bf16_bits(inp["phi"]))
    ref_b = oracle.mhc_coeffs(X, phi_b, inp["alpha"], inp["b"])
    for key in ("H_pre", "H_res"):
        check_coeffs(got[key], ref[key], key)
    assert max(np.abs(got[k] - ref_b[k]).max() for k in ("H_pre", "H_post", "H_res")) > 1e-4


def test_tf32_llm_workload_sampled_tokens():
    """T=8192, n=4, C=4096 with the tf32 phi (the benchmark's tf32 workload and launch
    configuration): 64 sampled tokens against the oracle."""
    wl = dict(synth.WORKLOADS["mhc_llm"])
    inp = synth.mhc_inputs(**wl, phi_dtype="tf32")
    X, F = dev(inp["X"]), dev(inp["F"])
    pair = M.mhc_phi_tf32_pair(phi_dev(inp["phi"]), 4)
    b = torch.from_numpy(inp["b"]).cuda()
    x_in, Hp, Ho, Hr = M.mhc_pre(X, pair, inp["alpha"], b, 20, 1e-6, phi_tf32_pair=True)
    Xn = M.mhc_post(X, F, Ho, Hr)
    torch.cuda.synchronize()
    M.mhc_sync_status()
    assert torch.isfinite(Xn.float()).all() and (Hr >= 0).all()
    rng = np.random.default_rng(9)
    toks = np.unique(np.concatenate([[0, 8191], rng.choice(8192, 62, replace=False)]))
    sel = torch.from_numpy(toks).cuda()
    got = dict(x_in=host(x_in[sel]), H_pre=host(Hp[sel]), H_post=host(Ho[sel]), H_res=host(Hr[sel]),
               X_next=host(Xn[sel]))
    _compare(dict(inp, X=inp["X"][toks], F=inp["F"][toks]), got)


def test_tf32_pair_rejections(restore_path):
    inp = synth.mhc_inputs(16, 8, 512, "bf16", seed=813, phi_dtype="tf32")
    pair = M.mhc_phi_tf32_pair(phi_dev(inp["phi"]), 8)
    b = torch.from_numpy(inp["b"]).cuda()
    M.mhc_set_path(M.MHC_PATH_TENSOR)          # n = 8: 2 RH + 128 > 256, no tensor-core form
    with pytest.raises(M.MhcError) as e:
        M.mhc_pre(dev(inp["X"]), pair, inp["alpha"], b, phi_tf32_pair=True)
    assert e.value.status == M.MHC_ERR_UNSUPPORTED
    M.mhc_set_path(M.MHC_PATH_AUTO)
    Xf = torch.zeros((16, 8, 512), dtype=torch.float32, device="cuda")
    with pytest.raises(M.MhcError) as e:
        M.mhc_pre(Xf, pair, inp["alpha"], b, phi_tf32_pair=True)
    assert e.value.status == M.MHC_ERR_UNSUPPORTED
