"""GPU parity of mhc_pre / mhc_post against the fp64 oracle, through the C ABI.

Small cases span several tiles and a ragged tail and are compared element by
element; the LLM-scale workload (T=8192, n=4, C=4096, bf16) runs in the
bench's launch configuration and is compared on sampled tokens."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import stream_residual_connections_b200 as M
import synth
from tests.parity import check_coeffs, check_mix, check_rounding, dev, host, phi_dev

pytestmark = pytest.mark.gpu


def _run(inp, phi_dtype=None):
    X, F, phi = dev(inp["X"]), dev(inp["F"]), phi_dev(inp["phi"])
    if phi_dtype == "f32":
        phi = phi_dev(oracle.widen(inp["phi"]).astype(np.float32))
    b = torch.from_numpy(inp["b"]).cuda()
    x_in, Hp, Ho, Hr = M.mhc_pre(X, phi, inp["alpha"], b, inp["t_iters"], inp["eps"])
    Xn = M.mhc_post(X, F, Ho, Hr)
    torch.cuda.synchronize()
    M.mhc_sync_status()
    return dict(x_in=host(x_in), H_pre=host(Hp), H_post=host(Ho), H_res=host(Hr), X_next=host(Xn))


def _compare(inp, got, tokens=None):
    sel = slice(None) if tokens is None else tokens
    X = oracle.widen(inp["X"][sel])
    F = oracle.widen(inp["F"][sel])
    ref = oracle.mhc_forward(X, F, inp["phi"], inp["alpha"], inp["b"], inp["t_iters"], inp["eps"])
    g = {k: v[sel] for k, v in got.items()}
    for key in ("H_pre", "H_post", "H_res"):
        check_coeffs(g[key], ref[key], key)
    dt = inp["dtype"]
    absX = np.abs(X).sum(1)
    miss = check_mix(g["x_in"], ref["x_in"], absX, dt, "x_in")
    miss += check_mix(g["X_next"], ref["X_next"], absX[:, None, :] + np.abs(F)[:, None, :], dt, "X_next")
    # rounding-only: the oracle's apply steps fed the GPU's own coefficients
    ref_in = oracle.mhc_apply_pre(X, g["H_pre"])
    check_rounding(g["x_in"], ref_in, np.einsum("ti,tic->tc", np.abs(g["H_pre"]), np.abs(X)), dt, "x_in")
    ref_n = oracle.mhc_post(X, F, g["H_post"], g["H_res"])
    prods = (np.einsum("tij,tjc->tic", np.abs(g["H_res"]), np.abs(X))
             + np.abs(g["H_post"])[:, :, None] * np.abs(F)[:, None, :])
    check_rounding(g["X_next"], ref_n, prods, dt, "X_next")
    # Sinkhorn output on the GPU: non-negative, rows sum to 1 (last step is T_r)
    assert (g["H_res"] >= 0).all()
    if inp["t_iters"] >= 1:
        np.testing.assert_allclose(g["H_res"].sum(-1), 1.0, atol=2e-6)
    return miss


def test_tiny_fp32_workload():
    """T=64, n=4, C=256, fp32 throughout (all outputs compared)."""
    inp = synth.mhc_inputs(**synth.WORKLOADS["mhc_tiny"])
    _compare(inp, _run(inp))


@pytest.mark.parametrize("T,n,C", [(1, 4, 64), (3, 1, 8), (67, 4, 264), (300, 4, 1024),
                                   (130, 2, 512), (40, 8, 512), (37, 3, 136), (20, 5, 256),
                                   (9, 6, 96), (11, 7, 64), (257, 4, 4096)])
def test_bf16_shapes(T, n, C):
    inp = synth.mhc_inputs(T, n, C, "bf16", seed=100 + T + n + C)
    _compare(inp, _run(inp))


def test_bf16_x_with_fp32_phi():
    inp = synth.mhc_inputs(70, 4, 512, "bf16", seed=7)
    inp32 = dict(inp, phi=oracle.widen(inp["phi"]).astype(np.float32))
    _compare(inp32, _run(inp, phi_dtype="f32"))


def test_fp32_shapes_all_n():
    for n in range(1, 9):
        inp = synth.mhc_inputs(19, n, 64, "f32", seed=200 + n)
        _compare(inp, _run(inp))


def test_t_iters_zero_and_one():
    for t in (0, 1, 3):
        inp = synth.mhc_inputs(25, 4, 128, "f32", seed=300 + t)
        inp["t_iters"] = t
        _compare(inp, _run(inp))


def test_post_in_place():
    inp = synth.mhc_inputs(50, 4, 256, "bf16", seed=11)
    X, F = dev(inp["X"]), dev(inp["F"])
    b = torch.from_numpy(inp["b"]).cuda()
    _, _, Ho, Hr = M.mhc_pre(X, phi_dev(inp["phi"]), inp["alpha"], b)
    ref = M.mhc_post(X, F, Ho, Hr)
    out = M.mhc_post(X, F, Ho, Hr, X_next=X)
    torch.cuda.synchronize()
    assert out.data_ptr() == X.data_ptr()
    assert torch.equal(ref, X)


def test_empty_T_is_a_no_op():
    X = torch.zeros((0, 4, 64), dtype=torch.bfloat16, device="cuda")
    phi = torch.zeros((24, 256), dtype=torch.bfloat16, device="cuda")
    b = torch.zeros(24, device="cuda")
    x_in, *_ = M.mhc_pre(X, phi, [0.01] * 3, b)
    assert x_in.shape == (0, 64)
    M.mhc_post(X, torch.zeros((0, 64), dtype=torch.bfloat16, device="cuda"),
               torch.zeros((0, 4), device="cuda"), torch.zeros((0, 4, 4), device="cuda"))


def test_plain_residual_and_permutation_reduction_exact():
    """mHC page Eq.(1) vs Eq.(3): alpha = 0 with +-40 biases gives H_res = P_sigma,
    H_pre = e_2, H_post = 1; x_in = X[2] and X_next[i] = X[sigma(i)] + F, both
    bit-exact after the single bf16 rounding."""
    T, n, C = 37, 4, 264
    inp = synth.mhc_inputs(T, n, C, "bf16", seed=12)
    sig = [1, 2, 0, 3]
    b = np.zeros(24, dtype=np.float32)
    b[:n] = -40.0; b[2] = 40.0
    res = np.full((n, n), -40.0, dtype=np.float32)
    for i in range(n):
        res[i, sig[i]] = 40.0
    b[2 * n:] = res.reshape(-1)
    inp["b"] = b
    inp["alpha"] = np.zeros(3, dtype=np.float32)
    got = _run(inp)
    X, F = oracle.widen(inp["X"]), oracle.widen(inp["F"])
    np.testing.assert_array_equal(got["x_in"], X[:, 2])
    expect = oracle.widen(synth.f32_to_bf16_bits((X[:, sig] + F[:, None, :]).astype(np.float32)))
    # bit-exact wherever X[sigma(i)] + F is not 0; where it cancels, the off-diagonal
    # H_res weights exp(-80) (the oracle's too) leave a value of order 1e-35
    nz = expect != 0
    np.testing.assert_array_equal(got["X_next"][nz], expect[nz])
    assert np.abs(got["X_next"][~nz]).max(initial=0.0) < 1e-30
    np.testing.assert_allclose(got["H_res"], np.broadcast_to(np.eye(n)[sig], (T, n, n)), atol=1e-30)


def test_n1_exact_identity():
    inp = synth.mhc_inputs(33, 1, 128, "bf16", seed=13)
    got = _run(inp)
    assert (got["H_res"] == 1.0).all()


def test_llm_workload_sampled_tokens():
    """T=8192, n=4, C=4096 bf16 (the benchmark's workload and launch configuration):
    every coefficient and output of 64 sampled tokens, plus properties over all tokens."""
    inp = synth.mhc_inputs(**synth.WORKLOADS["mhc_llm"])
    got = _run(inp)
    rng = np.random.default_rng(0)
    toks = np.unique(np.concatenate([[0, 1, 8191], rng.choice(8192, 61, replace=False)]))
    _compare(inp, got, toks)
    assert np.isfinite(got["X_next"]).all() and np.isfinite(got["x_in"]).all()
    assert (got["H_res"] >= 0).all()
    np.testing.assert_allclose(got["H_res"].sum(-1), 1.0, atol=2e-6)
    np.testing.assert_allclose(got["H_res"].sum(-2), 1.0, atol=1e-3)
    assert ((got["H_pre"] > 0) & (got["H_pre"] < 1)).all()
    assert ((got["H_post"] > 0) & (got["H_post"] < 2)).all()


def _run_sampled(inp, toks):
    """Full-size run on the GPU; the sampled tokens' outputs come back to the host,
    the structural properties are checked on the device over all tokens."""
    X, F, phi = dev(inp["X"]), dev(inp["F"]), phi_dev(inp["phi"])
    b = torch.from_numpy(inp["b"]).cuda()
    x_in, Hp, Ho, Hr = M.mhc_pre(X, phi, inp["alpha"], b, inp["t_iters"], inp["eps"])
    Xn = M.mhc_post(X, F, Ho, Hr)
    torch.cuda.synchronize()
    M.mhc_sync_status()                        # no expired wait, no failed self-check
    assert torch.isfinite(Xn.float()).all() and torch.isfinite(x_in.float()).all()
    assert (Hr >= 0).all() and ((Hp > 0) & (Hp < 1)).all() and ((Ho > 0) & (Ho < 2)).all()
    assert (Hr.sum(-1) - 1.0).abs().max().item() <= 2e-6
    sel = torch.from_numpy(np.asarray(toks)).cuda()
    return dict(x_in=host(x_in[sel]), H_pre=host(Hp[sel]), H_post=host(Ho[sel]), H_res=host(Hr[sel]),
                X_next=host(Xn[sel]))


@pytest.mark.parametrize("name", ["mhc_wide", "mhc_sweep_n2", "mhc_sweep_n8"])
def test_wide_and_n_sweep_workloads_sampled(name):
    """The remaining forward workloads at full size: T=32768, n=4, C=7168 (14 channel
    blocks per CTA on the tensor-core path), and n = 2 (tensor cores) and n = 8 (CUDA
    cores) at T=8192, C=4096; 48 sampled tokens compared with the oracle."""
    inp = synth.mhc_inputs(**synth.WORKLOADS[name])
    T = inp["T"]
    rng = np.random.default_rng(5)
    toks = np.unique(np.concatenate([[0, T - 1], rng.choice(T, 46, replace=False)]))
    got = _run_sampled(inp, toks)
    _compare(dict(inp, X=inp["X"][toks], F=inp["F"][toks]), got)


@pytest.fixture
def restore_path():
    yield
    M.mhc_set_path(M.MHC_PATH_AUTO)
    M.mhc_set_wait_limit(1 << 26)


@pytest.mark.parametrize("T,n,C", [(1, 4, 512), (3, 4, 512), (129, 4, 1024), (1000, 2, 512),
                                   (300, 3, 2048), (257, 4, 4096), (50, 4, 2048), (2500, 4, 1024),
                                   (700, 4, 7168), (333, 3, 7168), (901, 4, 1536), (450, 2, 3072),
                                   (5000, 4, 4096)])
def test_tensor_core_path_shapes(T, n, C, restore_path):
    """TMA + tcgen05 projection (8-CTA clusters): one and several tiles per
    cluster, ragged last tile (Mt from 8 to 64 rows), n = 2, 3 (a zero-filled
    fourth stream), 4; one to 14 channel blocks per CTA (C = 512 ... 7168)."""
    M.mhc_set_path(M.MHC_PATH_TENSOR)
    inp = synth.mhc_inputs(T, n, C, "bf16", seed=400 + T + n + C)
    _compare(inp, _run(inp))


@pytest.mark.parametrize("T,n,C", [(300, 8, 512), (1000, 5, 1024), (129, 6, 512), (77, 7, 1536), (1, 8, 512),
                                   (2048, 8, 2048)])
def test_tensor_core_path_n5_to_8(T, n, C, restore_path):
    """n = 5..8: projection kernel on tensor cores (one stream of a 128-token tile per
    stage, every stream accumulating into the same P columns) + streaming x_in pass."""
    M.mhc_set_path(M.MHC_PATH_TENSOR)
    inp = synth.mhc_inputs(T, n, C, "bf16", seed=450 + T + n + C)
    _compare(inp, _run(inp))


def test_n8_without_h_pre_buffer(restore_path):
    """No H_pre buffer from the caller: the gates wait in the x_in rows between the
    projection and the x_in pass; x_in must be the same."""
    inp = synth.mhc_inputs(200, 8, 512, "bf16", seed=460)
    got = _run(inp)
    X, phi = dev(inp["X"]), phi_dev(inp["phi"])
    b = torch.from_numpy(inp["b"]).cuda()
    x_in2, Hp2, _, _ = M.mhc_pre(X, phi, inp["alpha"], b, inp["t_iters"], inp["eps"], want_H_pre=False)
    torch.cuda.synchronize()
    assert Hp2 is None
    np.testing.assert_array_equal(host(x_in2), got["x_in"])


@pytest.mark.parametrize("n", [4, 8])
def test_tensor_and_fma_paths_agree(n, restore_path):
    inp = synth.mhc_inputs(700, n, 1024, "bf16", seed=21)
    M.mhc_set_path(M.MHC_PATH_FMA)
    a = _run(inp)
    M.mhc_set_path(M.MHC_PATH_TENSOR)
    b = _run(inp)
    for key in ("H_pre", "H_post", "H_res"):
        assert np.abs(a[key] - b[key]).max() <= 2e-6, key
    _compare(inp, b)


def test_tensor_path_rejects_unsupported_calls(restore_path):
    M.mhc_set_path(M.MHC_PATH_TENSOR)
    inp = synth.mhc_inputs(8, 4, 264, "bf16", seed=22)           # C % 512 != 0
    with pytest.raises(M.MhcError) as e:
        _run(inp)
    assert e.value.status == M.MHC_ERR_UNSUPPORTED


def test_bounded_wait_expiry_is_reported_and_context_survives(restore_path):
    """With a one-poll limit the tensor-core kernel's waits run out: it records
    the timeout, releases TMEM and returns; the host sees MHC_ERR_TIMEOUT and
    the next normal call is correct."""
    M.mhc_set_path(M.MHC_PATH_TENSOR)
    inp = synth.mhc_inputs(2000, 4, 2048, "bf16", seed=23)
    X, phi = dev(inp["X"]), phi_dev(inp["phi"])
    b = torch.from_numpy(inp["b"]).cuda()
    M.mhc_sync_status()
    M.mhc_set_wait_limit(1)
    seen = False
    for _ in range(5):
        M.mhc_pre(X, phi, inp["alpha"], b)
        try:
            M.mhc_sync_status()
        except M.MhcError as e:
            assert e.status == M.MHC_ERR_TIMEOUT
            seen = True
            break
    M.mhc_set_wait_limit(1 << 26)
    assert seen, "no wait expired with a one-poll limit"
    M.mhc_sync_status()                       # error word was cleared
    _compare(inp, _run(inp), tokens=np.arange(0, 2000, 37))
