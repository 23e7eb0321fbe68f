"""GPU parity of hc_pre (the HC tanh coefficients, mHC page section 3 Eq.(5), and
x_in = H_pre X of Eq.(3)) and mhc_amax_gain (the Amax Gain Magnitude of section
3.1) against the fp64 oracle, through the C ABI.

Small cases span several blocks and a ragged tail and are compared element by
element; the LLM-shaped workload (T=8192, n=4, C=4096, bf16) runs in the
benchmark's launch configuration and is compared on sampled tokens.  A stack of
layers run through the library shows what the diagnostic is for: the composite
residual map of HC layers drifts away from a gain of 1, that of mHC layers does
not (section 4.1, compositional closure)."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import stream_residual_connections_b200 as M
import synth
from tests.parity import check_coeffs, check_mix, check_rounding, dev, host, phi_dev

pytestmark = pytest.mark.gpu


def _run_hc(inp, theta_dtype=None):
    X, theta = dev(inp["X"]), dev(inp["theta"])
    if theta_dtype == "f32":
        theta = dev(oracle.widen(inp["theta"]).astype(np.float32))
    b = torch.from_numpy(inp["b"]).cuda()
    x_in, Hp, Ho, Hr = M.hc_pre(X, theta, inp["alpha"], b, inp["eps"])
    torch.cuda.synchronize()
    M.mhc_sync_status()
    return dict(x_in=host(x_in), H_pre=host(Hp), H_post=host(Ho), H_res=host(Hr))


def _compare_hc(inp, got, tokens=None):
    sel = slice(None) if tokens is None else tokens
    X = oracle.widen(inp["X"][sel])
    ref = oracle.hc_pre(X, inp["theta"], inp["alpha"], inp["b"], inp["eps"])
    g = {k: v[sel] for k, v in got.items()}
    for key in ("H_pre", "H_post", "H_res"):
        check_coeffs(g[key], ref[key], key)
    dt = inp["dtype"]
    absX = np.abs(X).sum(1)
    check_mix(g["x_in"], ref["x_in"], absX, dt, "x_in")
    ref_in = oracle.mhc_apply_pre(X, g["H_pre"])
    check_rounding(g["x_in"], ref_in, np.einsum("ti,tic->tc", np.abs(g["H_pre"]), np.abs(X)), dt, "x_in")


@pytest.mark.parametrize("T,n,C,dtype,tdt", [
    (64, 4, 256, "f32", None), (257, 4, 1024, "bf16", None), (100, 1, 128, "bf16", None),
    (33, 8, 512, "bf16", None), (45, 3, 2048, "bf16", "f32"), (1, 5, 8, "f32", None),
    (300, 6, 520, "bf16", None), (1000, 2, 4096, "bf16", None), (17, 7, 264, "f32", None)])
def test_hc_pre_matches_oracle(T, n, C, dtype, tdt):
    """Every coefficient and x_in element against the oracle; gates alpha = 0.8 so
    that the tanh terms carry weight (the workloads' 0.01 would hide them)."""
    inp = synth.hc_inputs(T, n, C, dtype, seed=500 + T + n + C, alpha=0.8)
    _compare_hc(inp, _run_hc(inp, tdt))


def test_hc_pre_without_h_pre_buffer_and_empty_batch():
    inp = synth.hc_inputs(50, 4, 512, "bf16", seed=531, alpha=0.8)
    got = _run_hc(inp)
    X, theta = dev(inp["X"]), dev(inp["theta"])
    b = torch.from_numpy(inp["b"]).cuda()
    x2, Hp2, _, _ = M.hc_pre(X, theta, inp["alpha"], b, inp["eps"], want_H_pre=False)
    torch.cuda.synchronize()
    assert Hp2 is None
    np.testing.assert_array_equal(host(x2), got["x_in"])
    e = torch.empty((0, 4, 512), dtype=torch.bfloat16, device="cuda")
    x0, _, _, _ = M.hc_pre(e, theta, inp["alpha"], b)
    assert x0.shape == (0, 512)


def test_hc_zero_gates_give_the_bias_and_a_plain_mix():
    """alpha = 0: H = b exactly (Eq.5), so x_in = sum_s b_pre[s] X[s]."""
    inp = synth.hc_inputs(40, 4, 256, "f32", seed=532, alpha=0.0)
    got = _run_hc(inp)
    n = 4
    b = inp["b"].astype(np.float64)
    np.testing.assert_array_equal(got["H_pre"], np.broadcast_to(b[:n].astype(np.float32), (40, n)))
    np.testing.assert_array_equal(got["H_res"], np.broadcast_to(b[2 * n:].reshape(n, n).astype(np.float32), (40, n, n)))
    _compare_hc(inp, got)


def test_hc_llm_workload_sampled_tokens():
    """T=8192, n=4, C=4096 bf16 (the benchmark's HC workload and launch
    configuration): 64 sampled tokens against the oracle, finite outputs overall."""
    inp = synth.hc_inputs(**synth.WORKLOADS["hc_llm"])
    X, theta = dev(inp["X"]), dev(inp["theta"])
    b = torch.from_numpy(inp["b"]).cuda()
    x_in, Hp, Ho, Hr = M.hc_pre(X, theta, inp["alpha"], b, inp["eps"])
    torch.cuda.synchronize()
    M.mhc_sync_status()
    assert torch.isfinite(x_in.float()).all() and torch.isfinite(Hr).all()
    rng = np.random.default_rng(1)
    toks = np.unique(np.concatenate([[0, 8191], rng.choice(8192, 62, replace=False)]))
    sel = torch.from_numpy(toks).cuda()
    got = dict(x_in=host(x_in[sel]), H_pre=host(Hp[sel]), H_post=host(Ho[sel]), H_res=host(Hr[sel]))
    _compare_hc(dict(inp, X=inp["X"][toks]), got)


# ------------------------------------------------------------------ Amax Gain

def _gain_tolerance(H: np.ndarray) -> np.ndarray:
    """First-order bound of the fp32 error of the gains: a rounding error made at
    depth k travels to depth d through the same maps as M itself, so each of the
    about n d roundings up to depth d adds at most a few ulps of |M_d| (the
    composite of the same fp32 matrices, in fp64): 4 n d 2^-24 times its largest
    absolute row / column sum (|sum_j M[i][j]| <= sum_j |M[i][j]|).  Deep random
    chains measured at under 1/30 of it."""
    Lz, T, n, _ = H.shape
    Mc = np.broadcast_to(np.eye(n), (T, n, n)).copy()
    tol = np.empty((Lz, T, 2))
    for d in range(Lz):
        Mc = np.einsum("tik,tkj->tij", H[d], Mc)
        A = np.abs(Mc)
        tol[d, :, 0] = A.sum(2).max(1)
        tol[d, :, 1] = A.sum(1).max(1)
        tol[d] *= 4 * n * (d + 1) * 2.0 ** -24
    return tol + 1e-30


@pytest.mark.parametrize("Lz,T,n", [(24, 1000, 4), (5, 300, 1), (9, 257, 3), (12, 64, 8), (1, 1, 2),
                                    (2, 80000, 2), (6200, 40, 2)])
def test_amax_gain_matches_oracle(Lz, T, n):
    """Includes more token groups than resident blocks (T = 80000: every block walks
    several groups) and more layers than the block maxima's shared memory holds
    (L = 6200: maxima straight to global memory)."""
    rng = np.random.default_rng(600 + Lz + T + n)
    sd = 0.3 if Lz <= 64 else 0.3 * np.sqrt(24 / Lz)   # deep stacks: keep the product finite
    H = (np.eye(n) + rng.normal(size=(Lz, T, n, n)) * sd).astype(np.float32)
    g, gm = M.mhc_amax_gain(torch.from_numpy(H).cuda())
    torch.cuda.synchronize()
    g, gm = host(g), host(gm)
    ref = oracle.amax_gain(H)
    err = np.abs(g - ref)
    tol = _gain_tolerance(H.astype(np.float64))
    assert (err <= tol).all(), f"worst excess {float((err - tol).max()):.3e}"
    # the maxima over tokens are the kernel's own per-token maxima, bit for bit
    np.testing.assert_array_equal(gm, g.max(axis=1))


def test_amax_gain_outputs_optional_and_empty():
    rng = np.random.default_rng(7)
    H = torch.from_numpy((np.eye(4) + rng.normal(size=(6, 100, 4, 4)) * 0.2).astype(np.float32)).cuda()
    g, gm = M.mhc_amax_gain(H)
    g2, gm2 = M.mhc_amax_gain(H, want_gain=False)
    torch.cuda.synchronize()
    assert g2 is None
    np.testing.assert_array_equal(host(gm2), host(gm))
    _, gm0 = M.mhc_amax_gain(H[:, :0].contiguous(), want_gain=False)
    torch.cuda.synchronize()
    assert (host(gm0) == 0).all()


def test_stacked_layers_hc_drifts_mhc_stays_at_one():
    """L = 16 layers, each a fresh sublayer (its own parameters, F_out drawn per
    layer), run through the library: hc_pre or mhc_pre, then mhc_post.  The
    diagnostic over the GPU's H_res stack matches the oracle's on the same
    matrices; the mHC composite keeps every row sum at 1 (forward gain 1), the
    HC composite does not."""
    Lz, T, n, C = 16, 256, 4, 512
    stacks = {}
    for kind in ("hc", "mhc"):
        X = dev(synth.mhc_inputs(T, n, C, "bf16", seed=700)["X"])
        Hs = []
        for layer in range(Lz):
            if kind == "hc":
                inp = synth.hc_inputs(T, n, C, "bf16", seed=710 + layer, alpha=0.5)
                _, _, Ho, Hr = M.hc_pre(X, dev(inp["theta"]), inp["alpha"],
                                        torch.from_numpy(inp["b"]).cuda(), inp["eps"])
            else:
                inp = synth.mhc_inputs(T, n, C, "bf16", seed=710 + layer, alpha=0.5)
                _, _, Ho, Hr = M.mhc_pre(X, phi_dev(inp["phi"]), inp["alpha"],
                                         torch.from_numpy(inp["b"]).cuda(), 20, inp["eps"])
            X = M.mhc_post(X, dev(inp["F"]), Ho, Hr)
            Hs.append(Hr)
        H = torch.stack(Hs).contiguous()
        g, gm = M.mhc_amax_gain(H)
        torch.cuda.synchronize()
        M.mhc_sync_status()
        Hh = host(H)
        ref = oracle.amax_gain(Hh)
        err = np.abs(host(g) - ref)
        assert (err <= _gain_tolerance(Hh)).all()
        stacks[kind] = (host(g), host(gm))
    g_m, _ = stacks["mhc"]
    np.testing.assert_allclose(g_m[..., 0], 1.0, atol=Lz * 3e-6)   # rows of each H_res: 1 within 2e-6
    g_h, gm_h = stacks["hc"]
    assert np.abs(g_h[-1, :, 0] - 1.0).max() > 0.1 and gm_h[-1, 0] > 1.1
