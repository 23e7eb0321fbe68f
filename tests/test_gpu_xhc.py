"""GPU parity of the xHC kernels against the fp64 oracle, through the C ABI.

[xHC] summary page: "temporal feature augmentation" (causal depthwise convs +
Gram-Schmidt), "sparse residual stream architecture" (routing, dense read,
sparse update + scatter)."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import stream_residual_connections_b200 as M
import synth
from tests.parity import dev, host

pytestmark = pytest.mark.gpu

# V is fp32; the GPU forms Gram-Schmidt from the 4x4 Gram matrix (LDL^T), which
# is exact in exact arithmetic but squares the conditioning of [out, g_1..g_r]
# in fp32: each component is held to 1e-4 of its own largest magnitude.
V_REL = 1e-4


def _check_V(Vg, Vr, name="V"):
    scale = np.abs(Vr).max(axis=-1, keepdims=True)
    err = np.abs(Vg - Vr)
    worst = float((err / np.maximum(scale, 1e-30)).max())
    assert worst <= V_REL, f"{name}: worst error / row max = {worst:.3e}"
    return worst


@pytest.mark.parametrize("T,C,kappa,dtype,seq", [
    (37, 264, (4, 8, 12), "bf16", None),
    (300, 2048, (4, 8, 12), "bf16", None),
    (64, 512, (4, 8, 12), "bf16", 20),
    (50, 128, (3,), "f32", None),
    (29, 256, (2, 5), "bf16", None),
    (40, 640, (1, 4, 7, 16), "f32", 9),
    (45, 768, (1, 4, 7, 16), "f32", 9),
    (70, 1024, (3, 9), "bf16", 33),
    (20, 512, (16, 16, 16, 16), "bf16", None),
])
def test_conv_gs_matches_oracle(T, C, kappa, dtype, seq):
    """r = 1..4, kappa up to 16, fp32 and bf16, tiles of 8 tokens with ragged ends,
    sequence restarts (seq)."""
    inp = synth.xhc_inputs(T, N=4, k=2, m=1, C=C, kappa=kappa, dtype=dtype, seed=500 + T + C)
    ws = [torch.from_numpy(w).cuda() for w in inp["conv_w"]]
    V = M.xhc_conv_gs(dev(inp["F"]), ws, seq_len=seq)
    torch.cuda.synchronize()
    ref = oracle.xhc_conv_gs(inp["F"], inp["conv_w"], seq_len=seq)
    _check_V(host(V), ref)


@pytest.mark.parametrize("C", [64, 256])
def test_conv_gs_zero_output_gives_zero_components(C):
    T = 9
    F = torch.zeros((T, C), dtype=torch.bfloat16, device="cuda")
    ws = [torch.randn(k, C, device="cuda") for k in (4, 8, 12)]
    V = M.xhc_conv_gs(F, ws)
    torch.cuda.synchronize()
    assert (V == 0).all()


def test_conv_gs_xhc_workload_sampled():
    """T=8192, C=2048, kappa {4, 8, 12}: 64 sampled tokens (with their 11-token halos)."""
    inp = synth.xhc_inputs(**synth.WORKLOADS["xhc"])
    ws = [torch.from_numpy(w).cuda() for w in inp["conv_w"]]
    V = host(M.xhc_conv_gs(dev(inp["F"]), ws))
    rng = np.random.default_rng(1)
    toks = np.unique(np.concatenate([[0, 1, 5, 11, 8191], rng.choice(8192, 59, replace=False)]))
    for t in toks:
        # the last row of a window of the 12 rows ending at t sees every tap of the
        # kappa = 12 conv, so it equals the full-sequence value (or starts at row 0)
        Fw = inp["F"][max(0, t - 11):t + 1]
        G = oracle.xhc_conv(Fw, inp["conv_w"])
        ref = oracle.xhc_gs(Fw[-1:], G[-1:])[0]
        _check_V(V[t][None], ref[None], f"V[{t}]")
    assert np.isfinite(V).all()


def _route_ref(inp):
    return oracle.xhc_route(inp["X"], inp["phi_read"], inp["alpha_read"], inp["b_read"], inp["k"], inp["m"])


def _update_case(inp, tokens=None, rt=None):
    """GPU sparse update on inputs whose idx, w and V come from the oracle; compares
    (all of, or the sampled `tokens` of) X_new, H_res, H_post."""
    from tests.parity import check_coeffs, check_mix
    T, N, C, k = inp["T"], inp["N"], inp["C"], inp["k"]
    rt = _route_ref(inp) if rt is None else rt
    V32 = oracle.xhc_conv_gs(inp["F"], inp["conv_w"]).astype(np.float32)
    w32 = rt["w"].astype(np.float32)
    Xd = dev(inp["X"])
    phiT = dev(np.ascontiguousarray(inp["phi_act"].T))
    _, Hr, Hp = M.xhc_sparse_update(Xd, torch.from_numpy(V32).cuda(), torch.from_numpy(rt["idx"]).cuda(),
                                    torch.from_numpy(w32).cuda(), phiT, inp["alpha_act"],
                                    torch.from_numpy(inp["b_act"]).cuda(), inp["t_iters"], inp["eps"])
    M.mhc_sync_status()
    sel = slice(None) if tokens is None else tokens
    X0 = oracle.widen(inp["X"][sel])
    ref, hr, hp = oracle.xhc_sparse_update(X0, V32[sel], rt["idx"][sel], w32[sel], inp["phi_act"],
                                          inp["alpha_act"], inp["b_act"], inp["t_iters"], inp["eps"])
    got = host(Xd)[sel]
    check_coeffs(host(Hr)[sel], hr, "H_res")
    check_coeffs(host(Hp)[sel], hp, "H_post")
    idx = rt["idx"][sel]
    for t in range(got.shape[0]):
        inactive = sorted(set(range(N)) - set(idx[t].tolist()))
        np.testing.assert_array_equal(got[t, inactive], X0[t, inactive])
        act = idx[t]
        absterms = (np.abs(X0[t, act]).sum(0)[None, :]
                    + np.abs(w32[sel][t])[:, None] * np.abs(V32[sel][t]).sum(0)[None, :])
        check_mix(got[t, act], ref[t, act], absterms, inp["dtype"], f"X_new[{t}]")


@pytest.mark.parametrize("T,N,k,m,C,dtype", [(37, 8, 4, 2, 128, "bf16"), (50, 6, 3, 1, 192, "f32"),
                                             (33, 16, 4, 2, 256, "bf16"), (20, 4, 2, 1, 64, "bf16")])
def test_sparse_update_matches_oracle(T, N, k, m, C, dtype):
    inp = synth.xhc_inputs(T, N=N, k=k, m=m, C=C, dtype=dtype, seed=600 + T + N)
    _update_case(inp)


def test_sparse_update_out_of_range_index_is_reported_and_token_untouched():
    T, N, k, C = 8, 8, 4, 64
    inp = synth.xhc_inputs(T, N=N, k=k, m=2, C=C, seed=7)
    idx = np.tile(np.array([0, 1, 2, 3], dtype=np.int32), (T, 1))
    idx[3, 2] = N + 5
    Xd = dev(inp["X"])
    X0 = host(Xd)
    V = torch.zeros((T, 4, C), device="cuda")
    M.xhc_sparse_update(Xd, V, torch.from_numpy(idx).cuda(), torch.ones((T, k), device="cuda"),
                        dev(np.ascontiguousarray(inp["phi_act"].T)), inp["alpha_act"],
                        torch.from_numpy(inp["b_act"]).cuda())
    with pytest.raises(M.MhcError) as e:
        M.mhc_sync_status()
    assert e.value.status == M.MHC_ERR_INVALID_ARG
    got = host(Xd)
    np.testing.assert_array_equal(got[3], X0[3])
    assert not np.array_equal(got[2], X0[2])
    M.mhc_sync_status()


@pytest.mark.parametrize("T,N,m,C,kappa", [(100, 16, 2, 512, (4, 8, 12)), (33, 8, 1, 1024, (4,)),
                                           (65, 6, 2, 512, (3, 5)), (1, 4, 0, 1536, (4, 8, 12)),
                                           (300, 16, 3, 2048, (2, 4, 6))])
def test_sparse_update_tensor_core_path_matches_oracle(T, N, m, C, kappa, update_path):
    """cp.async gather + TMA + tcgen05 projection for k = 4 active streams; Kr = 2, 3, 4;
    ragged last tile."""
    M.mhc_set_path(M.MHC_PATH_TENSOR)
    inp = synth.xhc_inputs(T, N=N, k=4, m=m, C=C, kappa=kappa, seed=800 + T + N + C)
    _update_case(inp)


def test_sparse_update_tensor_and_cuda_core_paths_agree(update_path):
    inp = synth.xhc_inputs(96, N=16, k=4, m=2, C=1024, seed=81)
    rt = _route_ref(inp)
    V = torch.from_numpy(oracle.xhc_conv_gs(inp["F"], inp["conv_w"]).astype(np.float32)).cuda()
    args = (V, torch.from_numpy(rt["idx"]).cuda(), torch.from_numpy(rt["w"].astype(np.float32)).cuda(),
            dev(np.ascontiguousarray(inp["phi_act"].T)), inp["alpha_act"], torch.from_numpy(inp["b_act"]).cuda(),
            inp["t_iters"], inp["eps"])
    outs = {}
    for path in (M.MHC_PATH_FMA, M.MHC_PATH_TENSOR):
        M.mhc_set_path(path)
        Xd = dev(inp["X"])
        _, Hr, Hp = M.xhc_sparse_update(Xd, *args)
        outs[path] = (host(Xd), host(Hr), host(Hp))
    a, t = outs[M.MHC_PATH_FMA], outs[M.MHC_PATH_TENSOR]
    assert np.abs(a[1] - t[1]).max() <= 2e-6 and np.abs(a[2] - t[2]).max() <= 2e-6
    # bf16 rows: equal up to a rounding flip where the fp32 sums differ in the last bits
    assert np.abs(a[0] - t[0]).max() <= 2 ** -6 * np.abs(a[0]).max()


def test_sparse_update_tensor_core_out_of_range_index_is_reported(update_path):
    M.mhc_set_path(M.MHC_PATH_TENSOR)
    T, N, k, C = 40, 8, 4, 512
    inp = synth.xhc_inputs(T, N=N, k=k, m=2, C=C, seed=17)
    idx = np.tile(np.array([0, 1, 2, 3], dtype=np.int32), (T, 1))
    idx[3, 2] = N + 5
    idx[35, 0] = -1
    Xd = dev(inp["X"])
    X0 = host(Xd)
    V = torch.zeros((T, 4, C), device="cuda")
    M.xhc_sparse_update(Xd, V, torch.from_numpy(idx).cuda(), torch.ones((T, k), device="cuda"),
                        dev(np.ascontiguousarray(inp["phi_act"].T)), inp["alpha_act"],
                        torch.from_numpy(inp["b_act"]).cuda())
    with pytest.raises(M.MhcError) as e:
        M.mhc_sync_status()
    assert e.value.status == M.MHC_ERR_INVALID_ARG
    got = host(Xd)
    np.testing.assert_array_equal(got[3], X0[3])
    np.testing.assert_array_equal(got[35], X0[35])
    assert not np.array_equal(got[2], X0[2])
    M.mhc_sync_status()


@pytest.fixture
def update_path():
    yield
    M.mhc_set_path(M.MHC_PATH_AUTO)


def test_sparse_update_xhc_workload_sampled():
    """T=8192, N=16, k=4 (m=2), C=2048 (the tensor-core path, as the benchmark runs
    it): the update runs on all tokens; 48 are compared."""
    inp, rt = xhc_full()
    rng = np.random.default_rng(2)
    toks = np.unique(np.concatenate([[0, 8191], rng.choice(8192, 46, replace=False)]))
    _update_case(inp, toks, rt)


def gapped(inp, gap=1e-4, max_rounds=30, with_route=False):
    """Redraw (from derived seeds) the X rows of tokens whose routed-score gap
    between the (k-m)-th and (k-m+1)-th highest score is <= gap (fp64 oracle),
    so that every TopK selection is decided well above rounding.  With
    with_route, also return the oracle's routing of the final inputs."""
    k, m, N = inp["k"], inp["m"], inp["N"]
    rows = np.arange(inp["T"])
    full = None
    for attempt in range(max_rounds + 1):
        out = oracle.xhc_route(inp["X"][rows], inp["phi_read"], inp["alpha_read"], inp["b_read"], k, m,
                               inp["eps"])
        if full is None:
            full = out
        else:
            for key in full:
                full[key][rows] = out[key]
        sc = out["score"]
        if k == m or k - m >= sc.shape[1]:
            break
        s = -np.sort(-sc, axis=1)
        bad = rows[(s[:, k - m - 1] - s[:, k - m]) <= gap]
        if bad.size == 0:
            break
        assert attempt < max_rounds, "could not separate the routing scores"
        synth.redraw_rows(inp["X"], bad, inp["seed"], attempt, inp["dtype"])
        rows = bad
    return (inp, full) if with_route else inp


_FULL = {}


def xhc_full():
    """The T=8192, N=16, k=4, m=2, C=2048 workload with separated scores, and its
    oracle routing (computed once per test session)."""
    if "v" not in _FULL:
        _FULL["v"] = gapped(synth.xhc_inputs(**synth.WORKLOADS["xhc"]), with_route=True)
    return _FULL["v"]


def _route_check(inp, tokens=None):
    from tests.parity import check_coeffs, check_mix
    k, m = inp["k"], inp["m"]
    x_in, Hp, sc, idx, w = M.xhc_route(dev(inp["X"]), dev(np.ascontiguousarray(inp["phi_read"].T)),
                                        inp["alpha_read"], torch.from_numpy(inp["b_read"]).cuda(), k, m,
                                        inp["eps"])
    torch.cuda.synchronize()
    sel = slice(None) if tokens is None else tokens
    ref = oracle.xhc_route(inp["X"][sel], inp["phi_read"], inp["alpha_read"], inp["b_read"], k, m, inp["eps"])
    np.testing.assert_array_equal(idx.cpu().numpy()[sel], ref["idx"])
    check_coeffs(host(Hp)[sel], ref["H_pre"], "H_pre")
    check_coeffs(host(sc)[sel], ref["score"], "score")
    check_coeffs(host(w)[sel], ref["w"], "w")
    X = oracle.widen(inp["X"][sel])
    check_mix(host(x_in)[sel], ref["x_in"], np.abs(X).sum(1), inp["dtype"], "x_in")


@pytest.mark.parametrize("T,N,k,m,C,dtype", [(41, 8, 4, 2, 128, "bf16"), (30, 16, 4, 2, 264, "bf16"),
                                             (25, 6, 3, 1, 64, "f32"), (20, 32, 8, 3, 64, "bf16"),
                                             (17, 5, 5, 2, 32, "bf16"), (16, 4, 2, 0, 64, "f32")])
def test_route_matches_oracle(T, N, k, m, C, dtype):
    inp = gapped(synth.xhc_inputs(T, N=N, k=k, m=m, C=C, dtype=dtype, seed=700 + T + N))
    _route_check(inp)


def test_route_ties_go_to_the_lower_index():
    T, N, k, m, C = 8, 8, 5, 2, 64
    inp = synth.xhc_inputs(T, N=N, k=k, m=m, C=C, seed=9)
    b = inp["b_read"].copy()
    b[N:] = 0.0                                          # every routed score sigma(0)
    _, _, sc, idx, w = M.xhc_route(dev(inp["X"]), dev(np.ascontiguousarray(inp["phi_read"].T)),
                                   [0.0, 0.0], torch.from_numpy(b).cuda(), k, m)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(idx.cpu().numpy(), np.tile(np.arange(k, dtype=np.int32), (T, 1)))
    np.testing.assert_allclose(w.cpu().numpy()[:, m:], 0.5)


@pytest.fixture
def route_path():
    yield
    M.mhc_set_path(M.MHC_PATH_AUTO)


@pytest.mark.parametrize("T,N,k,m,C", [(100, 16, 4, 2, 512), (33, 8, 4, 2, 1024), (65, 12, 5, 1, 512),
                                       (7, 4, 2, 0, 512), (300, 16, 8, 3, 2048), (40, 16, 2, 2, 512),
                                       (31, 8, 8, 2, 512), (1, 16, 4, 2, 1536)])
def test_route_tensor_core_path_matches_oracle(T, N, k, m, C, route_path):
    """TMA + tcgen05 route (groups of 4 streams, 32-token tiles): N = 4, 8, 12, 16;
    ragged last tile; m = 0; k = m (no routed pick); k = N (every stream active)."""
    M.mhc_set_path(M.MHC_PATH_TENSOR)
    inp = gapped(synth.xhc_inputs(T, N=N, k=k, m=m, C=C, seed=750 + T + N + C))
    _route_check(inp)


def test_route_tensor_and_cuda_core_paths_agree(route_path):
    inp = gapped(synth.xhc_inputs(200, N=16, k=4, m=2, C=1024, seed=77))
    Xd, phiT, b = dev(inp["X"]), dev(np.ascontiguousarray(inp["phi_read"].T)), torch.from_numpy(inp["b_read"]).cuda()
    outs = {}
    for path in (M.MHC_PATH_FMA, M.MHC_PATH_TENSOR):
        M.mhc_set_path(path)
        outs[path] = [host(t) for t in M.xhc_route(Xd, phiT, inp["alpha_read"], b, inp["k"], inp["m"], inp["eps"])]
    a, t = outs[M.MHC_PATH_FMA], outs[M.MHC_PATH_TENSOR]
    np.testing.assert_array_equal(a[3], t[3])                # idx
    for j, name in ((1, "H_pre"), (2, "score"), (4, "w")):
        assert np.abs(a[j] - t[j]).max() <= 2e-6, name


def test_route_tensor_core_ties_go_to_the_lower_index(route_path):
    M.mhc_set_path(M.MHC_PATH_TENSOR)
    T, N, k, m, C = 40, 16, 5, 2, 512
    inp = synth.xhc_inputs(T, N=N, k=k, m=m, C=C, seed=19)
    b = inp["b_read"].copy()
    b[N:] = 0.0                                          # every routed score sigma(0)
    _, _, sc, idx, w = M.xhc_route(dev(inp["X"]), dev(np.ascontiguousarray(inp["phi_read"].T)),
                                   [0.0, 0.0], torch.from_numpy(b).cuda(), k, m)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(idx.cpu().numpy(), np.tile(np.arange(k, dtype=np.int32), (T, 1)))
    np.testing.assert_allclose(w.cpu().numpy()[:, m:], 0.5)


def test_route_tensor_core_path_rejects_unsupported_calls(route_path):
    M.mhc_set_path(M.MHC_PATH_TENSOR)
    inp = synth.xhc_inputs(8, N=6, k=3, m=1, C=512, seed=20)       # N not a multiple of 4
    with pytest.raises(M.MhcError) as e:
        M.xhc_route(dev(inp["X"]), dev(np.ascontiguousarray(inp["phi_read"].T)), inp["alpha_read"],
                    torch.from_numpy(inp["b_read"]).cuda(), inp["k"], inp["m"])
    assert e.value.status == M.MHC_ERR_UNSUPPORTED


def test_route_xhc_workload_sampled():
    """T=8192, N=16, k=4, m=2, C=2048 (the tensor-core path, as the benchmark runs it):
    all tokens routed on the GPU, 64 sampled tokens compared (score gaps > 1e-4 after
    redrawing)."""
    inp, _ = xhc_full()
    rng = np.random.default_rng(3)
    toks = np.unique(np.concatenate([[0, 8191], rng.choice(8192, 62, replace=False)]))
    _route_check(inp, toks)
