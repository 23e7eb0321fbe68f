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
])
def test_conv_gs_matches_oracle(T, C, kappa, dtype, seq):
    inp = synth.xhc_inputs(T, N=4, k=2, m=1, C=C, kappa=kappa, dtype=dtype, seed=500 + T + C)
    ws = [torch.from_numpy(w).cuda() for w in inp["conv_w"]]
    V = M.xhc_conv_gs(dev(inp["F"]), ws, seq_len=seq)
    torch.cuda.synchronize()
    ref = oracle.xhc_conv_gs(inp["F"], inp["conv_w"], seq_len=seq)
    _check_V(host(V), ref)


def test_conv_gs_zero_output_gives_zero_components():
    T, C = 9, 64
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
