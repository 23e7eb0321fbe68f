"""Pins of the oracle's reverse mode (mHC page section 4.3.1: the backward
through the projection and through every Sinkhorn iteration).

Two independent checks: central finite differences of the oracle's own
forward, and torch float64 autograd of a direct restatement of the forward.
"""
from __future__ import annotations

import math

import numpy as np
import torch

import oracle


def _case(T=4, n=4, C=32, seed=21):
    rng = np.random.default_rng(seed)
    P = n * n + 2 * n
    X = rng.normal(size=(T, n, C))
    F = rng.normal(size=(T, C))
    phi = rng.normal(size=(n * C, P)) / math.sqrt(n * C)
    b = rng.normal(size=P) * 0.3
    b[2 * n:] += (1.0 * np.eye(n)).reshape(-1)
    a = np.array([0.7, -0.5, 1.1])   # gates large enough that every path matters
    gXn = rng.normal(size=(T, n, C))
    gxi = rng.normal(size=(T, C))
    return X, F, phi, a, b, gXn, gxi


def _loss(X, F, phi, a, b, gXn, gxi):
    co = oracle.mhc_forward(X, F, phi, a, b)
    return float((co["X_next"] * gXn).sum() + (co["x_in"] * gxi).sum())


def test_backward_matches_central_finite_differences():
    """T=4, C=32, n=4, h=1e-6: relative error <= 1e-6 on X, F_out, phi, alpha, b."""
    X, F, phi, a, b, gXn, gxi = _case()
    g = oracle.mhc_backward(X, F, phi, a, b, gXn, gxi)
    rng = np.random.default_rng(5)
    h = 1e-6
    args = dict(X=X, F=F, phi=phi, a=a, b=b)
    grads = dict(X=g["dX"], F=g["dF"], phi=g["dphi"], a=g["dalpha"], b=g["db"])
    for name, arr in args.items():
        flat = arr.reshape(-1)
        picks = rng.choice(flat.size, size=min(flat.size, 40), replace=False)
        for q in picks:
            old = flat[q]
            flat[q] = old + h
            lp = _loss(**args, gXn=gXn, gxi=gxi)
            flat[q] = old - h
            lm = _loss(**args, gXn=gXn, gxi=gxi)
            flat[q] = old
            fd = (lp - lm) / (2 * h)
            an = grads[name].reshape(-1)[q]
            assert abs(fd - an) <= 1e-6 * max(1.0, abs(an)), (name, q, fd, an)


def _torch_forward(X, F, phi, a, b, t_iters=20, eps=1e-6):
    """The forward restated with torch float64 ops (Eq.(3), (7)-(9))."""
    T, n, C = X.shape
    x = X.reshape(T, n * C)
    r = torch.sqrt((x * x).mean(1, keepdim=True) + eps)
    d = (x / r) @ phi
    aseg = torch.cat([a[0].expand(n), a[1].expand(n), a[2].expand(n * n)])
    z = aseg * d + b
    hpre = torch.sigmoid(z[:, :n])
    hpost = 2 * torch.sigmoid(z[:, n:2 * n])
    M = torch.exp(z[:, 2 * n:].reshape(T, n, n))
    for _ in range(t_iters):
        M = M / M.sum(1, keepdim=True)
        M = M / M.sum(2, keepdim=True)
    x_in = torch.einsum("ti,tic->tc", hpre, X)
    Xn = torch.einsum("tij,tjc->tic", M, X) + hpost[:, :, None] * F[:, None, :]
    return x_in, Xn


def test_backward_matches_torch_autograd():
    X, F, phi, a, b, gXn, gxi = _case(T=6, n=4, C=24, seed=22)
    g = oracle.mhc_backward(X, F, phi, a, b, gXn, gxi)
    tX, tF, tphi, ta, tb = (torch.tensor(v, dtype=torch.float64, requires_grad=True)
                            for v in (X, F, phi, a, b))
    x_in, Xn = _torch_forward(tX, tF, tphi, ta, tb)
    loss = (Xn * torch.tensor(gXn)).sum() + (x_in * torch.tensor(gxi)).sum()
    loss.backward()
    for mine, ref in ((g["dX"], tX.grad), (g["dF"], tF.grad), (g["dphi"], tphi.grad),
                      (g["dalpha"], ta.grad), (g["db"], tb.grad)):
        np.testing.assert_allclose(mine, ref.numpy(), rtol=1e-10, atol=1e-12)


def test_backward_n2_and_n8():
    for n in (2, 8):
        X, F, phi, a, b, gXn, gxi = _case(T=2, n=n, C=8, seed=30 + n)
        g = oracle.mhc_backward(X, F, phi, a, b, gXn, gxi)
        tX, tF, tphi, ta, tb = (torch.tensor(v, dtype=torch.float64, requires_grad=True)
                                for v in (X, F, phi, a, b))
        x_in, Xn = _torch_forward(tX, tF, tphi, ta, tb)
        ((Xn * torch.tensor(gXn)).sum() + (x_in * torch.tensor(gxi)).sum()).backward()
        np.testing.assert_allclose(g["dX"], tX.grad.numpy(), rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(g["dphi"], tphi.grad.numpy(), rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(g["db"], tb.grad.numpy(), rtol=1e-10, atol=1e-12)
