"""CPU checks of the C ABI: the library loads, exports every function that
include/*.h declares, and rejects bad arguments on the host before any launch
(no CUDA call is made by these tests)."""
from __future__ import annotations

import ctypes as ct
import glob
import os
import re
import subprocess

import pytest

import stream_residual_connections_b200 as M

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        src = open(h).read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        for m in re.finditer(r"^\s*[A-Za-z_][\w\s\*]*?\b(\w+)\s*\(", src, flags=re.M):
            name = m.group(1)
            if name not in ("if", "while", "for", "return", "sizeof"):
                names.add(name)
    return sorted(names)


def test_header_declares_the_api():
    names = _declared()
    for expected in ("mhc_pre", "mhc_post", "mhc_last_error", "mhc_sync_status"):
        assert expected in names


def test_library_exports_every_declared_symbol():
    lib = M.native()
    out = subprocess.check_output(["nm", "-D", "--defined-only", M.LIB_PATH], text=True)
    exported = {line.split()[-1] for line in out.splitlines() if line.strip()}
    missing = [n for n in _declared() if n not in exported]
    assert not missing, missing
    for n in _declared():
        getattr(lib, n)  # resolvable through ctypes too


def _fake(addr=0x10000):
    return ct.c_void_p(addr)


def _pre(**kw):
    args = dict(X=_fake(0x100000), x_dt=M.MHC_BF16, phi=_fake(0x200000), phi_dt=M.MHC_BF16,
                alpha=(ct.c_float * 3)(0.01, 0.01, 0.01), b=_fake(0x300000), T=16, n=4, C=64,
                t_iters=20, eps=1e-6, x_in=_fake(0x400000), H_pre=_fake(0x500000),
                H_post=_fake(0x600000), H_res=_fake(0x700000), stream=None)
    args.update(kw)
    return M.native().mhc_pre(*args.values())


@pytest.mark.parametrize("kw,code", [
    (dict(n=0), M.MHC_ERR_INVALID_ARG),
    (dict(n=9), M.MHC_ERR_INVALID_ARG),
    (dict(C=12), M.MHC_ERR_INVALID_ARG),
    (dict(C=0), M.MHC_ERR_INVALID_ARG),
    (dict(T=-1), M.MHC_ERR_INVALID_ARG),
    (dict(t_iters=-1), M.MHC_ERR_INVALID_ARG),
    (dict(eps=-1.0), M.MHC_ERR_INVALID_ARG),
    (dict(alpha=None), M.MHC_ERR_INVALID_ARG),
    (dict(x_dt=7), M.MHC_ERR_INVALID_ARG),
    (dict(X=None), M.MHC_ERR_INVALID_ARG),
    (dict(X=_fake(0x100004)), M.MHC_ERR_INVALID_ARG),
    (dict(H_post=None), M.MHC_ERR_INVALID_ARG),
    (dict(x_in=_fake(0x100000)), M.MHC_ERR_INVALID_ARG),          # x_in aliases X
    (dict(H_res=_fake(0x600000)), M.MHC_ERR_INVALID_ARG),         # outputs overlap
    (dict(x_dt=M.MHC_F32, phi_dt=M.MHC_BF16), M.MHC_ERR_UNSUPPORTED),
])
def test_mhc_pre_rejects_bad_arguments_on_host(kw, code):
    assert _pre(**kw) == code
    assert M.native().mhc_last_error().decode()


def test_mhc_pre_empty_is_a_no_op():
    assert _pre(T=0, X=None, x_in=None) == M.MHC_OK


def _post(**kw):
    args = dict(X=_fake(0x100000), F=_fake(0x200000), dt=M.MHC_BF16, H_post=_fake(0x300000),
                H_res=_fake(0x400000), T=8, n=4, C=64, X_next=_fake(0x800000), stream=None)
    args.update(kw)
    return M.native().mhc_post(*args.values())


@pytest.mark.parametrize("kw,code", [
    (dict(n=9), M.MHC_ERR_INVALID_ARG),
    (dict(C=4), M.MHC_ERR_INVALID_ARG),
    (dict(F=None), M.MHC_ERR_INVALID_ARG),
    (dict(X_next=_fake(0x100010)), M.MHC_ERR_INVALID_ARG),        # partial overlap with X
    (dict(X_next=_fake(0x200000)), M.MHC_ERR_INVALID_ARG),        # X_next over F_out
    (dict(dt=5), M.MHC_ERR_INVALID_ARG),
])
def test_mhc_post_rejects_bad_arguments_on_host(kw, code):
    assert _post(**kw) == code


def test_mhc_post_empty_is_a_no_op():
    assert _post(T=0) == M.MHC_OK


def test_binding_requires_cuda_tensors():
    import torch
    X = torch.zeros(2, 4, 8, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        M.mhc_post(X, torch.zeros(2, 8, dtype=torch.bfloat16), torch.zeros(2, 4),
                   torch.zeros(2, 4, 4), X_next=X)


def _hc(**kw):
    args = dict(X=_fake(0x100000), x_dt=M.MHC_BF16, theta=_fake(0x200000), t_dt=M.MHC_BF16,
                alpha=(ct.c_float * 3)(0.5, 0.5, 0.5), b=_fake(0x300000), T=16, n=4, C=64, eps=1e-6,
                x_in=_fake(0x400000), H_pre=_fake(0x500000), H_post=_fake(0x600000), H_res=_fake(0x700000),
                stream=None)
    args.update(kw)
    return M.native().hc_pre(*args.values())


@pytest.mark.parametrize("kw,code", [
    (dict(n=0), M.MHC_ERR_INVALID_ARG),
    (dict(n=9), M.MHC_ERR_INVALID_ARG),
    (dict(C=12), M.MHC_ERR_INVALID_ARG),
    (dict(T=-1), M.MHC_ERR_INVALID_ARG),
    (dict(eps=-1.0), M.MHC_ERR_INVALID_ARG),
    (dict(alpha=None), M.MHC_ERR_INVALID_ARG),
    (dict(t_dt=M.MHC_TF32_PAIR), M.MHC_ERR_INVALID_ARG),
    (dict(theta=None), M.MHC_ERR_INVALID_ARG),
    (dict(H_pre=_fake(0x500004)), M.MHC_ERR_INVALID_ARG),
    (dict(x_in=_fake(0x200000)), M.MHC_ERR_INVALID_ARG),          # x_in over theta
    (dict(x_dt=M.MHC_F32, t_dt=M.MHC_BF16), M.MHC_ERR_UNSUPPORTED),
])
def test_hc_pre_rejects_bad_arguments_on_host(kw, code):
    assert _hc(**kw) == code
    assert M.native().mhc_last_error().decode()


def test_hc_pre_empty_is_a_no_op():
    assert _hc(T=0, X=None, x_in=None) == M.MHC_OK


def _amax(**kw):
    args = dict(H=_fake(0x100000), L=4, T=16, n=4, gain=_fake(0x200000), gain_max=_fake(0x300000), stream=None)
    args.update(kw)
    return M.native().mhc_amax_gain(*args.values())


@pytest.mark.parametrize("kw,code", [
    (dict(n=0), M.MHC_ERR_INVALID_ARG),
    (dict(n=9), M.MHC_ERR_INVALID_ARG),
    (dict(L=-1), M.MHC_ERR_INVALID_ARG),
    (dict(T=-2), M.MHC_ERR_INVALID_ARG),
    (dict(gain=None, gain_max=None), M.MHC_ERR_INVALID_ARG),
    (dict(H=None), M.MHC_ERR_INVALID_ARG),
    (dict(gain_max=_fake(0x300004)), M.MHC_ERR_INVALID_ARG),
])
def test_mhc_amax_gain_rejects_bad_arguments_on_host(kw, code):
    assert _amax(**kw) == code


def test_mhc_amax_gain_no_layers_is_a_no_op():
    assert _amax(L=0, H=None) == M.MHC_OK


@pytest.mark.parametrize("n,C,code", [(0, 64, M.MHC_ERR_INVALID_ARG), (9, 64, M.MHC_ERR_INVALID_ARG),
                                      (4, 12, M.MHC_ERR_INVALID_ARG)])
def test_mhc_phi_tf32_pair_rejects_bad_arguments_on_host(n, C, code):
    assert M.native().mhc_phi_tf32_pair(_fake(0x100000), n, C, _fake(0x900000), None) == code


def test_tf32_pair_bytes_and_pre_rules():
    # RH = P rounded up to 16; the pair holds 2 RH rows of n C bf16
    assert M.native().mhc_phi_tf32_pair_bytes(4, 512) == 2 * 32 * 4 * 512 * 2
    assert M.native().mhc_phi_tf32_pair_bytes(8, 512) == 2 * 80 * 8 * 512 * 2
    assert M.native().mhc_phi_tf32_pair_bytes(0, 512) == 0
    # the pair needs bf16 X; it is not a dtype for X itself
    assert _pre(x_dt=M.MHC_F32, phi_dt=M.MHC_TF32_PAIR) == M.MHC_ERR_UNSUPPORTED
    assert _pre(x_dt=M.MHC_TF32_PAIR) == M.MHC_ERR_INVALID_ARG
