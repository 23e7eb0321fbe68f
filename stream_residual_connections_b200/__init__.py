"""B200 (sm_100a) residual-stream mixing: mHC pre/post, xHC routing / conv +
Gram-Schmidt / sparse update, the mHC backward, and the HC (tanh) pre half with
the Amax Gain diagnostic.

This module is a thin binding over the C ABI of ``libmhc.so`` (declared in
``include/mhc.h``): it checks tensor devices, dtypes and contiguity, allocates
outputs with torch when the caller does not pass them, and forwards raw
device pointers and the current CUDA stream.  Every step of the computation
runs in the library's CUDA kernels; there is no CPU or PyTorch fallback, and
every call fails loudly (ImportError) if the library has not been built.

Names and arguments follow the C ABI one to one.
"""
from __future__ import annotations

import ctypes as ct
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmhc.so")

MHC_OK, MHC_ERR_INVALID_ARG, MHC_ERR_UNSUPPORTED, MHC_ERR_CUDA, MHC_ERR_TIMEOUT = range(5)
MHC_F32, MHC_BF16, MHC_TF32_PAIR = 0, 1, 2
MHC_PATH_AUTO, MHC_PATH_FMA, MHC_PATH_TENSOR = 0, 1, 2
_STATUS = {0: "MHC_OK", 1: "MHC_ERR_INVALID_ARG", 2: "MHC_ERR_UNSUPPORTED", 3: "MHC_ERR_CUDA",
           4: "MHC_ERR_TIMEOUT"}


class MhcError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{_STATUS.get(status, status)}: {message}")
        self.status = status


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"libmhc.so not built ({LIB_PATH}); run "
                          "`python -m stream_residual_connections_b200.build`")
    L = ct.CDLL(LIB_PATH)
    vp, i64, i32, f32 = ct.c_void_p, ct.c_int64, ct.c_int, ct.c_float
    fp = ct.POINTER(ct.c_float)
    L.mhc_last_error.restype = ct.c_char_p
    L.mhc_version.restype = ct.c_int
    L.mhc_pre.argtypes = [vp, i32, vp, i32, fp, vp, i64, i32, i32, i32, f32, vp, vp, vp, vp, vp]
    L.mhc_post.argtypes = [vp, vp, i32, vp, vp, i64, i32, i32, vp, vp]
    L.mhc_sync_status.argtypes = [vp]
    L.mhc_set_path.argtypes = [i32]
    L.xhc_route.argtypes = [vp, i32, vp, fp, vp, i64, i32, i32, i32, i32, f32, vp, vp, vp, vp, vp, vp]
    L.mhc_backward_workspace_bytes.argtypes = [i64, i32, i32]
    L.mhc_backward_workspace_bytes.restype = ct.c_size_t
    L.mhc_backward.argtypes = [vp, vp, vp, i32, fp, vp, vp, vp, i64, i32, i32, i32, f32, vp, vp, vp, vp,
                               vp, vp, ct.c_size_t, vp]
    L.mhc_backward_noalloc.argtypes = [vp, vp, vp, i32, fp, vp, vp, vp, i64, i32, i32, i32, f32, vp, vp,
                                       vp, vp, vp, vp]
    L.xhc_conv_gs.argtypes = [vp, i32, vp, ct.POINTER(ct.c_int), i32, i64, i32, i64, vp, vp]
    L.xhc_sparse_update.argtypes = [vp, i32, vp, i32, vp, vp, vp, fp, vp, i64, i32, i32, i32, i32,
                                    f32, vp, vp, vp]
    L.mhc_set_wait_limit.argtypes = [ct.c_longlong]
    L.hc_pre.argtypes = [vp, i32, vp, i32, fp, vp, i64, i32, i32, f32, vp, vp, vp, vp, vp]
    L.mhc_amax_gain.argtypes = [vp, i32, i64, i32, vp, vp, vp]
    L.mhc_phi_tf32_pair.argtypes = [vp, i32, i32, vp, vp]
    L.mhc_phi_tf32_pair_bytes.argtypes = [i32, i32]
    L.mhc_phi_tf32_pair_bytes.restype = ct.c_size_t
    for name in ("mhc_pre", "mhc_post", "mhc_sync_status", "mhc_set_path", "mhc_set_wait_limit",
                 "xhc_conv_gs", "xhc_sparse_update", "xhc_route", "mhc_backward",
                 "mhc_backward_noalloc", "hc_pre", "mhc_amax_gain", "mhc_phi_tf32_pair"):
        getattr(L, name).restype = ct.c_int
    return L


_lib = None


def native():
    """The loaded libmhc.so (ctypes.CDLL).  Raises ImportError if it is not built."""
    global _lib
    if _lib is None:
        _lib = _load()
    return _lib


def _check(status: int) -> None:
    if status != MHC_OK:
        raise MhcError(status, native().mhc_last_error().decode())


def _dt(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return MHC_BF16
    if t.dtype == torch.float32:
        return MHC_F32
    raise TypeError(f"unsupported dtype {t.dtype}")


def _ptr(t):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("tensors must live on a CUDA device")
    if not t.is_contiguous():
        raise ValueError("tensors must be contiguous")
    return ct.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ct.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _host3(alpha, count=3):
    vals = [float(v) for v in (alpha.tolist() if hasattr(alpha, "tolist") else alpha)]
    if len(vals) != count:
        raise ValueError(f"alpha must have {count} values")
    return (ct.c_float * count)(*vals)


def mhc_phi_tf32_pair(phi, n: int, *, pair=None, stream=None):
    """The tf32 projection (the pages' Eq.10 dtype) as its exact bf16 pair, the phi
    operand of mhc_pre(..., phi_tf32_pair=True).  phi: fp32 phi^T [n^2+2n][nC]; every
    element is rounded to tf32 first.  Returns the pair [2*RH][nC] bf16."""
    P, K = phi.shape
    if phi.dtype != torch.float32 or P != n * n + 2 * n or K % n:
        raise ValueError("phi must be fp32 [n^2+2n][n*C]")
    C = K // n
    RH = (P + 15) // 16 * 16
    if pair is None:
        pair = torch.empty((2 * RH, K), dtype=torch.bfloat16, device=phi.device)
    _check(native().mhc_phi_tf32_pair(_ptr(phi), n, C, _ptr(pair), _stream(stream)))
    return pair


def mhc_pre(X, phi, alpha, b, t_iters: int = 20, eps: float = 1e-6, *, x_in=None, H_pre=None,
            H_post=None, H_res=None, want_H_pre: bool = True, phi_tf32_pair: bool = False, stream=None):
    """Pre half of one mHC sublayer (see include/mhc.h).  X [T][n][C], phi [n^2+2n][nC]
    (the projection stored transposed, like a linear layer's weight), or with
    phi_tf32_pair=True the pair from mhc_phi_tf32_pair; alpha: 3 host floats,
    b [n^2+2n] fp32.  Returns (x_in, H_pre, H_post, H_res)."""
    T, n, C = X.shape
    dev = X.device
    if x_in is None:
        x_in = torch.empty((T, C), dtype=X.dtype, device=dev)
    if H_pre is None and want_H_pre:
        H_pre = torch.empty((T, n), dtype=torch.float32, device=dev)
    if H_post is None:
        H_post = torch.empty((T, n), dtype=torch.float32, device=dev)
    if H_res is None:
        H_res = torch.empty((T, n, n), dtype=torch.float32, device=dev)
    pdt = MHC_TF32_PAIR if phi_tf32_pair else _dt(phi)
    _check(native().mhc_pre(_ptr(X), _dt(X), _ptr(phi), pdt, _host3(alpha), _ptr(b), T, n, C,
                       int(t_iters), float(eps), _ptr(x_in), _ptr(H_pre), _ptr(H_post),
                       _ptr(H_res), _stream(stream)))
    return x_in, H_pre, H_post, H_res


def hc_pre(X, theta, alpha, b, eps: float = 1e-6, *, x_in=None, H_pre=None, H_post=None, H_res=None,
           want_H_pre: bool = True, stream=None):
    """Pre half of one sublayer with the HC (tanh) coefficients (see include/mhc.h).
    X [T][n][C], theta [n+2][C] (rows pre, post, res_0..res_{n-1}), alpha: 3 host
    floats, b [n^2+2n] fp32.  Returns (x_in, H_pre, H_post, H_res); the post half is
    mhc_post."""
    T, n, C = X.shape
    dev = X.device
    if x_in is None:
        x_in = torch.empty((T, C), dtype=X.dtype, device=dev)
    if H_pre is None and want_H_pre:
        H_pre = torch.empty((T, n), dtype=torch.float32, device=dev)
    if H_post is None:
        H_post = torch.empty((T, n), dtype=torch.float32, device=dev)
    if H_res is None:
        H_res = torch.empty((T, n, n), dtype=torch.float32, device=dev)
    _check(native().hc_pre(_ptr(X), _dt(X), _ptr(theta), _dt(theta), _host3(alpha), _ptr(b), T, n, C,
                           float(eps), _ptr(x_in), _ptr(H_pre), _ptr(H_post), _ptr(H_res), _stream(stream)))
    return x_in, H_pre, H_post, H_res


def mhc_amax_gain(H_res, *, gain=None, gain_max=None, want_gain: bool = True, stream=None):
    """Amax Gain Magnitude of the composite maps H_res[d-1]..H_res[0], d = 1..L (see
    include/mhc.h).  H_res [L][T][n][n] fp32.  Returns (gain [L][T][2] or None,
    gain_max [L][2]): (forward, backward) = largest absolute row / column sum."""
    Lz, T, n, n2 = H_res.shape
    if n != n2 or H_res.dtype != torch.float32:
        raise ValueError("H_res must be fp32 [L][T][n][n]")
    if gain is None and want_gain:
        gain = torch.empty((Lz, T, 2), dtype=torch.float32, device=H_res.device)
    if gain_max is None:
        gain_max = torch.empty((Lz, 2), dtype=torch.float32, device=H_res.device)
    _check(native().mhc_amax_gain(_ptr(H_res), Lz, T, n, _ptr(gain), _ptr(gain_max), _stream(stream)))
    return gain, gain_max


def mhc_post(X, F_out, H_post, H_res, *, X_next=None, stream=None):
    """Post half: X_next = H_res X + H_post^T F_out.  Pass X_next=X for in place."""
    T, n, C = X.shape
    if X_next is None:
        X_next = torch.empty_like(X)
    if F_out.dtype != X.dtype:
        raise TypeError("X and F_out must share a dtype")
    _check(native().mhc_post(_ptr(X), _ptr(F_out), _dt(X), _ptr(H_post), _ptr(H_res), T, n, C,
                        _ptr(X_next), _stream(stream)))
    return X_next


def mhc_sync_status(stream=None) -> None:
    """Wait for the stream; raise MhcError(MHC_ERR_TIMEOUT) if a bounded wait expired."""
    _check(native().mhc_sync_status(_stream(stream)))


def mhc_set_path(path: int) -> None:
    """Process-wide mhc_pre projection kernel: MHC_PATH_AUTO / _FMA / _TENSOR."""
    _check(native().mhc_set_path(int(path)))


def mhc_set_wait_limit(polls: int) -> None:
    """Polls before a bounded on-device wait gives up (tests of the timeout path)."""
    _check(native().mhc_set_wait_limit(int(polls)))


def xhc_conv_gs(F_out, conv_w, seq_len=None, *, V=None, stream=None):
    """Causal depthwise convolutions + Gram-Schmidt (see include/mhc.h).
    F_out [T][C]; conv_w: a list of r fp32 weight tensors [kappa_j][C] or one
    concatenated tensor with `kappa` given as conv_w[1].  Returns V [T][r+1][C] fp32."""
    if isinstance(conv_w, (list, tuple)) and all(hasattr(w, "shape") for w in conv_w):
        kappa = [int(w.shape[0]) for w in conv_w]
        wcat = torch.cat([w.reshape(-1) for w in conv_w]).contiguous()
    else:
        wcat, kappa = conv_w
    T, C = F_out.shape
    r = len(kappa)
    if V is None:
        V = torch.empty((T, r + 1, C), dtype=torch.float32, device=F_out.device)
    ka = (ct.c_int * r)(*kappa)
    _check(native().xhc_conv_gs(_ptr(F_out), _dt(F_out), _ptr(wcat), ka, r, T, C,
                                int(seq_len or max(T, 1)), _ptr(V), _stream(stream)))
    return V


def xhc_sparse_update(X, V, idx, w, phi_act, alpha_act, b_act, t_iters: int = 20, eps: float = 1e-6,
                      *, H_res=None, H_post=None, want_coeffs: bool = True, stream=None):
    """Sparse k x k update + scatter, in place on X [T][N][C] (see include/mhc.h).
    phi_act is [k*k + k*Kr][k*C] (transposed).  Returns (X, H_res, H_post)."""
    T, N, C = X.shape
    k = idx.shape[1]
    Kr = V.shape[1]
    if want_coeffs:
        if H_res is None:
            H_res = torch.empty((T, k, k), dtype=torch.float32, device=X.device)
        if H_post is None:
            H_post = torch.empty((T, k, Kr), dtype=torch.float32, device=X.device)
    _check(native().xhc_sparse_update(_ptr(X), _dt(X), _ptr(V), Kr, _ptr(idx), _ptr(w), _ptr(phi_act),
                                      _host3(alpha_act, 2), _ptr(b_act), T, N, C, k, int(t_iters),
                                      float(eps), _ptr(H_res), _ptr(H_post), _stream(stream)))
    return X, H_res, H_post


def xhc_route(X, phi_read, alpha_read, b_read, k: int, m: int, eps: float = 1e-6, *, x_in=None,
              H_pre=None, score=None, idx=None, w=None, want_scores: bool = True, stream=None):
    """Routing + dense read (see include/mhc.h).  X [T][N][C]; phi_read [2N-m][N*C]
    (transposed).  Returns (x_in, H_pre, score, idx, w)."""
    T, N, C = X.shape
    dev = X.device
    if x_in is None:
        x_in = torch.empty((T, C), dtype=X.dtype, device=dev)
    if want_scores:
        if H_pre is None:
            H_pre = torch.empty((T, N), dtype=torch.float32, device=dev)
        if score is None:
            score = torch.empty((T, max(N - m, 1)), dtype=torch.float32, device=dev)
    if idx is None:
        idx = torch.empty((T, k), dtype=torch.int32, device=dev)
    if w is None:
        w = torch.empty((T, k), dtype=torch.float32, device=dev)
    _check(native().xhc_route(_ptr(X), _dt(X), _ptr(phi_read), _host3(alpha_read, 2), _ptr(b_read), T, N,
                              C, int(k), int(m), float(eps), _ptr(x_in), _ptr(H_pre), _ptr(score),
                              _ptr(idx), _ptr(w), _stream(stream)))
    return x_in, H_pre, score, idx, w


def mhc_backward_workspace_bytes(T: int, n: int, C: int) -> int:
    return int(native().mhc_backward_workspace_bytes(int(T), int(n), int(C)))


def mhc_backward(X, F_out, phi, alpha, b, dX_next, dx_in, t_iters: int = 20, eps: float = 1e-6, *,
                 dX=None, dF=None, dphi=None, dalpha=None, db=None, workspace=None, stream=None):
    """Gradients of one mHC sublayer (see include/mhc.h).  phi is [P][nC] (transposed).
    Returns (dX, dF, dphi [P][nC] fp32, dalpha [3], db [P])."""
    T, n, C = X.shape
    P = n * n + 2 * n
    dev = X.device
    dX = torch.empty_like(X) if dX is None else dX
    dF = torch.empty_like(F_out) if dF is None else dF
    dphi = torch.empty((P, n * C), dtype=torch.float32, device=dev) if dphi is None else dphi
    dalpha = torch.empty(3, dtype=torch.float32, device=dev) if dalpha is None else dalpha
    db = torch.empty(P, dtype=torch.float32, device=dev) if db is None else db
    need = mhc_backward_workspace_bytes(T, n, C)
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=dev)
    _check(native().mhc_backward(_ptr(X), _ptr(F_out), _ptr(phi), _dt(X), _host3(alpha), _ptr(b),
                                 _ptr(dX_next), _ptr(dx_in), T, n, C, int(t_iters), float(eps), _ptr(dX),
                                 _ptr(dF), _ptr(dphi), _ptr(dalpha), _ptr(db), ct.c_void_p(workspace.data_ptr()),
                                 workspace.numel() * workspace.element_size(), _stream(stream)))
    return dX, dF, dphi, dalpha, db


def mhc_backward_noalloc(X, F_out, phi, alpha, b, dX_next, dx_in, t_iters: int = 20, eps: float = 1e-6,
                         *, dX, dF, dphi, dalpha, db, stream=None):
    """mhc_backward using the library's built-in scratch instead of a workspace, for
    callers that cannot allocate (e.g. during CUDA graph capture).  All outputs are
    caller-provided; see include/mhc.h for the size limit and the sharing rules."""
    T, n, C = X.shape
    _check(native().mhc_backward_noalloc(_ptr(X), _ptr(F_out), _ptr(phi), _dt(X), _host3(alpha), _ptr(b),
                                         _ptr(dX_next), _ptr(dx_in), T, n, C, int(t_iters), float(eps),
                                         _ptr(dX), _ptr(dF), _ptr(dphi), _ptr(dalpha), _ptr(db),
                                         _stream(stream)))
    return dX, dF, dphi, dalpha, db
