"""B200 (sm_100a) RWKV-4 WKV operator: Python binding of the C ABI in ``include/wkv.h``.

This module only marshals arguments: it takes CUDA tensors, checks dtypes and
shapes, and passes raw device pointers and the current CUDA stream to
``libwkv_b200.so``.  Every step of the computation runs in the library's kernels;
there is no CPU fallback, and calling any function without the built library or
with CPU tensors raises.

Entry points (same names as the C ABI):

* ``wkv_forward(w, u, k, v, state_in=None, want_state=True, path="auto", chunk=0,
  workspace=None)`` -> ``(y, state_out)`` for k, v of shape [B, T, C]
  (fp32 or bf16; y has k's dtype; state_out is [3, B, C] fp32 or None).
* ``wkv_decode_step(w, u, k, v, state, y=None)`` -> ``y`` ([N, L, C]); updates
  ``state`` ([3, N, L, C]) in place.
* ``wkv_decode_step_fused(mu, w, u, x_t, x_prev, k, v, state, xbar=None, y=None)``
  -> ``(xbar, y)``.
* ``token_shift_mix(mu, x, x_last=None)`` -> ``xbar``.
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

from . import build as _build

__all__ = [
    "WkvError", "Workspace", "wkv_forward", "wkv_decode_step", "wkv_decode_step_fused", "token_shift_mix",
    "workspace_size", "forward_status", "auto_path", "lib", "LIB_PATH", "STATUS",
]

LIB_PATH = _build.LIB_PATH
STATUS = {0: "WKV_OK", 1: "WKV_ERR_INVALID_ARG", 2: "WKV_ERR_MISALIGNED", 3: "WKV_ERR_UNSUPPORTED",
          4: "WKV_ERR_CUDA", 5: "WKV_ERR_TIMEOUT"}
_DTYPE = {torch.float32: 0, torch.bfloat16: 1}
_PATH = {"auto": 0, "serial": 1, "chunked": 2}


class WkvError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {STATUS.get(status, status)}")


_lib = None
_lock = threading.Lock()


def lib():
    """Load (building first if needed) the CUDA library.  Raises if it cannot be built."""
    global _lib
    if _lib is None:
        with _lock:
            if _lib is None:
                if not os.path.exists(LIB_PATH) or not _build.up_to_date():
                    _build.build()
                L = ctypes.CDLL(LIB_PATH)
                i64, vp, sz, i32, u32 = ctypes.c_int64, ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int, ctypes.c_uint32
                L.wkv_forward.argtypes = [i64, i64, i64, i32, vp, vp, vp, vp, vp, vp, vp, sz, vp]
                L.wkv_forward_ex.argtypes = [i64, i64, i64, i32, vp, vp, vp, vp, vp, vp, vp, vp, sz, i32, i32, vp]
                L.wkv_forward_workspace_size.argtypes = [i64, i64, i64, i32]
                L.wkv_forward_workspace_size.restype = sz
                L.wkv_workspace_init.argtypes = [vp, sz, vp]
                L.wkv_forward_status.argtypes = [vp, sz, vp]
                L.wkv_get_device_status.argtypes = [vp]
                L.wkv_forward_gated.argtypes = [i64, i64, i64, i32, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, i32, i32, vp]
                L.token_shift_mix3.argtypes = [i64, i64, i64, vp, vp, vp, vp, vp, vp, vp, vp, vp]
                L.wkv_backward.argtypes = [i64, i64, i64] + [vp] * 10 + [sz, vp]
                L.wkv_backward_workspace_size.argtypes = [i64, i64, i64]
                L.wkv_backward_workspace_size.restype = sz
                L.wkv_decode_step.argtypes = [i64, i64, i64, vp, vp, vp, vp, vp, vp, vp]
                L.eagle_forward.argtypes = [i64, i64, i64] + [vp] * 8 + [sz, vp]
                L.eagle_forward_workspace_size.argtypes = [i64, i64, i64]
                L.eagle_forward_workspace_size.restype = sz
                L.eagle_forward_launches.argtypes = [i64, i64, i64]
                L.eagle_forward_launches.restype = i32
                L.eagle_decode_step.argtypes = [i64, i64, i64] + [vp] * 7
                L.wkv_decode_step_fused.argtypes = [i64, i64, i64, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp]
                L.token_shift_mix.argtypes = [i64, i64, i64, vp, vp, vp, vp, vp]
                L.wkv_status_string.argtypes = [i32]
                L.wkv_status_string.restype = ctypes.c_char_p
                L.wkv_forward_auto_path.argtypes = [i64, i64, i64, i32]
                L.wkv_testhook_forward_drop.argtypes = [i64, i64, i64, vp, vp, vp, vp, vp, vp, sz, i64, u32, vp]
                for f in (L.wkv_forward, L.wkv_forward_ex, L.wkv_workspace_init, L.wkv_forward_status,
                          L.wkv_get_device_status, L.wkv_forward_gated, L.token_shift_mix3, L.wkv_backward,
                          L.wkv_decode_step, L.wkv_decode_step_fused, L.token_shift_mix,
                          L.wkv_forward_auto_path, L.wkv_testhook_forward_drop):
                    f.restype = i32
                _lib = L
    return _lib


def _ptr(t):
    return None if t is None else t.data_ptr()


def _stream(dev):
    return torch.cuda.current_stream(dev).cuda_stream


def _check(status, what):
    if status != 0:
        raise WkvError(status, what)


def _cuda_f32(t, name, shape=None):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor (no CPU path exists)")
    if t.dtype != torch.float32:
        raise TypeError(f"{name} must be float32, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    return t


def workspace_size(B, T, C, dtype=torch.float32) -> int:
    return int(lib().wkv_forward_workspace_size(B, T, C, _DTYPE[dtype]))


def auto_path(B, T, C, dtype=torch.float32) -> str:
    return {1: "serial", 2: "chunked"}[int(lib().wkv_forward_auto_path(B, T, C, _DTYPE[dtype]))]


class Workspace:
    """Caller-owned scratch for the chunked forward: a zero-filled uint8 CUDA tensor
    that grows on demand.  One workspace must not serve two forwards that can run
    concurrently on the GPU."""

    def __init__(self, device=None, nbytes: int = 0):
        self.device = torch.device(device or "cuda")
        self.buf = None
        if nbytes:
            self.ensure(nbytes)

    def ensure(self, nbytes: int):
        if self.buf is None or self.buf.numel() < nbytes:
            self.buf = torch.empty(max(nbytes, 64), dtype=torch.uint8, device=self.device)
            _check(lib().wkv_workspace_init(self.buf.data_ptr(), self.buf.numel(), _stream(self.device)),
                   "wkv_workspace_init")
        return self.buf

    def for_shape(self, B, T, C, dtype):
        return self.ensure(workspace_size(B, T, C, dtype))


_default_ws = {}


def _workspace_for(dev, B, T, C, dtype):
    key = (dev.index, torch.cuda.current_stream(dev).cuda_stream)
    ws = _default_ws.get(key)
    if ws is None:
        ws = _default_ws[key] = Workspace(dev)
    return ws.for_shape(B, T, C, dtype)


def wkv_forward(w, u, k, v, state_in=None, want_state=True, path="auto", chunk=0, workspace=None, y=None,
                state_out=None, r=None):
    """Forward over [B, T, C].  Returns (y, state_out).  With r ([B, T, C], k's dtype) y is the
    gated output sigma(r) * wkv (wkv_forward_gated)."""
    if not isinstance(k, torch.Tensor) or not k.is_cuda:
        raise TypeError("k must be a CUDA tensor (no CPU path exists)")
    if k.dtype not in _DTYPE or v.dtype != k.dtype:
        raise TypeError("k and v must both be float32 or both bfloat16")
    if k.dim() != 3 or v.shape != k.shape or not k.is_contiguous() or not v.is_contiguous():
        raise ValueError("k, v must be contiguous [B, T, C] tensors of the same shape")
    B, T, C = k.shape
    dev = k.device
    _cuda_f32(w, "w", (C,))
    _cuda_f32(u, "u", (C,))
    if state_in is not None:
        _cuda_f32(state_in, "state_in", (3, B, C))
    if y is None:
        y = torch.empty_like(k)
    if want_state and state_out is None:
        state_out = torch.empty((3, B, C), dtype=torch.float32, device=dev)
    if not want_state:
        state_out = None
    ws = workspace.for_shape(B, T, C, k.dtype) if isinstance(workspace, Workspace) else (
        workspace if workspace is not None else _workspace_for(dev, B, T, C, k.dtype))
    if r is not None:
        if not isinstance(r, torch.Tensor) or not r.is_cuda or r.dtype != k.dtype or r.shape != k.shape \
                or not r.is_contiguous():
            raise ValueError("r must be a contiguous CUDA tensor shaped and typed like k")
        st = lib().wkv_forward_gated(B, T, C, _DTYPE[k.dtype], w.data_ptr(), u.data_ptr(), k.data_ptr(),
                                     v.data_ptr(), r.data_ptr(), _ptr(state_in), y.data_ptr(), _ptr(state_out),
                                     ws.data_ptr(), ws.numel(), _PATH[path], int(chunk), _stream(dev))
        _check(st, "wkv_forward_gated")
        return y, state_out
    st = lib().wkv_forward_ex(B, T, C, _DTYPE[k.dtype], w.data_ptr(), u.data_ptr(), k.data_ptr(), v.data_ptr(),
                              _ptr(state_in), y.data_ptr(), _ptr(state_out), ws.data_ptr(), ws.numel(),
                              _PATH[path], int(chunk), _stream(dev))
    _check(st, "wkv_forward")
    return y, state_out


def wkv_backward(w, u, k, v, gy, workspace=None):
    """Gradients of sum(gy * y) for the forward from the empty state over fp32 [B, T, C]:
    returns (gk, gv, gw, gu) with gk, gv [B, T, C] and gw, gu [C].  A workspace passed in must
    have been zero-filled before its first use (e.g. torch.zeros) and be reused only in order."""
    for t, name in ((k, "k"), (v, "v"), (gy, "gy")):
        _cuda_f32(t, name)
    if k.dim() != 3 or v.shape != k.shape or gy.shape != k.shape:
        raise ValueError("k, v, gy must be [B, T, C] tensors of one shape")
    B, T, C = k.shape
    _cuda_f32(w, "w", (C,))
    _cuda_f32(u, "u", (C,))
    gk, gv = torch.empty_like(k), torch.empty_like(v)
    gw = torch.empty(C, dtype=torch.float32, device=k.device)
    gu = torch.empty_like(gw)
    nbytes = int(lib().wkv_backward_workspace_size(B, T, C))
    ws = workspace if workspace is not None and workspace.numel() >= nbytes else \
        torch.zeros(max(nbytes, 64), dtype=torch.uint8, device=k.device)
    _check(lib().wkv_backward(B, T, C, w.data_ptr(), u.data_ptr(), k.data_ptr(), v.data_ptr(), gy.data_ptr(),
                              gk.data_ptr(), gv.data_ptr(), gw.data_ptr(), gu.data_ptr(), ws.data_ptr(), ws.numel(),
                              _stream(k.device)), "wkv_backward")
    return gk, gv, gw, gu


def eagle_forward(w, r, k, v, state_in=None, want_state=True, y=None, state_out=None, workspace=None):
    """Eagle (RWKV-5) matrix-state prefill over fp32 [B, T, C] (C a multiple of 64): returns
    (y, state_out) with state [B, C // 64, 64, 64] (None unless want_state or state_out)."""
    for t, name in ((r, "r"), (k, "k"), (v, "v")):
        _cuda_f32(t, name)
    if k.dim() != 3 or r.shape != k.shape or v.shape != k.shape:
        raise ValueError("r, k, v must be [B, T, C] tensors of one shape")
    B, T, C = k.shape
    _cuda_f32(w, "w", (C,))
    H = C // 64
    if state_in is not None:
        _cuda_f32(state_in, "state_in", (B, H, 64, 64))
    y = torch.empty_like(k) if y is None else y
    if state_out is None and want_state:
        state_out = torch.empty((B, H, 64, 64), dtype=torch.float32, device=k.device)
    nbytes = int(lib().eagle_forward_workspace_size(B, T, C))
    ws = workspace if workspace is not None and workspace.numel() >= nbytes else \
        torch.empty(max(nbytes, 16), dtype=torch.uint8, device=k.device)
    _check(lib().eagle_forward(B, T, C, w.data_ptr(), r.data_ptr(), k.data_ptr(), v.data_ptr(),
                               _ptr(state_in), y.data_ptr(), _ptr(state_out), ws.data_ptr(), ws.numel(),
                               _stream(k.device)), "eagle_forward")
    return y, state_out


def eagle_decode_step(w, r, k, v, state, y=None):
    """One Eagle token for [N, L, C] rows with [L, C] decay rates; state [N, L, C // 64, 64, 64]
    updated in place.  Returns y [N, L, C]."""
    _cuda_f32(k, "k")
    if k.dim() != 3:
        raise ValueError("k must be [N, L, C]")
    N, L, C = k.shape
    _cuda_f32(r, "r", (N, L, C))
    _cuda_f32(v, "v", (N, L, C))
    _cuda_f32(w, "w", (L, C))
    _cuda_f32(state, "state", (N, L, C // 64, 64, 64))
    y = torch.empty_like(k) if y is None else y
    _check(lib().eagle_decode_step(N, L, C, w.data_ptr(), r.data_ptr(), k.data_ptr(), v.data_ptr(), state.data_ptr(),
                                   y.data_ptr(), _stream(k.device)), "eagle_decode_step")
    return y


def forward_status(workspace=None, device=None):
    """Synchronise and report a device-side timeout of a forward (raises WkvError)."""
    dev = torch.device(device or "cuda")
    ptr, n = (workspace.data_ptr(), workspace.numel()) if workspace is not None else (None, 0)
    _check(lib().wkv_forward_status(ptr, n, _stream(dev)), "wkv_forward_status")


def get_device_status(device=None):
    """Synchronise the current stream and report (then clear) a device-side timeout of any
    forward on the device since the last call (raises WkvError)."""
    dev = torch.device(device or "cuda")
    _check(lib().wkv_get_device_status(_stream(dev)), "wkv_get_device_status")


def wkv_decode_step(w, u, k, v, state, y=None):
    """One decode step for [N, L, C] rows with [L, C] parameters; state [3, N, L, C] in place."""
    _cuda_f32(k, "k")
    if k.dim() != 3:
        raise ValueError("k must be [N, L, C]")
    N, L, C = k.shape
    _cuda_f32(v, "v", (N, L, C))
    _cuda_f32(w, "w", (L, C))
    _cuda_f32(u, "u", (L, C))
    _cuda_f32(state, "state", (3, N, L, C))
    y = torch.empty_like(k) if y is None else _cuda_f32(y, "y", (N, L, C))
    _check(lib().wkv_decode_step(N, L, C, w.data_ptr(), u.data_ptr(), k.data_ptr(), v.data_ptr(),
                                 state.data_ptr(), y.data_ptr(), _stream(k.device)), "wkv_decode_step")
    return y


def wkv_decode_step_fused(mu, w, u, x_t, x_prev, k, v, state, xbar=None, y=None):
    """Token-shift lerp + decode step in one kernel.  Returns (xbar, y); state updated in place."""
    _cuda_f32(k, "k")
    if k.dim() != 3:
        raise ValueError("k must be [N, L, C]")
    N, L, C = k.shape
    for t, name in ((v, "v"), (x_t, "x_t"), (x_prev, "x_prev")):
        _cuda_f32(t, name, (N, L, C))
    for t, name in ((mu, "mu"), (w, "w"), (u, "u")):
        _cuda_f32(t, name, (L, C))
    _cuda_f32(state, "state", (3, N, L, C))
    xbar = torch.empty_like(k) if xbar is None else _cuda_f32(xbar, "xbar", (N, L, C))
    y = torch.empty_like(k) if y is None else _cuda_f32(y, "y", (N, L, C))
    _check(lib().wkv_decode_step_fused(N, L, C, mu.data_ptr(), w.data_ptr(), u.data_ptr(), x_t.data_ptr(),
                                       x_prev.data_ptr(), xbar.data_ptr(), k.data_ptr(), v.data_ptr(),
                                       state.data_ptr(), y.data_ptr(), _stream(k.device)),
           "wkv_decode_step_fused")
    return xbar, y


def token_shift_mix3(mu_r, mu_k, mu_v, x, x_last=None):
    """The receptance, key and value lerps of x [B, T, C] in one pass, each with its own mu [C].
    Returns (xr, xk, xv)."""
    _cuda_f32(x, "x")
    if x.dim() != 3:
        raise ValueError("x must be [B, T, C]")
    B, T, C = x.shape
    for m, name in ((mu_r, "mu_r"), (mu_k, "mu_k"), (mu_v, "mu_v")):
        _cuda_f32(m, name, (C,))
    if x_last is not None:
        _cuda_f32(x_last, "x_last", (B, C))
    xr, xk, xv = (torch.empty_like(x) for _ in range(3))
    _check(lib().token_shift_mix3(B, T, C, mu_r.data_ptr(), mu_k.data_ptr(), mu_v.data_ptr(), x.data_ptr(),
                                  _ptr(x_last), xr.data_ptr(), xk.data_ptr(), xv.data_ptr(), _stream(x.device)),
           "token_shift_mix3")
    return xr, xk, xv


def token_shift_mix(mu, x, x_last=None, xbar=None):
    """xbar_t = mu * x_t + (1 - mu) * x_{t-1} over [B, T, C]; x_last [B, C] or None (zeros)."""
    _cuda_f32(x, "x")
    if x.dim() != 3:
        raise ValueError("x must be [B, T, C]")
    B, T, C = x.shape
    _cuda_f32(mu, "mu", (C,))
    if x_last is not None:
        _cuda_f32(x_last, "x_last", (B, C))
    xbar = torch.empty_like(x) if xbar is None else _cuda_f32(xbar, "xbar", (B, T, C))
    _check(lib().token_shift_mix(B, T, C, mu.data_ptr(), x.data_ptr(), _ptr(x_last), xbar.data_ptr(),
                                 _stream(x.device)), "token_shift_mix")
    return xbar
