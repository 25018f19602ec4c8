"""fp64 CPU oracle for the RWKV-4 WKV operator -- TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg
may import this package.  The CUDA library (``linear_attention_rnn_wkv_b200``)
never imports, links or calls it, and the two share no code.

The arithmetic lives in ``wkv_oracle.c`` (plain C, fp64, one loop per formula,
each citing the page and section it follows).  This module compiles it with gcc
and marshals numpy arrays; it does no arithmetic of its own.

Functions (all inputs are converted to contiguous float64):

* ``wkv_direct(w, u, k, v)`` -- the wkv_t equation evaluated as written
  (O(T^2) per channel).  Returns ``(y, s)``.
* ``wkv_recurrent(w, u, k, v, state_in=None, sacc_in=None)`` -- the running-
  maximum (a, b, p) recurrence.  Returns ``(y, s, state_out, sacc_out)``.
* ``wkv_naive(w, u, k, v)`` -- the plain (a, b) recurrence (in-range only).
* ``token_shift(mu, x, x_last=None)`` -- the two-tap lerp.
* ``decode_step(w, u, k, v, state, sacc)`` -- one token from a given state for
  ``[N, L, C]`` rows with ``[L, C]`` parameters: the recurrence with T = 1.
* ``gate(r, wkv)`` -- the receptance gate ``sigma(r) * wkv``, elementwise.
* ``wkv_backward(w, u, k, v, gy)`` -- the gradient of ``sum(gy * y)`` with respect to
  k, v (per element) and w, u (per channel, summed over batch and time), the
  wkv_t equation differentiated as written (O(T^2)).  Returns
  ``(gk, gv, gw, gu, (sk, sv, sw, su))`` with the terms' magnitude scales (|gy|,
  and |v| + |y| in place of v - y).
* ``token_shift3(mu_r, mu_k, mu_v, x, x_last=None)`` -- the lerp with the three
  projections' separate mu (three calls of ``token_shift``).
* ``eagle_recurrent(w, r, k, v, N=64, state_in=None)`` -- the Eagle (RWKV-5)
  matrix-state recurrence ``S_t = diag(e^{-w}) S_{t-1} + k_t v_t^T``, ``y_t = r_t^T S_t``
  per head of N channels.  Returns ``(y, s, state_out)`` (state ``[B, H, N, N]``).
* ``eagle_direct(w, r, k, v, N=64, state_in=None)`` -- the same outputs summed
  directly over the past (O(T^2 N^2) per head).

``s`` is the same weighted average with ``|v|`` in place of ``v`` (the error
scale the parity tests divide by); ``sacc`` is its accumulator in the state.

Parity status: every function is pinned by ``tests/test_oracle.py`` (worked
example, closed forms, invariants, high-precision brute force).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "wkv_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")

#: The empty-state running maximum used by the oracle (a = b = 0 there).
P_EMPTY = -1e38


def build(force: bool = False, src: str = _SRC, out: str = _LIB_PATH) -> str:
    """Compile the oracle with gcc: -O2, OpenMP, strict IEEE double (no fast-math,
    no contraction into fused multiply-adds)."""
    if force or not os.path.exists(out) or os.path.getmtime(out) < os.path.getmtime(src):
        tmp = out + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off",
                               "-fno-fast-math", "-std=c11", src, "-o", tmp, "-lm"])
        os.replace(tmp, out)
    return out


def load(path: str):
    L = ctypes.CDLL(path)
    i64, vp = ctypes.c_int64, ctypes.c_void_p
    L.oracle_wkv_direct.argtypes = [i64, i64, i64, vp, vp, vp, vp, vp, vp]
    L.oracle_wkv_recurrent.argtypes = [i64, i64, i64, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp]
    L.oracle_wkv_naive.argtypes = [i64, i64, i64, vp, vp, vp, vp, vp]
    L.oracle_token_shift.argtypes = [i64, i64, i64, vp, vp, vp, vp]
    L.oracle_gate.argtypes = [i64, vp, vp, vp]
    L.oracle_wkv_backward_direct.argtypes = [i64, i64, i64] + [vp] * 13
    L.oracle_eagle_recurrent.argtypes = [i64, i64, i64, i64] + [vp] * 8
    L.oracle_eagle_direct.argtypes = [i64, i64, i64, i64] + [vp] * 6
    for f in (L.oracle_wkv_direct, L.oracle_wkv_recurrent, L.oracle_wkv_naive, L.oracle_token_shift, L.oracle_gate,
              L.oracle_wkv_backward_direct, L.oracle_eagle_recurrent, L.oracle_eagle_direct):
        f.restype = None
    L.oracle_num_threads.restype = ctypes.c_int
    L.oracle_set_num_threads.argtypes = [ctypes.c_int]
    L.oracle_set_num_threads.restype = None
    return L


_lib = None


def lib():
    global _lib
    if _lib is None:
        _lib = load(build())
    return _lib


def num_threads() -> int:
    return int(lib().oracle_num_threads())


def set_num_threads(n: int) -> None:
    """Threads of the oracle's parallel loops (independent channels: results are unchanged)."""
    lib().oracle_set_num_threads(int(n))


def _f64(a):
    return np.ascontiguousarray(a, dtype=np.float64)


def _p(a):
    return None if a is None else a.ctypes.data


def _btc(k):
    k = np.asarray(k)
    if k.ndim == 1:
        return 1, k.shape[0], 1
    if k.ndim == 2:
        return 1, k.shape[0], k.shape[1]
    return k.shape


def wkv_direct(w, u, k, v, L=None):
    w, u, k, v = _f64(w), _f64(u), _f64(k), _f64(v)
    B, T, C = _btc(k)
    y = np.empty(k.shape, np.float64)
    s = np.empty(k.shape, np.float64)
    (L or lib()).oracle_wkv_direct(B, T, C, _p(w), _p(u), _p(k), _p(v), _p(y), _p(s))
    return y, s


def wkv_recurrent(w, u, k, v, state_in=None, sacc_in=None, L=None):
    w, u, k, v = _f64(w), _f64(u), _f64(k), _f64(v)
    B, T, C = _btc(k)
    state_in = None if state_in is None else _f64(state_in)
    sacc_in = None if sacc_in is None else _f64(sacc_in)
    y = np.empty(k.shape, np.float64)
    s = np.empty(k.shape, np.float64)
    st = np.empty((3, B, C), np.float64)
    sa = np.empty((B, C), np.float64)
    (L or lib()).oracle_wkv_recurrent(B, T, C, _p(w), _p(u), _p(k), _p(v), _p(state_in), _p(sacc_in),
                                      _p(y), _p(s), _p(st), _p(sa))
    return y, s, st, sa


def wkv_naive(w, u, k, v, L=None):
    w, u, k, v = _f64(w), _f64(u), _f64(k), _f64(v)
    B, T, C = _btc(k)
    y = np.empty(k.shape, np.float64)
    (L or lib()).oracle_wkv_naive(B, T, C, _p(w), _p(u), _p(k), _p(v), _p(y))
    return y


def token_shift(mu, x, x_last=None, L=None):
    mu, x = _f64(mu), _f64(x)
    B, T, C = _btc(x)
    x_last = None if x_last is None else _f64(x_last)
    xbar = np.empty(x.shape, np.float64)
    (L or lib()).oracle_token_shift(B, T, C, _p(mu), _p(x), _p(x_last), _p(xbar))
    return xbar


def gate(r, wkv, L=None):
    """sigma(r) * wkv elementwise; r and wkv of one shape."""
    r, wkv = _f64(r), _f64(wkv)
    if r.shape != wkv.shape:
        raise ValueError("r and wkv must have the same shape")
    out = np.empty(r.shape, np.float64)
    (L or lib()).oracle_gate(r.size, _p(r), _p(wkv), _p(out))
    return out


def wkv_backward(w, u, k, v, gy, L=None):
    w, u, k, v, gy = _f64(w), _f64(u), _f64(k), _f64(v), _f64(gy)
    B, T, C = _btc(k)
    gk, gv, sk, sv = (np.empty(k.shape, np.float64) for _ in range(4))
    gw, gu, sw, su = (np.empty(C, np.float64) for _ in range(4))
    (L or lib()).oracle_wkv_backward_direct(B, T, C, _p(w), _p(u), _p(k), _p(v), _p(gy), _p(gk), _p(gv), _p(gw),
                                            _p(gu), _p(sk), _p(sv), _p(sw), _p(su))
    return gk, gv, gw, gu, (sk, sv, sw, su)


def token_shift3(mu_r, mu_k, mu_v, x, x_last=None, L=None):
    """The token-shift lerp of the receptance, key and value projections, each with its
    own mu: returns ``(xr, xk, xv)``."""
    return tuple(token_shift(mu, x, x_last, L=L) for mu in (mu_r, mu_k, mu_v))


def decode_step(w, u, k, v, state, sacc=None, L=None):
    """One token for rows [N, L, C] with parameters [L, C]: the recurrence with T = 1
    over N sequences of L*C channels.  Returns ``(y, s, state, sacc)`` shaped like the
    inputs ([N, L, C] and [3, N, L, C])."""
    k = _f64(k)
    N = k.shape[0]
    LC = k[0].size
    y, s, st, sa = wkv_recurrent(_f64(w).reshape(LC), _f64(u).reshape(LC), k.reshape(N, 1, LC),
                                 _f64(v).reshape(N, 1, LC), _f64(state).reshape(3, N, LC),
                                 None if sacc is None else _f64(sacc).reshape(N, LC), L=L)
    return (y.reshape(k.shape), s.reshape(k.shape), st.reshape((3,) + k.shape), sa.reshape(k.shape))


def decode_token_shift(mu, x_t, x_prev, L=None):
    """The decode-step lerp for rows [N, L, C] with mu [L, C]."""
    x_t = _f64(x_t)
    N = x_t.shape[0]
    LC = x_t[0].size
    xb = token_shift(_f64(mu).reshape(LC), x_t.reshape(N, 1, LC), _f64(x_prev).reshape(N, LC), L=L)
    return xb.reshape(x_t.shape)


def _eagle_shapes(k, N, state_in):
    B, T, C = _btc(k)
    if C % N:
        raise ValueError(f"C = {C} is not a multiple of the head size {N}")
    H = C // N
    state_in = None if state_in is None else _f64(state_in).reshape(B, H, N, N)
    return B, T, C, H, state_in


def eagle_recurrent(w, r, k, v, N=64, state_in=None, L=None):
    w, r, k, v = _f64(w), _f64(r), _f64(k), _f64(v)
    B, T, C, H, state_in = _eagle_shapes(k, N, state_in)
    y = np.empty(k.shape, np.float64)
    s = np.empty(k.shape, np.float64)
    st = np.empty((B, H, N, N), np.float64)
    (L or lib()).oracle_eagle_recurrent(B, T, H, N, _p(w), _p(r), _p(k), _p(v), _p(state_in), _p(y), _p(s),
                                        _p(st))
    return y, s, st


def eagle_direct(w, r, k, v, N=64, state_in=None, L=None):
    w, r, k, v = _f64(w), _f64(r), _f64(k), _f64(v)
    B, T, C, H, state_in = _eagle_shapes(k, N, state_in)
    y = np.empty(k.shape, np.float64)
    (L or lib()).oracle_eagle_direct(B, T, H, N, _p(w), _p(r), _p(k), _p(v), _p(state_in), _p(y))
    return y
