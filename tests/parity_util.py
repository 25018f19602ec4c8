"""Helpers for comparing the CUDA path with the fp64 oracle.

Error measures (the readings of the tolerances):

* outputs: err_t = |y - y*| / s_t where s_t is eq. 1 evaluated with |v| in place of
  v (the oracle computes it alongside y; s_t >= |y*_t|).  A plain relative error is
  ill-posed where y* crosses zero while the terms that form it do not.
* states: (a, b, p) is defined only up to (a e^d, b e^d, p - d), so the CUDA state is
  first rescaled to the oracle's exponent p*: b~ = b e^{p - p*} is compared with b*
  relative to b*, a~ = a e^{p - p*} with a* relative to the oracle's magnitude
  accumulator (a with |v|), and p with p* relative to max(1, |p*|).
"""
from __future__ import annotations

import numpy as np

# Tolerances: outputs 1e-4 (fp32 I/O) / 2e-2 (bf16 I/O); states 1e-5.
TOL_Y = {"f32": 1e-4, "bf16": 2e-2}
TOL_STATE = 1e-5


def scaled_output_error(y, y_ref, s_ref):
    y = np.asarray(y, np.float64)
    assert np.all(np.isfinite(y)), "non-finite output"
    return float(np.max(np.abs(y - y_ref) / np.maximum(s_ref, 1e-300))) if y.size else 0.0


def state_errors(st, st_ref, sacc_ref):
    st = np.asarray(st, np.float64)
    assert np.all(np.isfinite(st)), "non-finite state"
    a, b, p = st[0], st[1], st[2]
    A, Bs, P = st_ref[0], st_ref[1], st_ref[2]
    scale = np.exp(p - P)
    eb = np.max(np.abs(b * scale - Bs) / Bs)
    ea = np.max(np.abs(a * scale - A) / np.maximum(sacc_ref, 1e-300))
    ep = np.max(np.abs(p - P) / np.maximum(1.0, np.abs(P)))
    return float(eb), float(ea), float(ep)


def assert_state_close(st, st_ref, sacc_ref, tol=TOL_STATE, what="state"):
    eb, ea, ep = state_errors(st, st_ref, sacc_ref)
    assert eb <= tol and ea <= tol and ep <= tol, f"{what}: b {eb:.2e} a {ea:.2e} p {ep:.2e} (tol {tol:g})"


def to_gpu(a, dtype=None):
    import torch
    t = torch.from_numpy(np.ascontiguousarray(a)).cuda()
    return t if dtype is None else t.to(dtype)


def gpu_forward(w, u, k, v, dtype="f32", state_in=None, path="auto", chunk=0, want_state=True):
    """Run wkv_forward on numpy inputs (k, v hold values exact in the I/O dtype)."""
    import torch
    import linear_attention_rnn_wkv_b200 as wkv
    td = torch.float32 if dtype == "f32" else torch.bfloat16
    y, st = wkv.wkv_forward(to_gpu(w), to_gpu(u), to_gpu(k, td), to_gpu(v, td),
                            state_in=None if state_in is None else to_gpu(state_in.astype(np.float32)),
                            want_state=want_state, path=path, chunk=chunk)
    torch.cuda.synchronize()
    return y.float().cpu().numpy(), None if st is None else st.cpu().numpy()
