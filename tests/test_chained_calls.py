"""Dependent calls back to back on one stream (GPU).

The forward and backward kernels are launched so that they may be scheduled while the stream's
previous kernel is still running; each waits in-kernel for it before its first access to global
memory.  Here every call reads what the call before it wrote, with no synchronisation in
between, and each result is checked against the oracle run on the inputs that call was given
(read back once the chain has finished): a kernel that started reading too early would not
match."""
import numpy as np
import pytest

import oracle
import synth
from parity_util import TOL_Y, scaled_output_error, to_gpu

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("shape", [(2, 700, 256), (1, 3000, 64), (3, 129, 36)], ids=lambda s: "x".join(map(str, s)))
def test_dependent_calls_on_one_stream(shape):
    import torch
    import linear_attention_rnn_wkv_b200 as wkv
    B, T, C = shape
    spec = synth.forward_spec_like("fwd_8x1024x768", B, T, C, seed=9700 + T)
    w, u, k, v = synth.forward_inputs(spec)
    gy = synth.grad_output(spec)
    wg, ug, kg, vg, gyg = (to_gpu(a) for a in (w, u, k, v, gy))
    y1, _ = wkv.wkv_forward(wg, ug, kg, vg)              # the plain forward
    y2, _ = wkv.wkv_forward(wg, ug, y1, vg)              # its output as the keys
    y3, _ = wkv.wkv_forward(wg, ug, kg, y2, r=y1)        # as the values, gated by the first output
    gk, gv, gw, gu = wkv.wkv_backward(wg, ug, y1, y3, gyg)
    torch.cuda.synchronize()
    y1h, y2h, y3h = (t.cpu().numpy() for t in (y1, y2, y3))

    ry, rs, _, _ = oracle.wkv_recurrent(w, u, k, v)
    assert scaled_output_error(y1h, ry, rs) <= TOL_Y["f32"]
    ry, rs, _, _ = oracle.wkv_recurrent(w, u, y1h, v)
    assert scaled_output_error(y2h, ry, rs) <= TOL_Y["f32"]
    ry, rs, _, _ = oracle.wkv_recurrent(w, u, k, y2h)
    assert scaled_output_error(y3h, oracle.gate(y1h, ry), rs) <= TOL_Y["f32"]
    rk, rv, rw, ru, (sk, sv, sw, su) = oracle.wkv_backward(w, u, y1h, y3h, gy)
    for name, g, r, s in (("gk", gk, rk, sk), ("gv", gv, rv, sv), ("gw", gw, rw, sw), ("gu", gu, ru, su)):
        err = np.abs(g.cpu().numpy() - r) / np.maximum(s, 1e-30)
        assert err.max() <= 2e-4, f"{name}: {err.max():.3e}"
