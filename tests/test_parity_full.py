"""The benchmark workloads at full size, in the launch configuration bench.py times
(the default path), against the fp64 oracle (GPU).

Every output element is compared with the stabilised fp64 recurrence; sampled
channels are also compared with the direct O(T^2) sum; the final state is
compared canonically."""
import numpy as np
import pytest

import oracle
import synth
from parity_util import TOL_Y, assert_state_close, gpu_forward, scaled_output_error

pytestmark = pytest.mark.gpu


def _check(name, n_direct, direct_seed):
    spec = synth.FORWARD[name]
    w, u, k, v = synth.forward_inputs(spec)
    y, st = gpu_forward(w, u, k, v, spec.dtype)
    y_ref, s_ref, st_ref, sa_ref = oracle.wkv_recurrent(w, u, k, v)
    err = scaled_output_error(y, y_ref, s_ref)
    assert err <= TOL_Y[spec.dtype], f"{name}: {err:.3e}"
    assert_state_close(st, st_ref, sa_ref, what=name)
    if n_direct:
        r = np.random.default_rng(direct_seed)
        bs = r.integers(0, spec.B, n_direct)
        cs = r.integers(0, spec.C, n_direct)
        cs[0], bs[0] = spec.C - 1, spec.B - 1
        kd = k[bs, :, cs].T[None].copy()  # [1, T, n]
        vd = v[bs, :, cs].T[None].copy()
        y_d, s_d = oracle.wkv_direct(w[cs], u[cs], kd, vd)
        yg = y[bs, :, cs].T[None]
        assert scaled_output_error(yg, y_d, s_d) <= TOL_Y[spec.dtype]
    return err


def test_fwd_64x64_direct_sum_all_elements():
    spec = synth.FORWARD["fwd_64x64"]
    w, u, k, v = synth.forward_inputs(spec)
    for path in ("auto", "serial", "chunked"):
        y, st = gpu_forward(w, u, k, v, path=path)
        y_d, s_d = oracle.wkv_direct(w, u, k, v)
        assert scaled_output_error(y, y_d, s_d) <= TOL_Y["f32"]
        _, _, st_ref, sa_ref = oracle.wkv_recurrent(w, u, k, v)
        assert_state_close(st, st_ref, sa_ref)


def test_fwd_8x1024x768_with_key_spikes():
    _check("fwd_8x1024x768", 64, 1)


def test_fwd_4x4096x2048_bf16():
    _check("fwd_4x4096x2048_bf16", 16, 2)


def test_fwd_1x16384x4096_long_context():
    _check("fwd_1x16384x4096", 6, 3)
