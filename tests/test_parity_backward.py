"""The WKV backward against the oracle (GPU).

Gradients of L = sum(gy * y) with respect to k, v (per element) and w, u (per channel),
for the forward from the empty state.  Each error is divided by the magnitude of the terms
that make up that gradient (the oracle adds them up with |gy|, and |v| + |y| in place of
v - y): gradients that cancel to near zero are not judged relative to themselves.  Bar: 2e-4 of that scale (fp32
throughout; the reverse scan compounds the forward's rounding over T steps).
"""
import numpy as np
import pytest

import oracle
import synth
from parity_util import to_gpu

pytestmark = pytest.mark.gpu

TOL_GRAD = 2e-4
# T = 3000 and 2049: 24 and 17 groups of 128 steps (eight 16-step segments each), so the
# look-backs take several hops and the last group is ragged; C = 129: a channel block of one lane;
# T = 128 and 256: one and two whole groups (no ragged group), the latter with rows of 37
# channels (not whole 16-byte units: the cp.async staging)
SHAPES = [(1, 1, 4), (2, 5, 3), (1, 64, 64), (1, 128, 32), (2, 256, 37), (3, 200, 96), (1, 1000, 32),
          (2, 130, 129), (1, 3000, 8), (2, 2049, 4)]


def _case(B, T, C, base, seed, k_shift=0.0):
    spec = synth.forward_spec_like(base, B, T, C, seed=seed)
    w, u, k, v = synth.forward_inputs(spec)
    return w, u, k + np.float32(k_shift), v, synth.grad_output(spec)


def _gpu_backward(w, u, k, v, gy):
    import torch
    import linear_attention_rnn_wkv_b200 as wkv
    gk, gv, gw, gu = wkv.wkv_backward(to_gpu(w), to_gpu(u), to_gpu(k), to_gpu(v), to_gpu(gy))
    torch.cuda.synchronize()
    return gk.cpu().numpy(), gv.cpu().numpy(), gw.cpu().numpy(), gu.cpu().numpy()


def _check(w, u, k, v, gy):
    gk, gv, gw, gu = _gpu_backward(w, u, k, v, gy)
    rk, rv, rw, ru, (sk, sv, sw, su) = oracle.wkv_backward(w, u, k, v, gy)
    for name, g, r, s in (("gk", gk, rk, sk), ("gv", gv, rv, sv), ("gw", gw, rw, sw), ("gu", gu, ru, su)):
        err = np.abs(g - r) / np.maximum(s, 1e-30)
        assert np.all(np.isfinite(g)), name
        assert err.max() <= TOL_GRAD, f"{name}: {err.max():.3e}"


@pytest.mark.parametrize("base", ["fwd_64x64", "fwd_8x1024x768"])
@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "x".join(map(str, s)))
def test_backward_matches_oracle(shape, base):
    B, T, C = shape
    _check(*_case(B, T, C, base, seed=9500 + B * 131 + T * 17 + C))


def test_backward_key_shift():
    """Keys shifted by +100 (exponents near 144 in base 2): the gradients do not change."""
    _check(*_case(2, 300, 64, "fwd_8x1024x768", seed=9601, k_shift=100.0))


def test_backward_mixed_frames():
    """Channels whose 16-step segments cannot share one exponent frame (w = 20, 9 and 12: 15 w
    log2 e is far beyond the frame's range; u = -40, +30 and -25: the bonus outside it) beside
    channels that can, in the same warps: the per-step lanes and the frame lanes agree with the
    oracle."""
    spec = synth.forward_spec_like("fwd_8x1024x768", 2, 500, 40, seed=9602)
    w, u, k, v = synth.forward_inputs(spec)
    w[[0, 3, 33]] = np.float32([20.0, 9.0, 12.0])
    u[[5, 6, 38]] = np.float32([-40.0, 30.0, -25.0])
    _check(w, u, k, v, synth.grad_output(spec))


def test_backward_workspace_reuse():
    """Three calls on one workspace (its counters and tags reset by each launch): each matches
    the oracle (bits may differ between calls: a look-back folds whichever records have been
    published by then)."""
    import torch
    import linear_attention_rnn_wkv_b200 as wkv
    w, u, k, v, gy = _case(3, 700, 96, "fwd_8x1024x768", seed=9603)
    args = [to_gpu(a) for a in (w, u, k, v, gy)]
    ws = torch.zeros(int(wkv.lib().wkv_backward_workspace_size(3, 700, 96)), dtype=torch.uint8, device="cuda")
    rk, rv, rw, ru, (sk, sv, sw, su) = oracle.wkv_backward(w, u, k, v, gy)
    for _ in range(3):
        got = [t.cpu().numpy() for t in wkv.wkv_backward(*args, workspace=ws)]
        for g, r, sc in zip(got, (rk, rv, rw, ru), (sk, sv, sw, su)):
            assert np.max(np.abs(g - r) / np.maximum(sc, 1e-30)) <= TOL_GRAD


def _check_sampled(spec, n_channels, seed):
    import linear_attention_rnn_wkv_b200 as wkv
    w, u, k, v = synth.forward_inputs(spec)
    gy = synth.grad_output(spec)
    gk, gv, gw, gu = (t.cpu().numpy() for t in wkv.wkv_backward(*(to_gpu(a) for a in (w, u, k, v, gy))))
    cs = np.sort(np.random.default_rng(seed).choice(spec.C - 1, n_channels - 1, replace=False))
    cs = np.append(cs, spec.C - 1)
    # one oracle call over all sampled channels (its threads split the channels)
    rk, rv, rw, ru, (sk, sv, sw, su) = oracle.wkv_backward(w[cs], u[cs], k[:, :, cs], v[:, :, cs], gy[:, :, cs])
    gk, gv = gk[:, :, cs], gv[:, :, cs]
    assert np.all(np.isfinite(gk)) and np.all(np.isfinite(gv))
    assert np.max(np.abs(gk - rk) / np.maximum(sk, 1e-30)) <= TOL_GRAD
    assert np.max(np.abs(gv - rv) / np.maximum(sv, 1e-30)) <= TOL_GRAD
    assert np.all(np.abs(gw[cs] - rw) <= TOL_GRAD * sw)
    assert np.all(np.abs(gu[cs] - ru) <= TOL_GRAD * su)


def test_backward_full_width_sampled():
    """fwd_8x1024x768's shape (B=8, T=1024, C=768) through the GPU, 96 sampled channels against
    the oracle (channels are independent; gw and gu of a channel sum over the whole batch)."""
    _check_sampled(synth.FORWARD["fwd_8x1024x768"], 96, 11)


def test_backward_long_context_sampled():
    """The long-context shape (B=1, T=16384, C=4096) through the GPU, 12 sampled channels against
    the oracle's O(T^2) gradient (the last channel included)."""
    _check_sampled(synth.FORWARD["fwd_1x16384x4096"], 12, 12)
