"""Eagle (RWKV-5) matrix-state WKV on the GPU against the fp64 oracle.

Recurrence ("RWKV (Attention-RNN Hybrid)", section "Versions: RWKV-4 -> Eagle -> Finch"):
S_t = diag(e^{-w}) S_{t-1} + k_t v_t^T, y_t = r_t^T S_t, per head of 64 channels.

Error measures: an output is compared with the oracle relative to its magnitude scale s (the
same read-out with |r|, |k|, |v| and |S_in|, so s >= |y|); a state entry relative to the state
of the same recurrence run on |k|, |v|, |S_in|.  Bar: TOL_EAGLE = 1e-4.  The kernels compute
in fp32: each state entry is a decayed sum whose terms carry a few fp32 roundings and at most
64 compounded products of the per-step decay (each e^{-w} good to ~2^-22), so its error stays
below ~64 * 2^-22 = 1.5e-5 of its magnitude scale; the read-out adds 64 fp32 additions.
1e-4 leaves a 5x margin over that bound and is the forward's fp32 output bar.
"""
import numpy as np
import pytest

import oracle
import synth
from parity_util import to_gpu

pytestmark = pytest.mark.gpu

TOL_EAGLE = 1e-4

SHAPES = [(1, 1, 64), (2, 3, 64), (1, 63, 128), (2, 64, 64), (2, 65, 128), (2, 128, 128), (1, 130, 192),
          (3, 200, 64), (1, 1000, 64)]


def _case(B, T, C, seed):
    spec = synth.eagle_spec_like("eagle_8x1024x768", B, T, C, seed=seed)
    return spec, synth.eagle_inputs(spec)


def _state_scale(w, k, v, state_in):
    """The state of the recurrence on |k|, |v| (and |S_in|): every state entry's magnitude scale."""
    r1 = np.ones_like(k)
    return oracle.eagle_recurrent(w, r1, np.abs(k), np.abs(v), state_in=None if state_in is None else np.abs(state_in))[2]


def _gpu_forward(w, r, k, v, state_in=None):
    import torch
    import linear_attention_rnn_wkv_b200 as wkv
    y, st = wkv.eagle_forward(to_gpu(w), to_gpu(r), to_gpu(k), to_gpu(v),
                              state_in=None if state_in is None else to_gpu(state_in))
    torch.cuda.synchronize()
    return y.cpu().numpy(), st.cpu().numpy()


def _check(y, st, w, r, k, v, state_in=None):
    y_ref, s_ref, st_ref = oracle.eagle_recurrent(w, r, k, v, state_in=state_in)
    assert np.all(np.isfinite(y)) and np.all(np.isfinite(st))
    ey = float(np.max(np.abs(y - y_ref) / np.maximum(s_ref, 1e-300))) if y.size else 0.0
    es = float(np.max(np.abs(st - st_ref) / np.maximum(_state_scale(w, k, v, state_in), 1e-300)))
    assert ey <= TOL_EAGLE, f"output error {ey:.3e}"
    assert es <= TOL_EAGLE, f"state error {es:.3e}"


@pytest.mark.parametrize("with_state", [False, True])
@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "x".join(map(str, s)))
def test_eagle_forward_matches_oracle(shape, with_state):
    B, T, C = shape
    spec, (w, r, k, v) = _case(B, T, C, seed=2100 + B * 131 + T * 17 + C)
    state_in = synth.eagle_state(spec) if with_state else None
    y, st = _gpu_forward(w, r, k, v, state_in)
    _check(y, st, w, r, k, v, state_in)


@pytest.mark.parametrize("shape", [(2, 700, 768), (4, 333, 512), (3, 1000, 512), (2, 1000, 256)],
                         ids=lambda s: "x".join(map(str, s)))
def test_eagle_forward_both_forms(shape):
    """Shapes on either side of the choice between the one-launch form (a block per sequence-head
    walking its chunks: 24 or more sequence-heads) and the three-launch form (few heads, more than
    8 chunks), ragged last chunks, with and without a given state, every element checked."""
    import linear_attention_rnn_wkv_b200 as wkv
    B, T, C = shape
    launches = wkv.lib().eagle_forward_launches(B, T, C)
    assert launches == (1 if B * (C // 64) >= 24 else 3)
    spec, (w, r, k, v) = _case(B, T, C, seed=2300 + B + T + C)
    y, st = _gpu_forward(w, r, k, v)
    _check(y, st, w, r, k, v)
    S0 = synth.eagle_state(spec)
    y, st = _gpu_forward(w, r, k, v, S0)
    _check(y, st, w, r, k, v, S0)


def test_eagle_forward_fast_decay_head():
    """A head holding one channel with w = 7 (decay e^-7 per token, beyond the range the
    one-launch form's scaled operands admit) runs token by token in the same launch while the
    other heads use the tensor cores; every element against the oracle, for both forms."""
    import linear_attention_rnn_wkv_b200 as wkv
    for B, T, C in ((3, 150, 512), (1, 600, 192)):
        spec, (w, r, k, v) = _case(B, T, C, seed=2310 + T)
        w = w.copy()
        w[64 + 5] = 7.0
        assert wkv.lib().eagle_forward_launches(B, T, C) == (1 if B * (C // 64) >= 24 or T <= 512 else 3)
        S0 = synth.eagle_state(spec)
        y, st = _gpu_forward(w, r, k, v, S0)
        _check(y, st, w, r, k, v, S0)


def test_eagle_forward_decay_extremes():
    """No decay (w = 0: causal linear attention) and total decay (w = 1e4: only the current
    token, y_t = (r_t . k_t) v_t) on the GPU."""
    B, T, C = 2, 150, 128
    spec, (w, r, k, v) = _case(B, T, C, seed=2201)
    for wx in (np.zeros_like(w), np.full_like(w, 1e4)):
        y, st = _gpu_forward(wx, r, k, v)
        _check(y, st, wx, r, k, v)
    y, _ = _gpu_forward(np.full_like(w, 1e4), r, k, v)
    for h in range(C // 64):
        sl = slice(h * 64, (h + 1) * 64)
        ref = (r[:, :, sl].astype(np.float64) * k[:, :, sl]).sum(-1, keepdims=True) * v[:, :, sl]
        assert np.allclose(y[:, :, sl], ref, rtol=1e-5, atol=1e-5)


def test_eagle_forward_empty_sequence():
    """T = 0 returns the given state (or zeros) as the final state."""
    import torch
    import linear_attention_rnn_wkv_b200 as wkv
    spec, (w, r, k, v) = _case(2, 0, 128, seed=2202)
    S0 = synth.eagle_state(spec)
    args = [to_gpu(a) for a in (w, r, k, v)]
    _, st = wkv.eagle_forward(*args, state_in=to_gpu(S0))
    _, st0 = wkv.eagle_forward(*args)
    torch.cuda.synchronize()
    assert np.array_equal(st.cpu().numpy(), S0)
    assert not np.any(st0.cpu().numpy())


def test_eagle_forward_resumes_from_state():
    """Prefill [0, cut) then [cut, T) from the returned state equals the whole prefill."""
    B, T, C = 2, 333, 128
    spec, (w, r, k, v) = _case(B, T, C, seed=2203)
    cut = 171
    y1, st1 = _gpu_forward(w, r[:, :cut], k[:, :cut], v[:, :cut])
    y2, st2 = _gpu_forward(w, r[:, cut:], k[:, cut:], v[:, cut:], state_in=st1)
    _check(np.concatenate([y1, y2], axis=1), st2, w, r, k, v)


def test_eagle_full_size_all_heads():
    """eagle_8x1024x768 at full size (the bench's launch): every sequence-head against the oracle."""
    spec = synth.EAGLE["eagle_8x1024x768"]
    w, r, k, v = synth.eagle_inputs(spec)
    y, st = _gpu_forward(w, r, k, v)
    _check(y, st, w, r, k, v)


def test_eagle_long_workload_sampled_heads():
    """eagle_4x4096x2048 at full size (32 heads, 4096 tokens): 24 sampled sequence-heads, the
    last one included, against the oracle."""
    spec = synth.EAGLE["eagle_4x4096x2048"]
    w, r, k, v = synth.eagle_inputs(spec)
    y, st = _gpu_forward(w, r, k, v)
    rng = np.random.default_rng(8)
    pairs = list(zip(rng.integers(0, spec.B, 23), rng.integers(0, spec.C // 64, 23))) + [(spec.B - 1, spec.C // 64 - 1)]
    for b, h in pairs:
        sl = slice(h * 64, (h + 1) * 64)
        _check(y[b:b + 1, :, sl], st[b:b + 1, h:h + 1], w[sl], r[b:b + 1, :, sl], k[b:b + 1, :, sl],
               v[b:b + 1, :, sl])


def test_eagle_decode_matches_oracle():
    """One token for N sessions x L layers from a given state, then a prefill -> decode hand-off:
    forward over T tokens and two decode steps give the outputs of a forward over T + 2."""
    import torch
    import linear_attention_rnn_wkv_b200 as wkv
    N, L, C = 3, 2, 128
    H = C // 64
    g = np.random.default_rng(2204)
    w = np.exp(g.uniform(-5, 1, (L, C))).astype(np.float32)
    r, k, v = (g.normal(0, 1, (N, L, C)).astype(np.float32) for _ in range(3))
    S = g.normal(0, 1, (N, L, H, 64, 64)).astype(np.float32)
    St = to_gpu(S)
    y = wkv.eagle_decode_step(to_gpu(w), to_gpu(r), to_gpu(k), to_gpu(v), St)
    torch.cuda.synchronize()
    y, St = y.cpu().numpy(), St.cpu().numpy()
    for l in range(L):
        _check(y[:, l:l + 1], St[:, l], w[l], r[:, l:l + 1], k[:, l:l + 1], v[:, l:l + 1], state_in=S[:, l])

    B, T = 2, 97
    spec, (w1, r1, k1, v1) = _case(B, T + 2, C, seed=2205)
    _, st = _gpu_forward(w1, r1[:, :T], k1[:, :T], v1[:, :T])
    st_g = to_gpu(st.reshape(B, 1, H, 64, 64))
    ys = []
    for t in (T, T + 1):
        ys.append(wkv.eagle_decode_step(to_gpu(w1[None]), to_gpu(r1[:, t:t + 1]), to_gpu(k1[:, t:t + 1]),
                                        to_gpu(v1[:, t:t + 1]), st_g).cpu().numpy())
    torch.cuda.synchronize()
    y_ref, s_ref, st_ref = oracle.eagle_recurrent(w1, r1, k1, v1)
    ydec = np.concatenate(ys, axis=1)
    assert np.max(np.abs(ydec - y_ref[:, T:]) / s_ref[:, T:]) <= TOL_EAGLE
    assert np.max(np.abs(st_g.cpu().numpy()[:, 0] - st_ref) / _state_scale(w1, k1, v1, None)) <= TOL_EAGLE
