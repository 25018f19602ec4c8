"""The receptance-gated forward and the three-mu token shift against the oracle (GPU).

Gate: y = sigma(r) * wkv channel by channel (transformer-math page, section "Receptance:
the gate on the way out").  The error of a gated output is measured like an ungated one,
|o - o*| / s with s the |v|-weighted scale of wkv: sigma <= 1, so the ungated bar holds.
"""
import numpy as np
import pytest

import oracle
import synth
from parity_util import TOL_Y, assert_state_close, scaled_output_error, to_gpu

pytestmark = pytest.mark.gpu

PATHS = [("auto", 0), ("serial", 0), ("chunked", 4), ("chunked", 8), ("chunked", 16)]
SHAPES = [(1, 1, 2), (2, 3, 5), (1, 65, 129), (3, 64, 32), (2, 257, 36), (2, 300, 256), (1, 130, 136)]


def _case(B, T, C, dtype, seed):
    spec = synth.forward_spec_like("fwd_8x1024x768", B, T, C, seed=seed)
    spec = synth.ForwardSpec(spec.name, B, T, C, dtype, spec.k_std, spec.w_lo, spec.w_hi, spec.spike_prob,
                             spec.spike_value, seed)
    w, u, k, v = synth.forward_inputs(spec)
    return w, u, k, v, synth.receptance(spec)


def _gpu_gated(w, u, k, v, r, dtype, path="auto", chunk=0, state_in=None):
    import torch
    import linear_attention_rnn_wkv_b200 as wkv
    td = torch.float32 if dtype == "f32" else torch.bfloat16
    y, st = wkv.wkv_forward(to_gpu(w), to_gpu(u), to_gpu(k, td), to_gpu(v, td), r=to_gpu(r, td),
                            state_in=None if state_in is None else to_gpu(state_in.astype(np.float32)),
                            path=path, chunk=chunk)
    torch.cuda.synchronize()
    return y.float().cpu().numpy(), st.cpu().numpy()


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("path,chunk", PATHS)
@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "x".join(map(str, s)))
def test_gated_forward_matches_oracle(shape, path, chunk, dtype):
    B, T, C = shape
    w, u, k, v, r = _case(B, T, C, dtype, seed=9100 + B * 131 + T * 17 + C)
    o, st = _gpu_gated(w, u, k, v, r, dtype, path, chunk)
    y_ref, s_ref, st_ref, sa_ref = oracle.wkv_recurrent(w, u, k, v)
    o_ref = oracle.gate(r, y_ref)
    assert scaled_output_error(o, o_ref, s_ref) <= TOL_Y[dtype]
    # the gate acts on the output only: the state is the plain recurrence's
    assert_state_close(st, st_ref, sa_ref)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_gated_forward_resumes_from_state(dtype):
    B, T, C = 2, 300, 192
    w, u, k, v, r = _case(B, T, C, dtype, seed=9301)
    cut = 173
    _, _, st0, sa0 = oracle.wkv_recurrent(w, u, k[:, :cut], v[:, :cut])
    o, st = _gpu_gated(w, u, k[:, cut:], v[:, cut:], r[:, cut:], dtype, state_in=st0)
    y_ref, s_ref, st_ref, sa_ref = oracle.wkv_recurrent(w, u, k[:, cut:], v[:, cut:], state_in=st0, sacc_in=sa0)
    assert scaled_output_error(o, oracle.gate(r[:, cut:], y_ref), s_ref) <= TOL_Y[dtype]
    assert_state_close(st, st_ref, sa_ref)


@pytest.mark.parametrize("path,chunk", [("auto", 0), ("serial", 0), ("chunked", 4)])
def test_gate_limits_are_exact(path, chunk):
    """r = +60: sigma rounds to 1 in fp32, so the gated output is the ungated one bit for bit
    (the fused and unfused gates see the same y); r = -200: the gate is exactly 0.  T = 100 keeps
    every path at one or two time segments, whose carries come from one fixed record (the first
    segment publishes only its inclusive prefix), so the two calls' carries agree bit for bit;
    with more segments a look-back may fold an aggregate or an inclusive prefix depending on
    timing, which changes the last bits only."""
    import torch
    import linear_attention_rnn_wkv_b200 as wkv
    B, T, C = 2, 100, 128
    w, u, k, v, _ = _case(B, T, C, "f32", seed=9401)
    args = [to_gpu(a) for a in (w, u, k, v)]
    y_plain, _ = wkv.wkv_forward(*args, path=path, chunk=chunk)
    y_open, _ = wkv.wkv_forward(*args, r=torch.full_like(args[2], 60.0), path=path, chunk=chunk)
    y_shut, _ = wkv.wkv_forward(*args, r=torch.full_like(args[2], -200.0), path=path, chunk=chunk)
    torch.cuda.synchronize()
    assert torch.equal(y_open, y_plain)
    assert torch.count_nonzero(y_shut).item() == 0


def test_gated_full_size_all_elements():
    """fwd_8x1024x768 at full size through the default path: every element of the gated output
    against the oracle's sigma(r) * wkv."""
    import linear_attention_rnn_wkv_b200 as wkv
    spec = synth.FORWARD["fwd_8x1024x768"]
    w, u, k, v = synth.forward_inputs(spec)
    r = synth.receptance(spec)
    o, _ = wkv.wkv_forward(to_gpu(w), to_gpu(u), to_gpu(k), to_gpu(v), r=to_gpu(r))
    o = o.cpu().numpy()
    y_ref, s_ref, _, _ = oracle.wkv_recurrent(w, u, k, v)
    o_ref = oracle.gate(r, y_ref)
    assert scaled_output_error(o, o_ref, s_ref) <= TOL_Y["f32"]


def test_token_shift_three_mu():
    import torch
    import linear_attention_rnn_wkv_b200 as wkv
    for (B, T, C) in [(2, 9, 64), (1, 5, 37), (3, 1, 8), (2, 70, 768)]:
        rng = np.random.default_rng(B * 100 + C + 7)
        mus = [rng.uniform(0, 1, C).astype(np.float32) for _ in range(3)]
        x = rng.normal(0, 1, (B, T, C)).astype(np.float32)
        xl = rng.normal(0, 1, (B, C)).astype(np.float32)
        for last in (None, xl):
            outs = wkv.token_shift_mix3(*(torch.from_numpy(m).cuda() for m in mus), torch.from_numpy(x).cuda(),
                                        None if last is None else torch.from_numpy(last).cuda())
            refs = oracle.token_shift3(*mus, x, last)
            prev = np.concatenate([np.zeros((B, 1, C)) if last is None else last[:, None], x[:, :-1]], axis=1)
            for o, ref, mu in zip(outs, refs, mus):
                scale = np.abs(mu * x) + np.abs((1 - mu) * prev)
                assert np.all(np.abs(o.cpu().numpy() - ref) <= 1e-6 * np.maximum(scale, 1e-30))
