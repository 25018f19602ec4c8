"""CUDA decode step (plain and fused with the token shift) vs the fp64 oracle (GPU)."""
import numpy as np
import pytest

import oracle
import synth
from parity_util import TOL_STATE, TOL_Y, assert_state_close, gpu_forward, scaled_output_error, to_gpu

pytestmark = pytest.mark.gpu


def _warm_state(spec, flat=None):
    """Oracle warm-up of `spec.warmup` tokens from the empty state, for all row-channels
    (flat=None) or for the flat row-channel indices `flat`.  Returns the fp32-rounded
    state [3, n] and the fp64 magnitude accumulator [n]."""
    mu, w, u = synth.decode_params(spec)
    n_all = spec.N * spec.L * spec.C
    if flat is None:
        flat = np.arange(n_all)
    lc = flat % (spec.L * spec.C)
    ks = np.empty((spec.warmup, flat.size), np.float32)
    vs = np.empty((spec.warmup, flat.size), np.float32)
    for t in range(spec.warmup):
        ks[t], vs[t] = synth.warmup_inputs_at(spec, t, flat)
    _, _, st, sa = oracle.wkv_recurrent(w.reshape(-1)[lc], u.reshape(-1)[lc], ks[None], vs[None])
    return st[:, 0].astype(np.float32), sa[0]


def _decode_case(N, L, C, seed, steps=128):
    return synth.DecodeSpec(f"decode_{N}x{L}x{C}", N, L, C, 512, steps, seed)


@pytest.mark.parametrize("shape", [(4, 3, 36), (2, 2, 130), (1, 1, 8), (3, 32, 64)],
                         ids=lambda s: "x".join(map(str, s)))
def test_fused_decode_128_steps(shape):
    import torch
    import linear_attention_rnn_wkv_b200 as wkv
    N, L, C = shape
    spec = _decode_case(N, L, C, 5000 + N + L + C)
    mu, w, u = synth.decode_params(spec)
    st32, sacc = _warm_state(spec)
    shape3 = (N, L, C)
    st_gpu = to_gpu(st32.reshape((3,) + shape3))
    st_ref = st32.reshape((3,) + shape3).astype(np.float64)
    sa_ref = sacc.reshape(shape3)
    x_prev = synth.warmup_last_x(spec)
    xp_gpu = to_gpu(x_prev)
    mu_g, w_g, u_g = to_gpu(mu), to_gpu(w), to_gpu(u)
    worst = 0.0
    for s in range(spec.steps):
        x_t, k, v = synth.decode_step_inputs(spec, s)
        xt_gpu = to_gpu(x_t)
        xbar, y = wkv.wkv_decode_step_fused(mu_g, w_g, u_g, xt_gpu, xp_gpu, to_gpu(k), to_gpu(v), st_gpu)
        torch.cuda.synchronize()
        xbar_ref = oracle.decode_token_shift(mu, x_t, x_prev)
        y_ref, s_ref, st_ref, sa_ref = oracle.decode_step(w, u, k, v, st_ref, sa_ref)
        xb = xbar.cpu().numpy()
        scale = np.abs(mu * x_t) + np.abs((1 - mu) * x_prev)
        assert np.all(np.abs(xb - xbar_ref) <= 1e-6 * np.maximum(scale, 1e-30)), f"xbar at step {s}"
        err = scaled_output_error(y.cpu().numpy(), y_ref, s_ref)
        assert err <= TOL_Y["f32"], f"y at step {s}: {err:.2e}"
        assert_state_close(st_gpu.cpu().numpy().reshape(3, -1), st_ref.reshape(3, -1), sa_ref.reshape(-1),
                           what=f"state after step {s}")
        worst = max(worst, err)
        x_prev, xp_gpu = x_t, xt_gpu


def test_unfused_decode_and_checkpoint_resume():
    """wkv_decode_step alone; and a state copied to the host mid-stream and reloaded
    continues bit for bit (the state is the whole session)."""
    import torch
    import linear_attention_rnn_wkv_b200 as wkv
    spec = _decode_case(3, 4, 64, 5100, steps=40)
    mu, w, u = synth.decode_params(spec)
    st32, sacc = _warm_state(spec)
    shape3 = (spec.N, spec.L, spec.C)
    w_g, u_g = to_gpu(w), to_gpu(u)
    st_a = to_gpu(st32.reshape((3,) + shape3))
    st_ref = st32.reshape((3,) + shape3).astype(np.float64)
    sa_ref = sacc.reshape(shape3)
    ys = []
    for s in range(spec.steps):
        _, k, v = synth.decode_step_inputs(spec, s)
        y = wkv.wkv_decode_step(w_g, u_g, to_gpu(k), to_gpu(v), st_a)
        y_ref, s_ref, st_ref, sa_ref = oracle.decode_step(w, u, k, v, st_ref, sa_ref)
        ys.append(y.cpu().numpy())
        assert scaled_output_error(ys[-1], y_ref, s_ref) <= TOL_Y["f32"]
        assert_state_close(st_a.cpu().numpy().reshape(3, -1), st_ref.reshape(3, -1), sa_ref.reshape(-1))
    # resume through the host at step 17
    st_b = to_gpu(st32.reshape((3,) + shape3))
    for s in range(spec.steps):
        if s == 17:
            saved = st_b.cpu().numpy().copy()
            del st_b
            st_b = torch.from_numpy(saved).cuda()
        _, k, v = synth.decode_step_inputs(spec, s)
        y = wkv.wkv_decode_step(w_g, u_g, to_gpu(k), to_gpu(v), st_b)
        assert np.array_equal(y.cpu().numpy(), ys[s])
    assert torch.equal(st_a, st_b)


@pytest.mark.parametrize("path,chunk", [("serial", 0), ("chunked", 8)])
def test_prefill_then_decode(path, chunk):
    """The forward's state_out continues the same sequences in the decode step (L = 1, N = B)."""
    import linear_attention_rnn_wkv_b200 as wkv
    B, T, C, extra = 4, 97, 48, 20
    spec = synth.ForwardSpec("pd", B, T + extra, C, "f32", 3.0, -5.0, 1.0, 0.01, 40.0, 5200)
    w, u, k, v = synth.forward_inputs(spec)
    y_ref, s_ref, st_ref, sa_ref = oracle.wkv_recurrent(w, u, k, v)
    y_pre, st = gpu_forward(w, u, k[:, :T], v[:, :T], path=path, chunk=chunk)
    assert scaled_output_error(y_pre, y_ref[:, :T], s_ref[:, :T]) <= TOL_Y["f32"]
    st_g = to_gpu(st.reshape(3, B, 1, C))
    w2, u2 = to_gpu(w.reshape(1, C)), to_gpu(u.reshape(1, C))
    for t in range(T, T + extra):
        y = wkv.wkv_decode_step(w2, u2, to_gpu(k[:, t:t + 1].copy()), to_gpu(v[:, t:t + 1].copy()), st_g)
        err = scaled_output_error(y.cpu().numpy()[:, 0], y_ref[:, t], s_ref[:, t])
        assert err <= TOL_Y["f32"], (t, err)
    assert_state_close(st_g.cpu().numpy().reshape(3, B, C), st_ref, sa_ref)


def test_full_size_decode_128_distinct_steps():
    """256 sessions x 32 layers x 4096 channels, 128 consecutive fused steps in the benchmark's
    launch configuration, each step's x, k, v drawn afresh from the counter-based generator.
    16384 sampled row-channels start from the oracle's 512-token warm-up, the rest from a valid
    filler state that the oracle carries as well (channels are independent), so every
    row-channel is checked: y and xbar after every step (on the device, in fp64, against the
    oracle's values), the whole state canonically after steps 0, 63 and 127, and the sampled
    row-channels' state after every step."""
    import torch
    import linear_attention_rnn_wkv_b200 as wkv
    spec = synth.DECODE["decode_256x32x4096"]
    n_all = spec.N * spec.L * spec.C
    shape3 = (spec.N, spec.L, spec.C)
    rng = np.random.default_rng(2024)
    flat = np.sort(rng.choice(n_all, 16384, replace=False))
    flat[0], flat[-1] = 0, n_all - 1  # include both ends
    mu, w, u = synth.decode_params(spec)
    st_host = synth.filler_state(spec).reshape(3, -1)
    st32, sacc = _warm_state(spec, flat)
    st_host[:, flat] = st32
    st_gpu = torch.from_numpy(st_host.reshape((3,) + shape3)).cuda()
    # the oracle's state and magnitude accumulator for every row-channel
    st_ref = st_host.astype(np.float64).reshape((3,) + shape3)
    sa_ref = np.abs(st_ref[0])
    sa_ref.reshape(-1)[flat] = sacc
    del st_host
    x_prev = synth.warmup_last_x(spec)
    xp_gpu = torch.from_numpy(x_prev).cuda()
    mu_g, w_g, u_g = to_gpu(mu), to_gpu(w), to_gpu(u)
    xbar = torch.empty(shape3, device="cuda")
    y = torch.empty(shape3, device="cuda")
    idx = torch.from_numpy(flat).cuda()
    for s in range(spec.steps):
        x_t, k, v = synth.decode_step_inputs(spec, s)
        xt_gpu = torch.from_numpy(x_t).cuda()
        wkv.wkv_decode_step_fused(mu_g, w_g, u_g, xt_gpu, xp_gpu, torch.from_numpy(k).cuda(),
                                  torch.from_numpy(v).cuda(), st_gpu, xbar=xbar, y=y)
        xbar_ref = oracle.decode_token_shift(mu, x_t, x_prev)
        y_ref, s_ref, st_ref, sa_ref = oracle.decode_step(w, u, k, v, st_ref, sa_ref)
        yerr = ((y.double() - torch.from_numpy(y_ref).cuda()).abs() / torch.from_numpy(s_ref).cuda()).max().item()
        assert torch.isfinite(y).all().item(), f"step {s}: non-finite y"
        assert yerr <= TOL_Y["f32"], f"y at step {s}: {yerr:.2e}"
        scale = torch.from_numpy(np.abs(mu * x_t) + np.abs((1 - mu) * x_prev)).cuda().clamp_min(1e-30)
        xerr = ((xbar.double() - torch.from_numpy(xbar_ref).cuda()).abs() / scale).max().item()
        assert xerr <= 1e-6, f"xbar at step {s}: {xerr:.2e}"
        stg = st_gpu.reshape(3, -1)[:, idx].cpu().numpy()
        assert_state_close(stg, st_ref.reshape(3, -1)[:, flat], sa_ref.reshape(-1)[flat], tol=TOL_STATE,
                           what=f"sampled state after step {s}")
        if s in (0, 63, spec.steps - 1):
            assert_state_close(st_gpu.cpu().numpy().reshape(3, -1), st_ref.reshape(3, -1), sa_ref.reshape(-1),
                               tol=TOL_STATE, what=f"whole state after step {s}")
        x_prev, xp_gpu = x_t, xt_gpu
