"""CUDA forward vs the fp64 oracle, element by element (GPU)."""
import numpy as np
import pytest

import oracle
import synth
from parity_util import TOL_Y, assert_state_close, gpu_forward, scaled_output_error

pytestmark = pytest.mark.gpu

PATHS = [("serial", 0), ("chunked", 4), ("chunked", 8), ("chunked", 16)]
SHAPES = [(1, 1, 1), (1, 2, 3), (2, 3, 5), (1, 63, 4), (3, 64, 32), (1, 65, 129), (2, 257, 36), (1, 64, 64),
          (2, 100, 768), (1, 33, 8), (1, 130, 136), (2, 128, 64), (1, 256, 72)]


def _inputs(B, T, C, base, dtype, seed):
    spec = synth.forward_spec_like(base, B, T, C, seed=seed)
    spec = synth.ForwardSpec(spec.name, B, T, C, dtype, spec.k_std, spec.w_lo, spec.w_hi, spec.spike_prob,
                             spec.spike_value, seed)
    return synth.forward_inputs(spec)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("path,chunk", PATHS)
@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: "x".join(map(str, s)))
def test_forward_matches_oracle(shape, path, chunk, dtype):
    B, T, C = shape
    base = "fwd_8x1024x768" if C % 2 else "fwd_64x64"
    w, u, k, v = _inputs(B, T, C, base, dtype, seed=7000 + B * 131 + T * 17 + C)
    y, st = gpu_forward(w, u, k, v, dtype, path=path, chunk=chunk)
    y_ref, s_ref, st_ref, sa_ref = oracle.wkv_recurrent(w, u, k, v)
    assert scaled_output_error(y, y_ref, s_ref) <= TOL_Y[dtype]
    assert_state_close(st, st_ref, sa_ref)
    if T <= 300:
        y_d, s_d = oracle.wkv_direct(w, u, k, v)
        assert scaled_output_error(y, y_d, s_d) <= TOL_Y[dtype]


@pytest.mark.parametrize("path,chunk", PATHS)
def test_first_position_is_v(path, chunk):
    w, u, k, v = _inputs(2, 40, 68, "fwd_8x1024x768", "f32", 11)
    y, _ = gpu_forward(w, u, k, v, path=path, chunk=chunk)
    assert np.array_equal(y[:, 0], v[:, 0])


@pytest.mark.parametrize("path,chunk", PATHS)
def test_key_shift_by_100(path, chunk):
    """k -> k + 100 (spikes reach 140, far past where e^k overflows fp32): y unchanged,
    no inf/NaN, and the state's exponent moves by 100."""
    w, u, k, v = _inputs(2, 200, 64, "fwd_8x1024x768", "f32", 12)
    k2 = (k + np.float32(100.0)).astype(np.float32)
    y, st = gpu_forward(w, u, k2, v, path=path, chunk=chunk)
    y_ref, s_ref, st_ref, sa_ref = oracle.wkv_recurrent(w, u, k2, v)
    assert scaled_output_error(y, y_ref, s_ref) <= TOL_Y["f32"]
    assert_state_close(st, st_ref, sa_ref, tol=2e-5)  # |p| ~ 100-140 carries 2^-24 * 140 per rounding


@pytest.mark.parametrize("path,chunk", PATHS)
def test_special_parameters(path, chunk):
    """u -> -inf (current token removed), w = 0 (running mean), w huge (two-tap softmax)."""
    B, T, C = 1, 70, 12
    r = np.random.default_rng(3)
    k = r.normal(0, 1, (B, T, C)).astype(np.float32)
    v = r.normal(0, 1, (B, T, C)).astype(np.float32)
    w = np.concatenate([np.zeros(4), np.full(4, 1e4), np.exp(r.uniform(-3, 1, 4))]).astype(np.float32)
    u = np.concatenate([np.zeros(4), r.normal(0, .5, 4), np.full(4, -1e4)]).astype(np.float32)
    y, st = gpu_forward(w, u, k, v, path=path, chunk=chunk)
    y_ref, s_ref, st_ref, sa_ref = oracle.wkv_recurrent(w, u, k, v)
    assert scaled_output_error(y, y_ref, s_ref) <= TOL_Y["f32"]
    kc = np.full((B, T, 4), 0.25, np.float32)
    y_mean, _ = gpu_forward(np.zeros(4, np.float32), np.zeros(4, np.float32), kc, v[..., :4], path=path, chunk=chunk)
    want = np.cumsum(v[..., :4].astype(np.float64), axis=1) / np.arange(1, T + 1)[None, :, None]
    assert np.max(np.abs(y_mean - want)) <= 1e-5


@pytest.mark.parametrize("path,chunk", PATHS)
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_resume_from_state(path, chunk, dtype):
    """Prefill in two pieces through state_out -> state_in gives the one-piece result."""
    B, T, C = 3, 150, 40
    w, u, k, v = _inputs(B, T, C, "fwd_8x1024x768", dtype, 13)
    y_ref, s_ref, st_ref, sa_ref = oracle.wkv_recurrent(w, u, k, v)
    for cut in (1, 37, 64, 149):
        y1, st1 = gpu_forward(w, u, k[:, :cut], v[:, :cut], dtype, path=path, chunk=chunk)
        y2, st2 = gpu_forward(w, u, k[:, cut:], v[:, cut:], dtype, state_in=st1, path=path, chunk=chunk)
        y = np.concatenate([y1, y2], axis=1)
        assert scaled_output_error(y, y_ref, s_ref) <= TOL_Y[dtype]
        assert_state_close(st2, st_ref, sa_ref)


def test_empty_and_degenerate_sizes():
    import torch
    import linear_attention_rnn_wkv_b200 as wkv
    w = torch.ones(8, device="cuda")
    u = torch.zeros(8, device="cuda")
    z = torch.zeros(2, 0, 8, device="cuda")
    y, st = wkv.wkv_forward(w, u, z, z)
    assert y.shape == (2, 0, 8)
    st = st.cpu().numpy()
    assert np.all(st[:2] == 0) and np.all(st[2] == np.float32(oracle.P_EMPTY))
    st_in = torch.randn(3, 2, 8, device="cuda")
    _, st2 = wkv.wkv_forward(w, u, z, z, state_in=st_in)
    assert torch.equal(st2, st_in)
    z0 = torch.zeros(0, 5, 8, device="cuda")
    y0, st0 = wkv.wkv_forward(w, u, z0, z0)
    assert y0.numel() == 0 and st0.numel() == 0


def test_misaligned_pointer_rejected():
    import torch
    import linear_attention_rnn_wkv_b200 as wkv
    L = wkv.lib()
    buf = torch.zeros(1 + 4 * 16, device="cuda")
    w = torch.ones(16, device="cuda")
    ws = wkv.Workspace(nbytes=wkv.workspace_size(1, 4, 16))
    st = L.wkv_forward(1, 4, 16, 0, w.data_ptr(), w.data_ptr(), buf.data_ptr() + 4, buf.data_ptr(), buf.data_ptr(),
                       None, ws.buf.data_ptr(), ws.buf.numel(), None)
    assert st == 2


def test_auto_path_matches_explicit_paths():
    for (B, T, C) in [(8, 1024, 768), (1, 16384, 4096), (4, 4096, 2048)]:
        import linear_attention_rnn_wkv_b200 as wkv
        assert wkv.auto_path(B, T, C) in ("serial", "chunked")
    w, u, k, v = _inputs(2, 300, 256, "fwd_8x1024x768", "f32", 14)
    y_a, st_a = gpu_forward(w, u, k, v)
    y_ref, s_ref, st_ref, sa_ref = oracle.wkv_recurrent(w, u, k, v)
    assert scaled_output_error(y_a, y_ref, s_ref) <= TOL_Y["f32"]
    assert_state_close(st_a, st_ref, sa_ref)


def test_token_shift_forward_mode():
    import torch
    import linear_attention_rnn_wkv_b200 as wkv
    for (B, T, C) in [(2, 9, 64), (1, 5, 37), (3, 1, 8)]:
        r = np.random.default_rng(B * 100 + C)
        mu = r.uniform(0, 1, C).astype(np.float32)
        x = r.normal(0, 1, (B, T, C)).astype(np.float32)
        xl = r.normal(0, 1, (B, C)).astype(np.float32)
        for last in (None, xl):
            xb = wkv.token_shift_mix(torch.from_numpy(mu).cuda(), torch.from_numpy(x).cuda(),
                                     None if last is None else torch.from_numpy(last).cuda()).cpu().numpy()
            ref = oracle.token_shift(mu, x, last)
            prev = np.concatenate([np.zeros((B, 1, C)) if last is None else last[:, None], x[:, :-1]], axis=1)
            scale = np.abs(mu * x) + np.abs((1 - mu) * prev)
            assert np.all(np.abs(xb - ref) <= 1e-6 * np.maximum(scale, 1e-30))
        ones = wkv.token_shift_mix(torch.ones(C, device="cuda"), torch.from_numpy(x).cuda()).cpu().numpy()
        assert np.array_equal(ones, x)
