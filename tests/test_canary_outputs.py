"""Every entry point writes exactly its outputs: each output is a view into a NaN-filled buffer
with canary padding on both sides; after the call the canaries are intact (nothing written
outside the output) and no output element is still NaN (nothing left unwritten)."""
import numpy as np
import pytest

import synth
from parity_util import to_gpu

pytestmark = pytest.mark.gpu

CANARY = 12288.0  # exact in fp32 and bf16
PAD = 64          # elements on each side (keeps 16-byte alignment)


def _padded(shape, dtype):
    import torch
    n = int(np.prod(shape))
    buf = torch.full((n + 2 * PAD,), float("nan"), dtype=dtype, device="cuda")
    buf[:PAD] = CANARY
    buf[-PAD:] = CANARY
    return buf, buf[PAD:PAD + n].view(*shape)


def _check(buf, out, what):
    import torch
    torch.cuda.synchronize()
    b = buf.float().cpu().numpy()
    assert np.all(b[:PAD] == CANARY) and np.all(b[-PAD:] == CANARY), f"{what}: wrote outside its output"
    assert np.all(np.isfinite(out.float().cpu().numpy())), f"{what}: output left unwritten"


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("path,chunk", [("auto", 0), ("serial", 0), ("chunked", 4)])
@pytest.mark.parametrize("shape", [(2, 77, 96), (1, 300, 64), (3, 5, 36)], ids=lambda s: "x".join(map(str, s)))
def test_forward_writes_exactly_its_outputs(shape, path, chunk, dtype):
    import torch
    import linear_attention_rnn_wkv_b200 as wkv
    B, T, C = shape
    spec = synth.forward_spec_like("fwd_8x1024x768", B, T, C, seed=7100 + T)
    spec = synth.ForwardSpec(spec.name, B, T, C, dtype, spec.k_std, spec.w_lo, spec.w_hi, spec.spike_prob,
                             spec.spike_value, spec.seed)
    w, u, k, v = synth.forward_inputs(spec)
    td = torch.float32 if dtype == "f32" else torch.bfloat16
    ybuf, y = _padded((B, T, C), td)
    sbuf, st = _padded((3, B, C), torch.float32)
    wkv.wkv_forward(to_gpu(w), to_gpu(u), to_gpu(k, td), to_gpu(v, td), y=y, state_out=st, path=path, chunk=chunk)
    _check(ybuf, y, "y")
    _check(sbuf, st, "state_out")


def test_eagle_writes_exactly_its_outputs():
    import torch
    import linear_attention_rnn_wkv_b200 as wkv
    for (B, T, C) in [(2, 70, 128), (1, 1, 64), (1, 200, 64)]:
        spec = synth.eagle_spec_like("eagle_8x1024x768", B, T, C, seed=7200 + T)
        w, r, k, v = synth.eagle_inputs(spec)
        ybuf, y = _padded((B, T, C), torch.float32)
        sbuf, st = _padded((B, C // 64, 64, 64), torch.float32)
        wkv.eagle_forward(to_gpu(w), to_gpu(r), to_gpu(k), to_gpu(v), y=y, state_out=st)
        _check(ybuf, y, "eagle y")
        _check(sbuf, st, "eagle state_out")


def test_decode_and_shift_write_exactly_their_outputs():
    import torch
    import linear_attention_rnn_wkv_b200 as wkv
    N, L, C = 3, 2, 100
    g = np.random.default_rng(7300)
    f32 = lambda *s: g.normal(0, 1, s).astype(np.float32)
    mu = g.uniform(0, 1, (L, C)).astype(np.float32)
    w = np.exp(g.uniform(-5, 1, (L, C))).astype(np.float32)
    u = (0.5 * f32(L, C)).astype(np.float32)
    state = np.stack([f32(N, L, C), np.abs(f32(N, L, C)) + 1, f32(N, L, C)]).astype(np.float32)
    sbuf, st = _padded((3, N, L, C), torch.float32)
    st.copy_(to_gpu(state))
    xbuf, xbar = _padded((N, L, C), torch.float32)
    ybuf, y = _padded((N, L, C), torch.float32)
    wkv.wkv_decode_step_fused(to_gpu(mu), to_gpu(w), to_gpu(u), to_gpu(f32(N, L, C)), to_gpu(f32(N, L, C)),
                              to_gpu(f32(N, L, C)), to_gpu(f32(N, L, C)), st, xbar=xbar, y=y)
    _check(xbuf, xbar, "xbar")
    _check(ybuf, y, "decode y")
    _check(sbuf, st, "decode state")

    B, T = 2, 33
    tbuf, xb = _padded((B, T, C), torch.float32)
    wkv.token_shift_mix(to_gpu(mu[0]), to_gpu(f32(B, T, C)), xbar=xb)
    _check(tbuf, xb, "token shift")

    Ce = 128
    we = np.exp(g.uniform(-5, 1, (1, Ce))).astype(np.float32)
    ebuf, es = _padded((N, 1, Ce // 64, 64, 64), torch.float32)
    es.copy_(to_gpu(f32(N, 1, Ce // 64, 64, 64)))
    eybuf, ey = _padded((N, 1, Ce), torch.float32)
    wkv.eagle_decode_step(to_gpu(we), to_gpu(f32(N, 1, Ce)), to_gpu(f32(N, 1, Ce)), to_gpu(f32(N, 1, Ce)), es, y=ey)
    _check(eybuf, ey, "eagle decode y")
    _check(ebuf, es, "eagle decode state")
