"""The no-allocation chunked forward (wkv_forward_chunked_noalloc).

Some callers cannot call cudaMalloc (they run inside another framework's memory pool or
under a budget that forbids device allocations after start-up).  For them the library
offers the chunked forward with its scratch in a fixed device array inside the library.
This test calls it through the C ABI, twice in a row, and checks both results against
the ordinary entry point (wkv_forward_ex, chunked path, caller-owned workspace) within
the tolerances the other parity tests use.  It sits in its own file, collected last.
"""
import ctypes

import numpy as np
import pytest

import oracle
import synth
from parity_util import TOL_Y, assert_state_close, scaled_output_error

pytestmark = pytest.mark.gpu


def _noalloc(L):
    f = L.wkv_forward_chunked_noalloc
    i64, vp = ctypes.c_int64, ctypes.c_void_p
    f.argtypes = [i64, i64, i64, ctypes.c_int, vp, vp, vp, vp, vp, vp, vp, vp]
    f.restype = ctypes.c_int
    return f


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_noalloc_matches_workspace_entry_point_twice(dtype):
    import torch
    import linear_attention_rnn_wkv_b200 as wkv
    L = wkv.lib()
    noalloc = _noalloc(L)
    td = torch.float32 if dtype == "f32" else torch.bfloat16
    B, T, C = 3, 700, 264
    spec = synth.ForwardSpec("noalloc", B, T, C, dtype, 3.0, -5.0, 1.0, 0.01, 40.0, 9100)
    w, u, k, v = synth.forward_inputs(spec)
    st_in = np.stack([np.abs(np.random.default_rng(1).normal(0, 1, (B, C))) + 1,
                      np.abs(np.random.default_rng(2).normal(0, 1, (B, C))) + 1,
                      np.random.default_rng(3).normal(0, 1, (B, C))]).astype(np.float32)
    st_in[0] *= np.sign(np.random.default_rng(4).normal(0, 1, (B, C))).astype(np.float32)
    wg, ug = torch.from_numpy(w).cuda(), torch.from_numpy(u).cuda()
    kg, vg = torch.from_numpy(k).cuda().to(td), torch.from_numpy(v).cuda().to(td)
    sig = torch.from_numpy(st_in).cuda()
    stream = torch.cuda.current_stream().cuda_stream

    # ordinary entry point: chunked path with a caller-owned workspace
    y_ref, st_ref = wkv.wkv_forward(wg, ug, kg, vg, state_in=sig, path="chunked")
    torch.cuda.synchronize()
    y_ref = y_ref.float().cpu().numpy()
    st_ref = st_ref.cpu().numpy()

    # the oracle supplies the error scale (|v|-weighted average) and magnitude accumulator
    _, s_o, st_o, sa_o = oracle.wkv_recurrent(w, u, k, v, state_in=st_in.astype(np.float64),
                                               sacc_in=np.abs(st_in[0]).astype(np.float64))
    for call in range(2):
        y = torch.full_like(kg, float("nan"))
        st = torch.full((3, B, C), float("nan"), device="cuda")
        rc = noalloc(B, T, C, 0 if dtype == "f32" else 1, wg.data_ptr(), ug.data_ptr(), kg.data_ptr(),
                     vg.data_ptr(), sig.data_ptr(), y.data_ptr(), st.data_ptr(), stream)
        assert rc == 0, wkv.STATUS.get(rc, rc)
        torch.cuda.synchronize()
        yn = y.float().cpu().numpy()
        assert scaled_output_error(yn, y_ref, s_o) <= TOL_Y[dtype], f"call {call}"
        stn = st.cpu().numpy()
        # against the workspace path's state (the oracle's magnitude accumulator, moved to
        # that state's exponent, scales the a-plane error)
        st_ref64 = st_ref.astype(np.float64)
        assert_state_close(stn, st_ref64, sa_o * np.exp(st_o[2] - st_ref64[2]), what=f"call {call} vs workspace path")
        assert_state_close(stn, st_o, sa_o, what=f"call {call} vs oracle")


def test_noalloc_rejects_shapes_beyond_its_scratch():
    import torch
    import linear_attention_rnn_wkv_b200 as wkv
    noalloc = _noalloc(wkv.lib())
    # a shape whose scratch exceeds 32 MiB on every tile the library may pick
    # (65536 x 8192 channel-steps: at least 2 x 16 B x 8192 x 512 = 128 MiB of records):
    # refused before any launch
    need = wkv.workspace_size(1, 65536, 8192)
    assert need > 32 << 20
    rc = noalloc(1, 65536, 8192, 0, 16, 16, 16, 16, None, 16, None, torch.cuda.current_stream().cuda_stream)
    assert rc == 1  # WKV_ERR_INVALID_ARG
    assert noalloc(2, 0, 8, 0, 16, 16, 16, 16, None, 16, None, None) == 1
    assert noalloc(0, 5, 8, 0, 16, 16, 16, 16, None, 16, None, None) == 0
