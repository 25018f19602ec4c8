"""The no-allocation chunked forward (wkv_forward_chunked_noalloc).

Some callers cannot call cudaMalloc (they run inside another framework's memory pool or
under a budget that forbids device allocations after start-up).  For them the library
offers the chunked forward with its scratch in a fixed device array inside the library.
These tests call it through the C ABI, several times in a row, and check every result
against the ordinary entry point (wkv_forward_ex, chunked path, caller-owned workspace)
and against the fp64 oracle, within the tolerances the other parity tests use.  The
calls alternate between the pipelined kernel (rows of a multiple of 16 bytes) and the
one-tile-per-block kernel (ragged rows), whose records sit differently in the shared
array, with no synchronisation between them.  The file is collected last.
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


class _Case:
    """Inputs of one shape, on the host and the device, with the oracle's and the workspace
    entry point's results."""

    def __init__(self, B, T, C, dtype, seed):
        import torch
        import linear_attention_rnn_wkv_b200 as wkv
        self.B, self.T, self.C, self.dtype = B, T, C, dtype
        td = torch.float32 if dtype == "f32" else torch.bfloat16
        spec = synth.ForwardSpec("noalloc", B, T, C, dtype, 3.0, -5.0, 1.0, 0.01, 40.0, seed)
        w, u, k, v = synth.forward_inputs(spec)
        r = np.random.default_rng(seed)
        st_in = np.stack([np.abs(r.normal(0, 1, (B, C))) + 1, np.abs(r.normal(0, 1, (B, C))) + 1,
                          r.normal(0, 1, (B, C))]).astype(np.float32)
        st_in[0] *= np.sign(r.normal(0, 1, (B, C))).astype(np.float32)
        self.st_in = st_in
        self.wg, self.ug = torch.from_numpy(w).cuda(), torch.from_numpy(u).cuda()
        self.kg, self.vg = torch.from_numpy(k).cuda().to(td), torch.from_numpy(v).cuda().to(td)
        self.sig = torch.from_numpy(st_in).cuda()
        y_ref, st_ref = wkv.wkv_forward(self.wg, self.ug, self.kg, self.vg, state_in=self.sig, path="chunked")
        torch.cuda.synchronize()
        self.y_ws = y_ref.float().cpu().numpy()
        self.st_ws = st_ref.cpu().numpy().astype(np.float64)
        self.y_o, self.s_o, self.st_o, self.sa_o = oracle.wkv_recurrent(
            w, u, k, v, state_in=st_in.astype(np.float64), sacc_in=np.abs(st_in[0]).astype(np.float64))

    def launch(self, noalloc):
        """Enqueue one no-allocation call into NaN-filled outputs; returns (status, y, state)."""
        import torch
        y = torch.full_like(self.kg, float("nan"))
        st = torch.full((3, self.B, self.C), float("nan"), device="cuda")
        rc = noalloc(self.B, self.T, self.C, 0 if self.dtype == "f32" else 1, self.wg.data_ptr(),
                     self.ug.data_ptr(), self.kg.data_ptr(), self.vg.data_ptr(), self.sig.data_ptr(),
                     y.data_ptr(), st.data_ptr(), torch.cuda.current_stream().cuda_stream)
        return rc, y, st

    def check(self, y, st, what):
        yn = y.float().cpu().numpy()
        assert np.all(np.isfinite(yn)), what
        tol = TOL_Y[self.dtype]
        assert scaled_output_error(yn, self.y_o, self.s_o) <= tol, f"{what}: y vs oracle"
        assert scaled_output_error(yn, self.y_ws, self.s_o) <= tol, f"{what}: y vs workspace path"
        stn = st.cpu().numpy()
        assert_state_close(stn, self.st_o, self.sa_o, what=f"{what} vs oracle")
        # the oracle's magnitude accumulator, moved to the workspace state's exponent, scales
        # the a-plane error against that state
        assert_state_close(stn, self.st_ws, self.sa_o * np.exp(self.st_o[2] - self.st_ws[2]),
                           what=f"{what} vs workspace path")


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_noalloc_matches_workspace_entry_point_twice(dtype):
    import torch
    import linear_attention_rnn_wkv_b200 as wkv
    noalloc = _noalloc(wkv.lib())
    case = _Case(3, 700, 264, dtype, 9100)
    for call in range(2):
        rc, y, st = case.launch(noalloc)
        assert rc == 0, wkv.STATUS.get(rc, rc)
        torch.cuda.synchronize()
        case.check(y, st, f"call {call}")
    wkv.get_device_status()


def test_noalloc_alternating_kernels_on_one_stream():
    """Pipelined, ragged, pipelined, ragged (fp32 and bf16): each call reuses the array the
    previous one left behind, with a different record layout, and nothing waits between them."""
    import torch
    import linear_attention_rnn_wkv_b200 as wkv
    noalloc = _noalloc(wkv.lib())
    cases = [_Case(3, 700, 264, "f32", 9200), _Case(2, 517, 37, "f32", 9201), _Case(2, 300, 136, "bf16", 9202),
             _Case(3, 333, 37, "bf16", 9203)]
    order = [0, 1, 2, 3, 0, 3, 1, 2]
    outs = []
    for i in order:
        rc, y, st = cases[i].launch(noalloc)
        assert rc == 0, wkv.STATUS.get(rc, rc)
        outs.append((i, y, st))
    torch.cuda.synchronize()
    for n, (i, y, st) in enumerate(outs):
        c = cases[i]
        cases[i].check(y, st, f"call {n} ({c.B}x{c.T}x{c.C} {c.dtype})")
    wkv.get_device_status()


def test_noalloc_without_tokens_passes_the_state_through():
    import torch
    import linear_attention_rnn_wkv_b200 as wkv
    noalloc = _noalloc(wkv.lib())
    B, C = 2, 40
    w = torch.ones(C, device="cuda")
    st_in = torch.randn((3, B, C), device="cuda")
    st = torch.full((3, B, C), float("nan"), device="cuda")
    s = torch.cuda.current_stream().cuda_stream
    assert noalloc(B, 0, C, 0, w.data_ptr(), w.data_ptr(), None, None, st_in.data_ptr(), None, st.data_ptr(), s) == 0
    torch.cuda.synchronize()
    assert torch.equal(st, st_in)
    # no state_in: the empty state (a = b = 0, p the empty exponent)
    assert noalloc(B, 0, C, 0, w.data_ptr(), w.data_ptr(), None, None, None, None, st.data_ptr(), s) == 0
    torch.cuda.synchronize()
    ref = torch.empty_like(st)
    lib = wkv.lib()
    ws = torch.zeros(64, dtype=torch.uint8, device="cuda")
    assert lib.wkv_forward_ex(B, 0, C, 0, w.data_ptr(), w.data_ptr(), None, None, None, None, ref.data_ptr(),
                              ws.data_ptr(), 64, 2, 0, s) == 0
    torch.cuda.synchronize()
    assert torch.equal(st, ref)


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
    assert noalloc(2, 3, 8, 0, 16, 16, None, 16, None, 16, None, None) == 1  # no k
    assert noalloc(0, 5, 8, 0, 16, 16, 16, 16, None, 16, None, None) == 0
    assert noalloc(2, 5, 8, 0, 16, 24, 16, 16, None, 16, None, None) == 2  # misaligned u
