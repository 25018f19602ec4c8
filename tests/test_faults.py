"""Failure detection without a GPU fault: a bounded device-side wait that runs out
returns an error status the host reads, and the CUDA context stays usable."""
import numpy as np
import pytest

import oracle
import synth
from parity_util import TOL_Y, gpu_forward, scaled_output_error

pytestmark = pytest.mark.gpu


def test_missing_carry_times_out_and_context_survives():
    import torch
    import linear_attention_rnn_wkv_b200 as wkv
    L = wkv.lib()
    B, T, C = 1, 512, 128          # chunked: 16 time segments of 32 steps, one channel group
    spec = synth.forward_spec_like("fwd_8x1024x768", B, T, C, seed=77)
    w, u, k, v = synth.forward_inputs(spec)
    wg, ug, kg, vg = (torch.from_numpy(a).cuda() for a in (w, u, k, v))
    y = torch.empty_like(kg)
    ws = wkv.Workspace(nbytes=wkv.workspace_size(B, T, C))
    stream = torch.cuda.current_stream().cuda_stream
    L.wkv_get_device_status(stream)  # start from a clear device-wide word
    # unit 5 never publishes its carry; waits give up after 20000 polls (milliseconds)
    st = L.wkv_testhook_forward_drop(B, T, C, wg.data_ptr(), ug.data_ptr(), kg.data_ptr(), vg.data_ptr(),
                                     y.data_ptr(), ws.buf.data_ptr(), ws.buf.numel(), 5, 20000, stream)
    assert st == 0
    assert L.wkv_forward_status(ws.buf.data_ptr(), ws.buf.numel(), stream) == 5  # WKV_ERR_TIMEOUT
    # the device-wide word saw it too, independently of the workspace
    assert L.wkv_get_device_status(stream) == 5
    # both errors were cleared and the same workspace and context work again
    assert L.wkv_forward_status(ws.buf.data_ptr(), ws.buf.numel(), stream) == 0
    assert L.wkv_get_device_status(stream) == 0
    y2, _ = wkv.wkv_forward(wg, ug, kg, vg, workspace=ws, path="chunked")
    wkv.forward_status(ws.buf)
    wkv.get_device_status()
    y_ref, s_ref, _, _ = oracle.wkv_recurrent(w, u, k, v)
    assert scaled_output_error(y2.cpu().numpy(), y_ref, s_ref) <= TOL_Y["f32"]


def test_status_is_clean_after_normal_runs():
    import linear_attention_rnn_wkv_b200 as wkv
    w, u, k, v = synth.forward_inputs(synth.forward_spec_like("fwd_64x64", 2, 200, 96))
    gpu_forward(w, u, k, v, path="serial")
    wkv.forward_status()  # the library's own status word (serial path, no workspace)
    ws = wkv.Workspace(nbytes=wkv.workspace_size(2, 200, 96))
    import torch
    wkv.wkv_forward(*(torch.from_numpy(a).cuda() for a in (w, u, k, v)), workspace=ws)
    wkv.forward_status(ws.buf)
    wkv.get_device_status()  # no launch on the device gave up a wait
