"""Calls captured in one CUDA graph and replayed (GPU).

A replay repeats every launch with the same arguments, so the workspaces see the same shapes
again and again: the launch epoch that tags the published records must advance from replay to
replay (a record left by the previous replay must never read as fresh), and launches that may
overlap their predecessor must still see its writes.  One graph holds two forwards on different
inputs that share one workspace, a backward and an Eagle prefill; after each of three replays
every output is checked against the oracle."""
import numpy as np
import pytest

import oracle
import synth
from parity_util import TOL_Y, scaled_output_error, to_gpu

pytestmark = pytest.mark.gpu

TOL_EAGLE = 1e-4


def test_graph_replays_match_the_oracle():
    import torch
    import linear_attention_rnn_wkv_b200 as wkv
    B, T, C = 2, 700, 256
    sa = synth.forward_spec_like("fwd_8x1024x768", B, T, C, seed=9801)
    sb = synth.forward_spec_like("fwd_8x1024x768", B, T, C, seed=9802)
    wa, ua, ka, va = synth.forward_inputs(sa)
    wb, ub, kb, vb = synth.forward_inputs(sb)
    gy = synth.grad_output(sa)
    se = synth.eagle_spec_like("eagle_8x1024x768", 2, 300, 256, seed=9803)
    ew, er, ek, ev = synth.eagle_inputs(se)
    g = {n: to_gpu(a) for n, a in (("wa", wa), ("ua", ua), ("ka", ka), ("va", va), ("wb", wb), ("ub", ub),
                                    ("kb", kb), ("vb", vb), ("gy", gy), ("ew", ew), ("er", er), ("ek", ek),
                                    ("ev", ev))}
    fws = wkv.Workspace(torch.device("cuda"), wkv.workspace_size(B, T, C))
    bws = torch.zeros(int(wkv.lib().wkv_backward_workspace_size(B, T, C)), dtype=torch.uint8, device="cuda")
    ya, yb = torch.empty_like(g["ka"]), torch.empty_like(g["kb"])
    sta, stb = (torch.empty((3, B, C), device="cuda") for _ in range(2))
    ey = torch.empty_like(g["ek"])
    est = torch.empty((se.B, se.C // 64, 64, 64), device="cuda")
    out = {}

    def calls():
        wkv.wkv_forward(g["wa"], g["ua"], g["ka"], g["va"], workspace=fws, y=ya, state_out=sta)
        wkv.wkv_forward(g["wb"], g["ub"], g["kb"], g["vb"], workspace=fws, y=yb, state_out=stb)
        out["bwd"] = wkv.wkv_backward(g["wa"], g["ua"], g["ka"], g["va"], g["gy"], workspace=bws)
        wkv.eagle_forward(g["ew"], g["er"], g["ek"], g["ev"], y=ey, state_out=est)

    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        calls()  # warm-up outside the capture (attributes, workspaces)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        calls()

    ref_a = oracle.wkv_recurrent(wa, ua, ka, va)
    ref_b = oracle.wkv_recurrent(wb, ub, kb, vb)
    rk, rv, rw, ru, (sk, sv, sw, su) = oracle.wkv_backward(wa, ua, ka, va, gy)
    ye_ref, se_ref, _ = oracle.eagle_recurrent(ew, er, ek, ev)
    for _ in range(3):
        for t in (ya, yb, ey):
            t.fill_(float("nan"))  # a replay that skipped a launch would leave these
        graph.replay()
        torch.cuda.synchronize()
        assert scaled_output_error(ya.cpu().numpy(), ref_a[0], ref_a[1]) <= TOL_Y["f32"]
        assert scaled_output_error(yb.cpu().numpy(), ref_b[0], ref_b[1]) <= TOL_Y["f32"]
        for name, gg, r, sc in zip(("gk", "gv", "gw", "gu"), out["bwd"], (rk, rv, rw, ru), (sk, sv, sw, su)):
            err = np.abs(gg.cpu().numpy() - r) / np.maximum(sc, 1e-30)
            assert err.max() <= 2e-4, f"{name}: {err.max():.3e}"
        eyh = ey.cpu().numpy()
        assert np.all(np.isfinite(eyh))
        assert float(np.max(np.abs(eyh - ye_ref) / np.maximum(se_ref, 1e-300))) <= TOL_EAGLE
    wkv.forward_status(fws.buf)  # no bounded wait gave up (raises otherwise)
    wkv.get_device_status()
