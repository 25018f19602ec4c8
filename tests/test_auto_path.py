"""WKV_PATH_AUTO follows the measured path table, and on the GPU it is never slower than the
fastest explicit path by more than the timing noise.

The table (csrc/wkv_path_table.h) and the timings it came from (tune_b200.json) are written by
the package's tuning script on a B200; the library picks the winner of the nearest grid point.
"""
import json
import os
import statistics

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
TIMINGS = os.path.join(ROOT, "linear_attention_rnn_wkv_b200", "tune_b200.json")


def _shape_for(bc):
    from linear_attention_rnn_wkv_b200.tune import shape_for
    return shape_for(bc)


def test_auto_path_follows_the_measured_table():
    import linear_attention_rnn_wkv_b200 as wkv
    L = wkv.lib()
    rows = json.load(open(TIMINGS))
    assert rows, "no measured grid points"
    for r in rows:
        B, C = _shape_for(r["BC"])
        got = L.wkv_forward_auto_path(B, r["T"], C, 1 if r["dtype"] == "bf16" else 0)
        want = 1 if r["best"] == "serial" else 2
        assert got == want, (r["dtype"], r["BC"], r["T"], r["best"])


def _time(fn, calls=20, replays=5):
    import torch
    for i in range(3):
        fn(i)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for i in range(calls):
            fn(i)
    g.replay()
    torch.cuda.synchronize()
    ms = []
    for _ in range(replays):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        g.replay()
        e1.record()
        torch.cuda.synchronize()
        ms.append(e0.elapsed_time(e1) / calls)
    del g
    return statistics.median(ms)


@pytest.mark.gpu
@pytest.mark.parametrize("shape", [(1, 16, 4096, "f32"), (64, 64, 4096, "f32"), (8, 1024, 768, "f32"),
                                   (4, 4096, 2048, "bf16"), (256, 16, 4096, "bf16"), (16, 256, 4096, "f32")],
                         ids=lambda s: "x".join(map(str, s)))
def test_auto_is_not_slower_than_the_best_explicit_path(shape):
    import torch
    import linear_attention_rnn_wkv_b200 as wkv
    B, T, C, dt = shape
    td = torch.bfloat16 if dt == "bf16" else torch.float32
    g = torch.Generator(device="cuda")
    g.manual_seed(77)
    w = torch.exp(torch.rand(C, generator=g, device="cuda") * 6 - 5)
    u = torch.randn(C, generator=g, device="cuda") * 0.5
    n_sets = max(1, min(4, int(3e8 // (3 * B * T * C * (2 if dt == "bf16" else 4))) + 1))
    sets = [tuple(torch.randn((B, T, C), generator=g, device="cuda").to(td) for _ in range(2)) + (
        torch.empty((B, T, C), dtype=td, device="cuda"), torch.empty((3, B, C), device="cuda")) for _ in range(n_sets)]
    ws = wkv.Workspace(nbytes=wkv.workspace_size(B, T, C, td))
    times = {}
    for name, (path, chunk) in {"auto": ("auto", 0), "serial": ("serial", 0), "chunked8": ("chunked", 8),
                                "chunked16": ("chunked", 16)}.items():
        def fn(i, path=path, chunk=chunk):
            k, v, y, st = sets[i % n_sets]
            wkv.wkv_forward(w, u, k, v, path=path, chunk=chunk, workspace=ws, y=y, state_out=st)
        times[name] = _time(fn)
    wkv.forward_status(ws.buf)
    best = min(v for k, v in times.items() if k != "auto")
    assert times["auto"] <= 1.15 * best + 0.003, times
