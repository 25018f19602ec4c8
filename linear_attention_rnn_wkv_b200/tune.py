"""Measure which forward path is fastest over a grid of shapes and write the table that
WKV_PATH_AUTO follows.

    python -m linear_attention_rnn_wkv_b200.tune [--out PATH] [--json PATH]

For every grid point (I/O dtype, channels B*C, tokens T) the forward runs on each
candidate -- the serial path (one thread per channel over all of T) and the chunked path
with 8- and 16-step chunks -- as back-to-back launches captured in a CUDA graph, on
rotating input sets larger than twice the L2, and the median of five replays is kept.
The winner of each point goes into a C header (csrc/wkv_path_table.h by default), which
the library's path choice reads; rebuild the library afterwards.  The inputs follow the
long-context forward workload's distributions (keys N(0, 3) with 1% at +40, values
N(0, 1), w = exp(U(-5, 1)), u ~ N(0, 0.5)).
"""
from __future__ import annotations

import argparse
import datetime
import json
import os
import statistics

import torch

from . import Workspace, wkv_forward, workspace_size

HERE = os.path.dirname(os.path.abspath(__file__))
TABLE = os.path.join(HERE, "csrc", "wkv_path_table.h")

# grid: channels B*C and tokens T (log-spaced); a point is measured when its elements fit
GRID_BC = (64, 512, 4096, 32768, 262144, 1048576)
GRID_T = (1, 4, 16, 64, 256, 1024, 4096, 16384)
MAX_ELEMENTS = 1 << 28
CANDIDATES = (("serial", 0), ("chunked", 8), ("chunked", 16))
CODE = {("serial", 0): 1, ("chunked", 8): 8, ("chunked", 16): 16}
L2_BYTES = 126e6


def shape_for(bc):
    """B and C for a channel count: C up to 4096 (a multiple of 64), the rest in B."""
    c = min(bc, 4096)
    return bc // c, c


def time_point(bc, t, dtype, dev):
    B, C = shape_for(bc)
    td = torch.bfloat16 if dtype == "bf16" else torch.float32
    esz = 2 if dtype == "bf16" else 4
    per_set = 3 * B * t * C * esz
    n_sets = max(1, min(6, int(2 * L2_BYTES // per_set) + 1))
    g = torch.Generator(device=dev)
    g.manual_seed(1004 + bc + t)
    w = torch.exp(torch.rand(C, generator=g, device=dev) * 6 - 5)
    u = torch.randn(C, generator=g, device=dev) * 0.5
    sets = []
    for _ in range(n_sets):
        k = torch.randn((B, t, C), generator=g, device=dev) * 3
        k = torch.where(torch.rand((B, t, C), generator=g, device=dev) < 0.01, torch.full_like(k, 40.0), k)
        v = torch.randn((B, t, C), generator=g, device=dev)
        sets.append((k.to(td), v.to(td), torch.empty((B, t, C), dtype=td, device=dev),
                     torch.empty((3, B, C), device=dev)))
    ws = Workspace(dev, workspace_size(B, t, C, td))
    calls = max(n_sets, min(40, int(4e6 / (B * t * C)) + 2))
    out = {}
    for path, chunk in CANDIDATES:
        def fn(i):
            k, v, y, st = sets[i % n_sets]
            wkv_forward(w, u, k, v, path=path, chunk=chunk, workspace=ws, y=y, state_out=st)

        for i in range(n_sets):
            fn(i)
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            for i in range(calls):
                fn(i)
        graph.replay()
        torch.cuda.synchronize()
        ms = []
        for _ in range(5):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            graph.replay()
            e1.record()
            torch.cuda.synchronize()
            ms.append(e0.elapsed_time(e1) / calls)
        del graph
        out[f"{path}{chunk}" if chunk else path] = statistics.median(ms)
    del sets, ws
    torch.cuda.empty_cache()
    return out


def write_header(path, table, device_name):
    lines = [
        "// Fastest forward path per (I/O dtype, channels B*C, tokens T), measured on " + device_name,
        "// by linear_attention_rnn_wkv_b200/tune.py on " + datetime.date.today().isoformat() + " (CUDA-event",
        "// timings of back-to-back launches on inputs larger than the L2).  Entries: 1 the serial",
        "// path, 8 or 16 the chunked path with that chunk length; 0 a point not measured (too",
        "// large), which takes its nearest measured neighbour in T.  Regenerate with the tuning",
        "// script and rebuild the library.",
        "#pragma once",
        "",
        "namespace wkvb {",
        "",
        f"constexpr int kTuneNumBC = {len(GRID_BC)};",
        f"constexpr int kTuneNumT = {len(GRID_T)};",
        "constexpr long long kTuneBC[kTuneNumBC] = {" + ", ".join(str(x) for x in GRID_BC) + "};",
        "constexpr long long kTuneT[kTuneNumT] = {" + ", ".join(str(x) for x in GRID_T) + "};",
        "// [dtype: 0 fp32, 1 bf16][B*C][T]",
        "constexpr signed char kTunePath[2][kTuneNumBC][kTuneNumT] = {",
    ]
    for d in ("f32", "bf16"):
        lines.append("    {")
        for bc in GRID_BC:
            row = [str(table[d].get((bc, t), 0)) for t in GRID_T]
            lines.append("        {" + ", ".join(row) + "},  // B*C = " + str(bc))
        lines.append("    },")
    lines += ["};", "", "}  // namespace wkvb", ""]
    with open(path, "w") as f:
        f.write("\n".join(lines))


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--out", default=TABLE, help="header to write")
    ap.add_argument("--json", default=None, help="also write every timing here")
    args = ap.parse_args()
    dev = torch.device("cuda", 0)
    table = {"f32": {}, "bf16": {}}
    rows = []
    for d in ("f32", "bf16"):
        for bc in GRID_BC:
            for t in GRID_T:
                if bc * t > MAX_ELEMENTS:
                    continue
                ms = time_point(bc, t, d, dev)
                best = min(ms, key=ms.get)
                code = {"serial": 1, "chunked8": 8, "chunked16": 16}[best]
                table[d][(bc, t)] = code
                rows.append({"dtype": d, "BC": bc, "T": t, "ms": ms, "best": best})
                print(json.dumps(rows[-1]), flush=True)
    write_header(args.out, table, torch.cuda.get_device_name(dev))
    if args.json:
        with open(args.json, "w") as f:
            json.dump(rows, f, indent=1)


if __name__ == "__main__":
    main()
