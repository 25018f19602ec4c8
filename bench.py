#!/usr/bin/env python
"""Benchmark of the RWKV-4 WKV operator on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Headline workload (one step = one pass of the whole hot path over one batch): the prefill
of the largest forward configuration, B=1 sequence x T=16384 tokens x C=4096 channels in
fp32 (keys N(0,3) with 1% set to +40, values N(0,1), w = exp(U(-5,1)), u ~ N(0,0.5))
through wkv_forward, which also returns the final state, then one fused decode step (token
shift + WKV update) that continues the sequence from that state.  Metric: WKV forward
B*T*C elements/s.

Timing: W untimed warm-up steps, then the K-step CUDA graph is replayed R times; each
replay is exactly K steps, bracketed by a barrier and a device synchronise and timed with
CUDA events on the launching stream; the median replay gives ms_per_step, and the max over
ranks is taken.  The inputs of one step (805 MB) are over six times the 126 MB L2, so no
step finds its inputs in L2.  The forward kernel's own launch duration (for the roofline)
is timed right after: a graph of back-to-back forwards, events around whole replays.

The same JSON line carries one row per benchmark configuration ("configs": the four
forward workloads and the 256 x 32 x 4096 decode step), each timed the same way on
rotating input sets larger than twice the L2, with its algorithmic bandwidth, its fraction
of the measured copy peak and the fp64 oracle's rate on the host cores; and the next rows
(gated forward, three-mu token shift, backward, Eagle prefill and decode).

--impl reference times the fp64 CPU oracle (plain C, OpenMP) on the headline workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

WORKLOAD = "fwd_1x16384x4096"
METRIC = "WKV forward B*T*C elements/s"
L2_BYTES = 126e6
GRAPH_STEPS = 60
REPLAYS = 9
REF_CHANNELS = 512                                # channels per step of the CPU reference arm
ALG_BYTES_PER_ELEM = {"f32": 12, "bf16": 6}     # k + v read, y written, per element
DECODE_ALG_BYTES_PER_ELEM = 48                    # x_t, x_prev, k, v, a, b, p in; a, b, p, y, xbar out
FORWARD_CONFIGS = ("fwd_64x64", "fwd_8x1024x768", "fwd_4x4096x2048_bf16", "fwd_1x16384x4096")


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--no-configs", action="store_true", help="skip the per-configuration rows")
    ap.add_argument("--no-next", action="store_true", help="skip the next rows (gated, shift3, backward, Eagle)")
    ap.add_argument("--profile-forward", metavar="WORKLOAD", default=None,
                    help="only run 2 + 3 eager forward launches of a forward workload (e.g. fwd_1x16384x4096) "
                         "and exit: a short, self-contained command to capture under a profiler")
    ap.add_argument("--profile-step", action="store_true",
                    help="only run 3 + 2 eager headline steps (forward with state + fused decode) and exit")
    ap.add_argument("--profile-eagle", action="store_true",
                    help="only run 2 + 3 eager Eagle prefills on eagle_8x1024x768 and exit, for a profiler")
    ap.add_argument("--profile-backward", metavar="WORKLOAD", default=None,
                    help="only run 2 + 3 eager backward calls on a forward workload's shape (fp32) and exit, "
                         "for a profiler")
    return ap.parse_args()


# ----------------------------------------------------------------------------
# clocks
# ----------------------------------------------------------------------------

class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 50 ms in the background."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.samples = []
        self.proc = None
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.samples.append((time.time(), line.strip()))

    def stop(self):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
        if self.thread:
            self.thread.join(timeout=5)

    def summary(self, t0, t1):
        rows = [s for (t, s) in self.samples if t0 <= t <= t1]
        window = "timed"
        if len(rows) < 3:
            rows = [s for (t, s) in self.samples if t0 - 1.5 <= t <= t1 + 0.2]
            window = "timed+preroll"
        if not rows:
            return None
        mhz, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            p = [x.strip() for x in r.split(",")]
            try:
                mhz.append(float(p[1]))
                mx.append(float(p[2]))
            except (ValueError, IndexError):
                continue
            for name, val in zip(names, p[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(name)
        if not mhz:
            return None
        return {"sm_mhz": statistics.median(mhz), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(mhz), "window": window}


# ----------------------------------------------------------------------------
# helpers
# ----------------------------------------------------------------------------

def measured_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return json.load(f), "measured"
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0}, "fallback"


def kernel_source_digest():
    """A digest of the forward kernel's code (its sources with comments and whitespace
    removed), recorded in each committed ncu summary: a summary counts only while it matches."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "linear_attention_rnn_wkv_b200", "csrc")
    for name in ("wkv_device.cuh", "wkv_vec.cuh", "wkv_internal.h", "wkv_pipe_common.cuh", "wkv_forward_chunked.cu",
                 "wkv_forward_tmem.cu"):
        with open(os.path.join(csrc, name), encoding="utf-8") as f:
            code = re.sub(r"/\*.*?\*/", " ", f.read(), flags=re.S)
        code = re.sub(r"//[^\n]*", " ", code)
        h.update(re.sub(r"\s+", " ", code).encode())
    return h.hexdigest()[:16]


def profiled_traffic(workload):
    """DRAM bytes per launch of the forward kernel from the committed ncu summary, if it
    was taken on the current kernel source (else None), and the file it came from."""
    rel = os.path.join("profiles", f"tmem_kernel_{workload}.md")
    try:
        txt = open(os.path.join(ROOT, rel)).read()
    except OSError:
        return None, None
    m_src = re.search(r"kernel_source_digest:\s*([0-9a-f]+)", txt)
    m_tr = re.search(r"dram_bytes_per_launch:\s*([0-9.eE+]+)", txt)
    if not m_src or not m_tr or m_src.group(1) != kernel_source_digest():
        return None, None
    return float(m_tr.group(1)), rel


def dist_setup(n_gpus):
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    else:
        torch.cuda.set_device(0)
    return rank, world, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x, world):
    """The largest of every rank's x (a time): one all-reduce of a scalar, on the GPU under
    NCCL, on the host under gloo.  Every rank must call it, in the same order."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def rank_set_seed(base_seed, rank, i):
    """Seed of input set i on a rank: every rank draws its own batch (weak scaling)."""
    return base_seed + 100 * rank + i


def weak_scaling_value(world, n_elem_per_rank, ms_max):
    """Whole-job throughput: the elements all ranks processed over the slowest rank's time."""
    return world * n_elem_per_rank / (ms_max * 1e-3)


def sets_for(bytes_per_set, floor=1, cap=8):
    """Rotating input sets whose total exceeds twice the L2."""
    n = int(-(-2 * L2_BYTES // max(bytes_per_set, 1))) + 1
    return max(floor, min(cap, n))


# ----------------------------------------------------------------------------
# CPU oracle timing (cpu_baseline legs and --impl reference)
# ----------------------------------------------------------------------------

def time_oracle(spec, inputs, min_seconds, min_passes):
    import oracle
    w, u, k, v = inputs
    passes, t0 = 0, time.perf_counter()
    while True:
        oracle.wkv_recurrent(w, u, k, v)
        passes += 1
        el = time.perf_counter() - t0
        if passes >= min_passes and el >= min_seconds:
            break
    n = spec.B * spec.T * spec.C
    return n * passes / el, passes, el, oracle.num_threads()


def oracle_row(spec, seconds=2.0):
    """The fp64 oracle's stabilised recurrence on one forward workload, on the host cores,
    whole prefills of the workload for about `seconds` (at least one)."""
    import synth
    rate, passes, el, cores = time_oracle(spec, synth.forward_inputs(spec), seconds, 1)
    return {"value": rate, "unit": "elements/s", "cores": cores, "kind": "oracle",
            "sample": f"{passes} passes of the whole {spec.B}x{spec.T}x{spec.C} prefill through the fp64 "
                      f"stabilised recurrence ({el:.1f} s)"}


def oracle_decode_row(seconds=2.0, n_sample=32):
    """The fp64 oracle's decode step (one token through the stabilised recurrence, token shift
    included) on the first n_sample sessions of the 256 x 32 x 4096 decode workload."""
    import numpy as np
    import oracle
    import synth
    spec = synth.DECODE["decode_256x32x4096"]
    mu, w, u = synth.decode_params(spec)
    x_t, k, v = (np.ascontiguousarray(a[:n_sample]) for a in synth.decode_step_inputs(spec, 0))
    x_p = np.ascontiguousarray(synth.warmup_last_x(spec)[:n_sample])
    st = np.ascontiguousarray(synth.filler_state(spec)[:, :n_sample], dtype=np.float64)
    sa = np.abs(st[0])
    passes, t0 = 0, time.perf_counter()
    while True:
        oracle.decode_token_shift(mu, x_t, x_p)
        oracle.decode_step(w, u, k, v, st, sa)
        passes += 1
        el = time.perf_counter() - t0
        if el >= seconds and passes >= 1:
            break
    rows = n_sample * spec.L * spec.C
    return {"value": n_sample * passes / el, "unit": "tokens/s", "cores": oracle.num_threads(), "kind": "oracle",
            "row_channels_per_s": rows * passes / el,
            "sample": f"{passes} fp64 decode steps (token shift + stabilised update) of {n_sample} of the 256 "
                      f"sessions x 32 layers x 4096 channels ({el:.1f} s)"}


def time_oracle_extras(spec, inputs, seconds=2.0):
    """The oracle's two other timings: the same recurrence on one host thread (a bounded sample
    of whole prefills of the workload), and the direct O(T^2) form on the 1x64x64 workload."""
    import oracle
    import synth
    cores = oracle.num_threads()
    oracle.set_num_threads(1)
    try:
        rate1, passes1, el1, _ = time_oracle(spec, inputs, seconds, 1)
    finally:
        oracle.set_num_threads(cores)
    small = synth.FORWARD["fwd_64x64"]
    w, u, k, v = synth.forward_inputs(small)
    passes, t0 = 0, time.perf_counter()
    while True:
        oracle.wkv_direct(w, u, k, v)
        passes += 1
        el = time.perf_counter() - t0
        if el >= seconds / 4 and passes >= 3:
            break
    n_small = small.B * small.T * small.C
    return {"single_thread": {"value": rate1, "cores": 1,
                              "sample": f"{passes1} passes of the whole prefill ({el1:.1f} s)"},
            "direct_64x64": {"value": n_small * passes / el, "unit": "elements/s", "cores": cores,
                             "sample": f"{passes} passes of eq. 1 as written, O(T^2), on 1x64x64"}}


def run_reference(args):
    """The oracle as it stands on the host cores, on the headline workload's distributions:
    each step is a bounded sample of the prefill, the first REF_CHANNELS channels over all T
    tokens (the channels are independent, so the rate does not depend on which)."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import numpy as np
    import synth
    import oracle
    spec = synth.FORWARD[WORKLOAD]
    w, u, k, v = synth.forward_inputs(spec)
    c = REF_CHANNELS
    inputs = (w[:c].copy(), u[:c].copy(), np.ascontiguousarray(k[:, :, :c]), np.ascontiguousarray(v[:, :, :c]))
    del k, v
    for _ in range(max(args.warmup, 0)):
        oracle.wkv_recurrent(*inputs)
    n = spec.B * spec.T * c
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle.wkv_recurrent(*inputs)
    el = time.perf_counter() - t0
    value = n * args.steps / el
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "elements/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": el / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": WORKLOAD, "B": spec.B, "T": spec.T, "C": spec.C, "io": "f32"},
        "cpu_baseline": {"value": value, "unit": "elements/s", "cores": oracle.num_threads(), "kind": "oracle",
                         "sample": f"each step: channels 0..{c - 1} of the {spec.B}x{spec.T}x{spec.C} prefill "
                                   f"({n} elements) through the fp64 stabilised recurrence (no decode step)"},
        "e2e": {"value": value, "unit": "elements/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------
# GPU arm
# ----------------------------------------------------------------------------

class ForwardSet:
    """One rotating input set of a forward workload plus the decode token that follows it."""

    def __init__(self, spec, seed, dev, with_decode=True, with_r=False):
        import numpy as np
        import torch
        import synth
        s = synth.ForwardSpec(spec.name, spec.B, spec.T, spec.C, spec.dtype, spec.k_std, spec.w_lo, spec.w_hi,
                              spec.spike_prob, spec.spike_value, seed)
        w, u, k, v = synth.forward_inputs(s)
        td = torch.bfloat16 if spec.dtype == "bf16" else torch.float32
        self.host = (k, v)
        self.w = torch.from_numpy(w).to(dev)
        self.u = torch.from_numpy(u).to(dev)
        self.k = torch.from_numpy(k).to(dev).to(td)
        self.v = torch.from_numpy(v).to(dev).to(td)
        self.y = torch.empty_like(self.k)
        self.state = torch.empty((3, spec.B, spec.C), dtype=torch.float32, device=dev)
        self.r = torch.from_numpy(synth.receptance(s)).to(dev).to(td) if with_r else None
        if with_decode:
            B, C = spec.B, spec.C
            r = np.random.default_rng(seed)
            self.mu = torch.from_numpy(r.uniform(0, 1, (1, C)).astype(np.float32)).to(dev)
            self.w1 = self.w.reshape(1, C)
            self.u1 = self.u.reshape(1, C)
            self.x_t = torch.from_numpy(r.normal(0, 1, (B, 1, C)).astype(np.float32)).to(dev)
            self.x_prev = torch.from_numpy(r.normal(0, 1, (B, 1, C)).astype(np.float32)).to(dev)
            self.k1 = torch.from_numpy(r.normal(0, 1, (B, 1, C)).astype(np.float32)).to(dev)
            self.v1 = torch.from_numpy(r.normal(0, 1, (B, 1, C)).astype(np.float32)).to(dev)
            self.xbar1 = torch.empty_like(self.x_t)
            self.y1 = torch.empty_like(self.x_t)
            self.state4 = self.state.view(3, B, 1, C)


def step(wkv, s, ws):
    """One pass of the hot path: prefill forward (with state_out) then the fused decode step."""
    wkv.wkv_forward(s.w, s.u, s.k, s.v, workspace=ws, y=s.y, state_out=s.state)
    wkv.wkv_decode_step_fused(s.mu, s.w1, s.u1, s.x_t, s.x_prev, s.k1, s.v1, s.state4, xbar=s.xbar1, y=s.y1)


def capture(torch, fn, n_calls):
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for i in range(n_calls):
            fn(i)
    return g


def graph_ms(torch, fn, n_calls, replays=5):
    """Per-call time of fn(i), i in range(n_calls), captured in one CUDA graph: the median over
    `replays` replays, CUDA events around each whole replay on the current stream."""
    for i in range(min(n_calls, 8)):
        fn(i)
    torch.cuda.synchronize()
    g = capture(torch, fn, n_calls)
    g.replay()
    torch.cuda.synchronize()
    out = []
    for _ in range(replays):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        g.replay()
        e1.record()
        torch.cuda.synchronize()
        out.append(e0.elapsed_time(e1) / n_calls)
    del g
    return statistics.median(out)


def event_node_ms(torch, fn, n_calls):
    """Per-call time of fn(i) from event-record nodes captured around every call inside one
    graph (each node adds a little time to the call it brackets)."""
    evs = [(torch.cuda.Event(enable_timing=True, external=True), torch.cuda.Event(enable_timing=True, external=True))
           for _ in range(n_calls)]
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for i in range(n_calls):
            evs[i][0].record()
            fn(i)
            evs[i][1].record()
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    ms = statistics.mean(a.elapsed_time(b) for a, b in evs)
    del g
    return ms


def forward_config_row(torch, wkv, dev, name, peak, cpu_seconds):
    """One forward benchmark configuration: the default path on rotating input sets (total
    over twice the L2), back-to-back launches in a graph, median of 5 replays."""
    import synth
    spec = synth.FORWARD[name]
    esz = 2 if spec.dtype == "bf16" else 4
    n = spec.B * spec.T * spec.C
    per_set = 3 * n * esz
    n_sets = sets_for(per_set) if per_set > 4096 * 16 else 1
    sets = [ForwardSet(spec, spec.seed + 17 * i, dev, with_decode=False) for i in range(n_sets)]
    td = torch.bfloat16 if spec.dtype == "bf16" else torch.float32
    ws = wkv.Workspace(dev, wkv.workspace_size(spec.B, spec.T, spec.C, td))

    def fwd(i):
        s = sets[i % n_sets]
        wkv.wkv_forward(s.w, s.u, s.k, s.v, workspace=ws, y=s.y, state_out=s.state)

    calls = GRAPH_STEPS if n < 1e6 else 4 * n_sets * max(1, 20 // (4 * n_sets))
    ms = graph_ms(torch, fwd, calls)
    wkv.forward_status(ws.buf)
    alg = ALG_BYTES_PER_ELEM[spec.dtype] * n
    row = {"workload": name, "B": spec.B, "T": spec.T, "C": spec.C, "io": spec.dtype,
           "path": wkv.auto_path(spec.B, spec.T, spec.C, td), "launch_ms": ms, "elements_per_s": n / (ms * 1e-3),
           "alg_bytes_per_launch": alg, "achieved_gbs": alg / (ms * 1e-3) / 1e9,
           "frac": alg / (ms * 1e-3) / 1e9 / peak,
           "l2": f"{n_sets} rotating input set(s) of {per_set / 1e6:.1f} MB",
           "timing": f"graph of {calls} back-to-back forwards (with state_out), median of 5 replays"}
    if name == "fwd_64x64":
        # latency of one launch: events around a single eager call, median of 50
        lat = []
        for _ in range(50):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            fwd(0)
            e1.record()
            torch.cuda.synchronize()
            lat.append(e0.elapsed_time(e1))
        row["latency_ms"] = statistics.median(lat)
        row["latency_timing"] = "events around one eager call, median of 50"
        row["frac_note"] = "a 50 KB problem is latency-bound: the fraction is reported, not a target"
    if cpu_seconds:
        row["cpu_baseline"] = oracle_row(spec, cpu_seconds)
    del sets, ws
    torch.cuda.empty_cache()
    return row


def decode_bench(torch, wkv, dev, steps, peak):
    """256 sessions x 32 layers x 4096 channels, fused decode, 4 input sets in rotation
    (each 403 MB of x, k, v)."""
    N, L, C = 256, 32, 4096
    g = torch.Generator(device=dev)
    g.manual_seed(1005)
    mu = torch.rand((L, C), generator=g, device=dev)
    w = torch.exp(torch.rand((L, C), generator=g, device=dev) * 6 - 5)
    u = torch.randn((L, C), generator=g, device=dev) * 0.5
    st = torch.empty((3, N, L, C), device=dev)
    st[2].normal_(1.0, 1.0, generator=g)
    st[1].normal_(0.0, 1.0, generator=g).abs_().add_(1.0)
    st[0].normal_(0.0, 1.0, generator=g).mul_(st[1])
    sets = [tuple(torch.randn((N, L, C), generator=g, device=dev) for _ in range(3)) for _ in range(4)]
    xbar = torch.empty((N, L, C), device=dev)
    y = torch.empty((N, L, C), device=dev)

    def one(i):
        x_t, k, v = sets[i % 4]
        x_prev = sets[(i - 1) % 4][0]
        wkv.wkv_decode_step_fused(mu, w, u, x_t, x_prev, k, v, st, xbar=xbar, y=y)

    ms = graph_ms(torch, one, 8, replays=max(3, steps // 8))
    alg = DECODE_ALG_BYTES_PER_ELEM * N * L * C
    del sets, st
    torch.cuda.empty_cache()
    return {"workload": f"decode_{N}x{L}x{C}", "metric": "decode tokens/s (session steps through all 32 layers)",
            "value": N / (ms * 1e-3), "unit": "tokens/s", "ms_per_step": ms, "alg_bytes_per_step": alg,
            "achieved_gbs": alg / (ms * 1e-3) / 1e9, "frac": alg / (ms * 1e-3) / 1e9 / peak,
            "l2": "4 rotating sets of x, k, v (403 MB each); state 403 MB updated in place",
            "timing": "graph of 8 fused decode steps, median over replays"}


def next_rows_bench(torch, wkv, dev, peak):
    """The fused receptance-gated forward (y = sigma(r) * wkv: k, v, r read and y written once,
    16 B/element fp32), the three-mu token shift (x read, three blends written, 16 B/element)
    and the backward (k, v, gy read, gk, gv written: 20 B/element) on the 8 x 1024 x 768
    workload, rotating input sets, next to the plain forward timed the same way."""
    import synth
    spec = synth.FORWARD["fwd_8x1024x768"]
    n = spec.B * spec.T * spec.C
    sets = [ForwardSet(spec, rank_set_seed(spec.seed, 0, i), dev, with_decode=False, with_r=True) for i in range(4)]
    ws = wkv.Workspace(dev, wkv.workspace_size(spec.B, spec.T, spec.C))

    def plain(i):
        s = sets[i % len(sets)]
        wkv.wkv_forward(s.w, s.u, s.k, s.v, workspace=ws, y=s.y, state_out=s.state)

    def gated(i):
        s = sets[i % len(sets)]
        wkv.wkv_forward(s.w, s.u, s.k, s.v, workspace=ws, y=s.y, state_out=s.state, r=s.r)

    mu = [torch.rand(spec.C, device=dev) for _ in range(3)]

    def shift3(i):
        s = sets[i % len(sets)]
        wkv.token_shift_mix3(mu[0], mu[1], mu[2], s.k)

    gy = torch.randn_like(sets[0].k)
    bws = torch.zeros(int(wkv.lib().wkv_backward_workspace_size(spec.B, spec.T, spec.C)), dtype=torch.uint8,
                      device=dev)

    def backward(i):
        s = sets[i % len(sets)]
        wkv.wkv_backward(s.w, s.u, s.k, s.v, gy, workspace=bws)

    plain_ms = graph_ms(torch, plain, GRAPH_STEPS)
    gated_ms = graph_ms(torch, gated, GRAPH_STEPS)
    shift_ms = graph_ms(torch, shift3, GRAPH_STEPS)
    bwd_ms = graph_ms(torch, backward, 8)
    b_gbs = 20 * n / (bwd_ms * 1e-3) / 1e9
    g_gbs = 16 * n / (gated_ms * 1e-3) / 1e9
    t_gbs = 16 * n / (shift_ms * 1e-3) / 1e9
    del sets, ws, bws
    torch.cuda.empty_cache()
    return {
        "gated_forward": {"workload": spec.name, "launch_ms": gated_ms, "alg_bytes_per_launch": 16 * n,
                          "achieved_gbs": g_gbs, "frac": g_gbs / peak, "plain_forward_launch_ms": plain_ms,
                          "timing": f"graph of {GRAPH_STEPS} back-to-back launches, median of 5 replays"},
        "token_shift3": {"workload": spec.name, "launch_ms": shift_ms, "alg_bytes_per_launch": 16 * n,
                         "achieved_gbs": t_gbs, "frac": t_gbs / peak},
        "backward": {"workload": spec.name, "launch_ms": bwd_ms, "alg_bytes_per_launch": 20 * n,
                     "achieved_gbs": b_gbs, "frac": b_gbs / peak,
                     "note": "k, v, gy read and gk, gv written once (20 B/element)"},
    }


def eagle_bench(torch, wkv, dev, peak, decode=True):
    """Eagle (RWKV-5) matrix-state WKV: the prefill on eagle_8x1024x768 (three rotating input
    sets, > 2x L2) and eagle_4x4096x2048 (two sets of 1.6 GB), r, k, v read and y written once:
    16 B/element, plus the final state, 16 KiB per sequence-head; and the decode step for 256
    sessions x 32 layers x 4096 channels (each 64 x 64 state read and written once, r, k, v read
    and y written)."""
    import synth
    out = {}
    g = torch.Generator(device=dev)
    for key, name, n_sets in (("eagle_forward", "eagle_8x1024x768", 3), ("eagle_forward_long", "eagle_4x4096x2048", 2)):
        spec = synth.EAGLE[name]
        B, T, C = spec.B, spec.T, spec.C
        H = C // 64
        g.manual_seed(spec.seed)
        w = torch.exp(torch.rand(C, generator=g, device=dev) * (spec.w_hi - spec.w_lo) + spec.w_lo)
        sets = [[torch.randn((B, T, C), generator=g, device=dev) for _ in range(3)] for _ in range(n_sets)]
        y = torch.empty((B, T, C), device=dev)
        st = torch.empty((B, H, 64, 64), device=dev)
        ws = torch.empty(int(wkv.lib().eagle_forward_workspace_size(B, T, C)), dtype=torch.uint8, device=dev)

        def fwd(i, sets=sets, w=w, y=y, st=st, ws=ws):
            r, k, v = sets[i % len(sets)]
            wkv.eagle_forward(w, r, k, v, y=y, state_out=st, workspace=ws)

        n = B * T * C
        alg = 16 * n + B * H * 64 * 64 * 4
        f_ms = graph_ms(torch, fwd, 12)
        out[key] = {"workload": spec.name, "launch_ms": f_ms, "alg_bytes_per_launch": alg,
                    "achieved_gbs": alg / (f_ms * 1e-3) / 1e9, "frac": alg / (f_ms * 1e-3) / 1e9 / peak,
                    "elements_per_s": n / (f_ms * 1e-3), "launches": int(wkv.lib().eagle_forward_launches(B, T, C)),
                    "l2": f"{n_sets} rotating input sets of {3 * n * 4 / 1e6:.0f} MB"}
        del sets, ws, y, st, w
        torch.cuda.empty_cache()
    if decode:
        N, L, Cd = 256, 32, 4096
        Hd = Cd // 64
        wd = torch.exp(torch.rand((L, Cd), generator=g, device=dev) * 6 - 5)
        S = torch.randn((N, L, Hd, 64, 64), generator=g, device=dev)
        dsets = [[torch.randn((N, L, Cd), generator=g, device=dev) for _ in range(3)] for _ in range(2)]
        yd = torch.empty((N, L, Cd), device=dev)

        def dec(i):
            r, k, v = dsets[i % 2]
            wkv.eagle_decode_step(wd, r, k, v, S, y=yd)

        d_ms = graph_ms(torch, dec, 4)
        d_alg = 2 * S.numel() * 4 + 4 * N * L * Cd * 4
        out["eagle_decode"] = {"workload": "eagle_decode_256x32x4096", "ms_per_step": d_ms,
                               "tokens_per_s": N / (d_ms * 1e-3), "alg_bytes_per_step": d_alg,
                               "achieved_gbs": d_alg / (d_ms * 1e-3) / 1e9,
                               "frac": d_alg / (d_ms * 1e-3) / 1e9 / peak}
        del S, dsets
    torch.cuda.empty_cache()
    return out


def e2e_bench(torch, wkv, sets, ws, steps):
    """Through the public API with host buffers: per step, copy k and v from pinned host
    memory, run the step, read y back to pinned host memory.  Uploads and downloads ride
    streams of their own (each direction has its own copy engine), so with two input sets a
    step's upload overlaps the previous step's kernels and download; every step's copies lie
    inside the timed region, which starts before the first upload and ends after the last
    download."""
    pinned_in = [(torch.from_numpy(s.host[0]).pin_memory(), torch.from_numpy(s.host[1]).pin_memory()) for s in sets]
    pinned_out = [torch.empty(s.y.shape, dtype=s.y.dtype).pin_memory() for s in sets]
    h2d = sum(a.numel() * a.element_size() for a in pinned_in[0])
    d2h = pinned_out[0].numel() * pinned_out[0].element_size()
    comp = torch.cuda.current_stream()
    up, down = torch.cuda.Stream(), torch.cuda.Stream()
    n = len(sets)
    uploaded = [torch.cuda.Event() for _ in sets]
    computed = [torch.cuda.Event() for _ in sets]   # the step has read k, v and written y
    read_back = [torch.cuda.Event() for _ in sets]  # y is in host memory
    for j in range(n):
        computed[j].record(comp)
        read_back[j].record(down)

    def run(k):
        for i in range(k):
            j = i % n
            s = sets[j]
            with torch.cuda.stream(up):
                up.wait_event(computed[j])
                s.k.copy_(pinned_in[j][0], non_blocking=True)
                s.v.copy_(pinned_in[j][1], non_blocking=True)
                uploaded[j].record(up)
            comp.wait_event(uploaded[j])
            comp.wait_event(read_back[j])
            step(wkv, s, ws)
            computed[j].record(comp)
            with torch.cuda.stream(down):
                down.wait_event(computed[j])
                pinned_out[j].copy_(s.y, non_blocking=True)
                read_back[j].record(down)

    run(n)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(comp)
    up.wait_event(e0)
    run(steps)
    comp.wait_stream(down)
    e1.record(comp)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / steps
    return ms, h2d, d2h


def run_ours(args):
    import torch
    rank, world, local = dist_setup(args.gpus)
    dev = torch.device("cuda", torch.cuda.current_device())
    import linear_attention_rnn_wkv_b200 as wkv
    import synth

    spec = synth.FORWARD[WORKLOAD]
    n_elem = spec.B * spec.T * spec.C
    n_sets = 2  # each set's k, v, y (805 MB) is over six times the L2 by itself
    sets = [ForwardSet(spec, rank_set_seed(spec.seed, rank, i), dev) for i in range(n_sets)]
    ws = wkv.Workspace(dev, wkv.workspace_size(spec.B, spec.T, spec.C))
    path = wkv.auto_path(spec.B, spec.T, spec.C)

    def one(i):
        step(wkv, sets[i % n_sets], ws)

    # eager warm-up (sets kernel attributes, first-touch), then W untimed graph steps
    for i in range(n_sets):
        one(i)
    torch.cuda.synchronize()
    wkv.forward_status(ws.buf)

    K = args.steps
    main_g = capture(torch, one, K)
    warm_g = capture(torch, one, max(args.warmup, 3))
    warm_g.replay()
    torch.cuda.synchronize()
    del warm_g

    clocks = ClockSampler(local)
    if rank == 0:
        clocks.start()
    # pre-roll the same graph for ~1 s so the clock record covers sustained load
    t_pre = time.time()
    while time.time() - t_pre < 1.0:
        main_g.replay()
        torch.cuda.synchronize()

    replay_ms = []
    t_wall0 = time.time()
    for _ in range(REPLAYS):
        barrier(world)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        main_g.replay()
        e1.record()
        torch.cuda.synchronize()
        barrier(world)
        replay_ms.append(max_over_ranks(e0.elapsed_time(e1), world))
    t_wall1 = time.time()
    clocks.stop()
    wkv.forward_status(ws.buf)
    del main_g

    ms_per_step = statistics.median(replay_ms) / K
    value = weak_scaling_value(world, n_elem, ms_per_step)

    def fwd(i):
        s = sets[i % n_sets]
        wkv.wkv_forward(s.w, s.u, s.k, s.v, workspace=ws, y=s.y, state_out=s.state)

    # The forward's own launch duration, right after the timed region: back-to-back forwards
    # in a graph, events around whole replays (median of 5).  Event nodes inside a graph add a
    # little to the launch they bracket; that figure is reported beside it.
    fwd_ms = max_over_ranks(graph_ms(torch, fwd, 20), world)
    try:
        nodes_ms = event_node_ms(torch, fwd, 10)
    except Exception:
        nodes_ms = float("nan")
    nodes_ms = max_over_ranks(nodes_ms, world)  # every rank takes part, failed or not
    nodes_ms = None if nodes_ms != nodes_ms else nodes_ms

    peaks, peak_kind = measured_peaks()
    peak = peaks["hbm_gbs"]
    alg = ALG_BYTES_PER_ELEM[spec.dtype] * n_elem
    achieved = alg / (fwd_ms * 1e-3) / 1e9
    traffic, traffic_src = profiled_traffic(WORKLOAD)

    e2e = None
    if not args.no_e2e:
        ms_e2e, h2d, d2h = e2e_bench(torch, wkv, sets[:2], ws, max(3, min(K, 20)))
        ms_e2e = max_over_ranks(ms_e2e, world)
        e2e = {"value": weak_scaling_value(world, n_elem, ms_e2e), "unit": "elements/s", "ms_per_step": ms_e2e,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h}
    del sets
    torch.cuda.empty_cache()

    cpu_s = 0.0 if (args.no_cpu or rank != 0 or world != 1) else 2.0
    configs = None
    if not args.no_configs:
        configs = {}
        for name in FORWARD_CONFIGS:
            configs[name] = forward_config_row(torch, wkv, dev, name, peak, cpu_s)
        if not args.no_decode:
            d = decode_bench(torch, wkv, dev, 200, peak)
            if cpu_s:
                d["cpu_baseline"] = oracle_decode_row(cpu_s)
            configs[d["workload"]] = d
    nxt = None
    if not args.no_next:
        nxt = next_rows_bench(torch, wkv, dev, peak)
        nxt.update(eagle_bench(torch, wkv, dev, peak, decode=not args.no_decode))

    cpu = None
    if cpu_s:
        rate, passes, el, cores = time_oracle(spec, synth.forward_inputs(spec), 5.0, 3)
        cpu = {"value": rate, "unit": "elements/s", "cores": cores, "kind": "oracle",
               "sample": f"{passes} passes of the whole {spec.B}x{spec.T}x{spec.C} prefill through the fp64 "
                         f"stabilised recurrence ({el:.1f} s)"}
        cpu.update(time_oracle_extras(spec, synth.forward_inputs(spec)))

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "elements/s", "n_gpus": world, "steps": K,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": {"workload": WORKLOAD, "B": spec.B, "T": spec.T, "C": spec.C, "io": spec.dtype,
                       "state_out": True,
                       "step": "prefill forward (with final state) + one fused decode step of the same batch",
                       "forward_path": path,
                       "l2": f"inputs larger than L2: each step reads {2 * n_elem * 4 / 1e6:.0f} MB and writes "
                             f"{n_elem * 4 / 1e6:.0f} MB; {n_sets} sets rotate",
                       "graph": f"one CUDA graph of {K} steps, replayed {REPLAYS} times; median replay",
                       "replay_ms": replay_ms},
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                         "frac": achieved / peak, "traffic": traffic,
                         "traffic_source": (f"{traffic_src} (ncu dram__bytes of the same kernel source; not "
                                            "measured in this run)") if traffic_src else None,
                         "kernel": f"wkv_forward ({path})", "launch_ms": fwd_ms,
                         "launch_timing": "graph of 20 back-to-back forwards on the rotating input sets, CUDA "
                                          "events around each replay, median of 5, right after the timed region",
                         "launch_ms_event_nodes": nodes_ms,
                         "alg_bytes_per_launch": alg, "peak_kind": f"{peak_kind} hbm_gbs"},
            "cpu_baseline": cpu,
            "e2e": e2e,
            "gpu_launches": 2 * K,
            "configs": configs,
            "next_rows": nxt,
            "clocks": clocks.summary(t_wall0, t_wall1) if rank == 0 else None,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def profile_forward(name):
    """Two warm-up and three profiled eager forward launches (with the final state) of one
    forward workload on one input set; checks the workspace status afterwards."""
    import torch
    import linear_attention_rnn_wkv_b200 as wkv
    import synth
    spec = synth.FORWARD[name]
    dev = torch.device("cuda", 0)
    w, u, k, v = synth.forward_inputs(spec)
    td = torch.bfloat16 if spec.dtype == "bf16" else torch.float32
    w, u = torch.from_numpy(w).to(dev), torch.from_numpy(u).to(dev)
    k, v = torch.from_numpy(k).to(dev).to(td), torch.from_numpy(v).to(dev).to(td)
    y = torch.empty_like(k)
    st = torch.empty((3, spec.B, spec.C), dtype=torch.float32, device=dev)
    ws = wkv.Workspace(dev, wkv.workspace_size(spec.B, spec.T, spec.C, td))
    for _ in range(5):
        wkv.wkv_forward(w, u, k, v, want_state=True, workspace=ws, y=y, state_out=st)
    torch.cuda.synchronize()
    wkv.forward_status(ws.buf)
    print(json.dumps({"profile_forward": name, "launches": 5, "B": spec.B, "T": spec.T, "C": spec.C,
                      "io": spec.dtype}))


def profile_step():
    """Three warm-up and two profiled eager headline steps (forward with state + fused decode)
    on one input set."""
    import torch
    import linear_attention_rnn_wkv_b200 as wkv
    import synth
    spec = synth.FORWARD[WORKLOAD]
    dev = torch.device("cuda", 0)
    s = ForwardSet(spec, spec.seed, dev)
    ws = wkv.Workspace(dev, wkv.workspace_size(spec.B, spec.T, spec.C))
    for _ in range(5):
        step(wkv, s, ws)
    torch.cuda.synchronize()
    wkv.forward_status(ws.buf)
    print(json.dumps({"profile_step": WORKLOAD, "steps": 5}))


def profile_backward(name):
    """Two warm-up and three profiled eager backward calls on one forward workload's shape, in
    fp32 (the backward's only I/O type)."""
    import torch
    import linear_attention_rnn_wkv_b200 as wkv
    import synth
    spec = synth.FORWARD[name]
    dev = torch.device("cuda", 0)
    w, u, k, v = synth.forward_inputs(spec)
    gy = synth.grad_output(spec)
    t = [torch.from_numpy(a.astype("float32")).to(dev) for a in (w, u, k, v, gy)]
    ws = torch.zeros(int(wkv.lib().wkv_backward_workspace_size(spec.B, spec.T, spec.C)), dtype=torch.uint8,
                     device=dev)
    for _ in range(5):
        wkv.wkv_backward(*t, workspace=ws)
    torch.cuda.synchronize()
    print(json.dumps({"profile_backward": name, "calls": 5, "B": spec.B, "T": spec.T, "C": spec.C}))


def profile_eagle():
    """Two warm-up and three profiled eager Eagle prefills (with the final state) on
    eagle_8x1024x768."""
    import torch
    import linear_attention_rnn_wkv_b200 as wkv
    import synth
    spec = synth.EAGLE["eagle_8x1024x768"]
    dev = torch.device("cuda", 0)
    w, r, k, v = (torch.from_numpy(a).to(dev) for a in synth.eagle_inputs(spec))
    for _ in range(5):
        wkv.eagle_forward(w, r, k, v)
    torch.cuda.synchronize()
    wkv.get_device_status()
    print(json.dumps({"profile_eagle": spec.name, "calls": 5}))


def main():
    args = parse()
    if args.profile_forward:
        profile_forward(args.profile_forward)
        return
    if args.profile_step:
        profile_step()
        return
    if args.profile_backward:
        profile_backward(args.profile_backward)
        return
    if args.profile_eagle:
        profile_eagle()
        return
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
