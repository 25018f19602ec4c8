"""Seeded synthetic inputs for the WKV workloads (shared by tests, bench and smoke).

This module only draws numbers; it holds none of the WKV arithmetic.  The
generator is counter-based (SplitMix64 hashing of (seed, stream, index), with
Box-Muller normals; see ``synth.c``), so element ``i`` of any array is a pure
function of ``(seed, stream, i)``: a sampled channel can be regenerated alone,
and results do not depend on the thread count.

Workload recipes follow the five configurations of the WKV benchmark table:
shapes, dtypes and distributions (``N(m, s)`` takes ``s`` as the standard
deviation).  Decode-workload distributions that the table leaves open use the
forward workloads' choices: ``w = exp(U(-5, 1))``, ``u ~ N(0, 0.5)``, and
``x, k, v ~ N(0, 1)``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "synth.c")
_LIB_PATH = os.path.join(_HERE, "libsynth.so")

# Stream identifiers: one independent stream per named array.
S_W, S_U, S_K, S_KSPIKE, S_V, S_MU, S_X = 1, 2, 3, 4, 5, 6, 7
S_WARM_K, S_WARM_V, S_WARM_X = 8, 9, 10
S_DEC_K, S_DEC_V, S_DEC_X = 11, 12, 13
S_STATE_P, S_STATE_B, S_STATE_A = 14, 15, 16
S_R, S_RSPIKE = 17, 18
S_GY = 19
S_EAGLE_W, S_EAGLE_R, S_EAGLE_K, S_EAGLE_V, S_EAGLE_STATE = 20, 21, 22, 23, 24


def build(force: bool = False) -> str:
    """Compile ``libsynth.so`` with gcc (OpenMP over elements)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off",
                               "-fno-fast-math", _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


_lib = None


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB_PATH)
        u64, i64, dbl, vp = ctypes.c_uint64, ctypes.c_int64, ctypes.c_double, ctypes.c_void_p
        for name in ("synth_normal_f32", "synth_uniform_f32", "synth_exp_uniform_f32"):
            getattr(L, name).argtypes = [u64, u64, u64, i64, dbl, dbl, vp]
            getattr(L, name).restype = None
        L.synth_spike_f32.argtypes = [u64, u64, u64, i64, dbl, dbl, vp]
        L.synth_normal_f32_at.argtypes = [u64, u64, vp, i64, dbl, dbl, vp]
        L.synth_spike_f32_at.argtypes = [u64, u64, vp, i64, dbl, dbl, vp]
        L.synth_words.argtypes = [u64, u64, u64, i64, vp]
        for f in (L.synth_spike_f32, L.synth_normal_f32_at, L.synth_spike_f32_at, L.synth_words):
            f.restype = None
        _lib = L
    return _lib


def _ptr(a: np.ndarray) -> int:
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data


def normal(seed, stream, shape, mean=0.0, std=1.0, offset=0, out=None) -> np.ndarray:
    out = np.empty(shape, np.float32) if out is None else out
    lib().synth_normal_f32(seed, stream, offset, out.size, mean, std, _ptr(out))
    return out


def uniform(seed, stream, shape, lo, hi, offset=0) -> np.ndarray:
    out = np.empty(shape, np.float32)
    lib().synth_uniform_f32(seed, stream, offset, out.size, lo, hi, _ptr(out))
    return out


def exp_uniform(seed, stream, shape, lo, hi, offset=0) -> np.ndarray:
    out = np.empty(shape, np.float32)
    lib().synth_exp_uniform_f32(seed, stream, offset, out.size, lo, hi, _ptr(out))
    return out


def spike(seed, stream, arr: np.ndarray, prob, value, offset=0) -> np.ndarray:
    lib().synth_spike_f32(seed, stream, offset, arr.size, prob, value, _ptr(arr))
    return arr


def normal_at(seed, stream, idx: np.ndarray, mean=0.0, std=1.0) -> np.ndarray:
    idx = np.ascontiguousarray(idx, dtype=np.int64)
    out = np.empty(idx.shape, np.float32)
    lib().synth_normal_f32_at(seed, stream, _ptr(idx), idx.size, mean, std, _ptr(out))
    return out


def spike_at(seed, stream, idx: np.ndarray, arr: np.ndarray, prob, value) -> np.ndarray:
    idx = np.ascontiguousarray(idx, dtype=np.int64)
    lib().synth_spike_f32_at(seed, stream, _ptr(idx), idx.size, prob, value, _ptr(arr))
    return arr


def words(seed, stream, n, offset=0) -> np.ndarray:
    out = np.empty(n, np.uint64)
    lib().synth_words(seed, stream, offset, n, _ptr(out))
    return out


def to_bf16_exact(a: np.ndarray) -> np.ndarray:
    """Round fp32 values to the nearest bf16 (ties to even); return them as fp32.

    The CUDA path receives the bf16 values; the oracle receives the same values
    widened to fp64, so both see identical inputs.
    """
    b = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    lsb = (b >> np.uint64(16)) & np.uint64(1)
    r = ((b + np.uint64(0x7FFF) + lsb) >> np.uint64(16)) << np.uint64(16)
    return r.astype(np.uint32).view(np.float32).reshape(a.shape)


# --------------------------------------------------------------------------
# Workload recipes
# --------------------------------------------------------------------------

@dataclass(frozen=True)
class ForwardSpec:
    name: str
    B: int
    T: int
    C: int
    dtype: str            # "f32" or "bf16" (I/O type; state is always fp32)
    k_std: float
    w_lo: float
    w_hi: float
    spike_prob: float     # fraction of k entries overwritten with spike_value
    spike_value: float
    seed: int
    u_std: float = 0.5
    v_std: float = 1.0


FORWARD = {
    # B=1 T=64 C=64 fp32, k,v ~ N(0,1), w = exp(U(-3,1)), u ~ N(0,0.5)
    "fwd_64x64": ForwardSpec("fwd_64x64", 1, 64, 64, "f32", 1.0, -3.0, 1.0, 0.0, 0.0, 1001),
    # B=8 T=1024 C=768 fp32, k ~ N(0,3) with 1% set to +40, w = exp(U(-5,1))
    "fwd_8x1024x768": ForwardSpec("fwd_8x1024x768", 8, 1024, 768, "f32", 3.0, -5.0, 1.0, 0.01, 40.0, 1002),
    # B=4 T=4096 C=2048 bf16 I/O, k ~ N(0,2), w = exp(U(-6,1))
    "fwd_4x4096x2048_bf16": ForwardSpec("fwd_4x4096x2048_bf16", 4, 4096, 2048, "bf16", 2.0, -6.0, 1.0,
                                        0.0, 0.0, 1003),
    # B=1 T=16384 C=4096 fp32, distributions as the 8x1024x768 workload
    "fwd_1x16384x4096": ForwardSpec("fwd_1x16384x4096", 1, 16384, 4096, "f32", 3.0, -5.0, 1.0, 0.01, 40.0,
                                    1004),
}


def forward_spec_like(base: str, B: int, T: int, C: int, seed: int | None = None) -> ForwardSpec:
    """Same distributions as workload ``base`` at another shape (parity cases)."""
    s = FORWARD[base]
    return ForwardSpec(f"{base}@{B}x{T}x{C}", B, T, C, s.dtype, s.k_std, s.w_lo, s.w_hi, s.spike_prob,
                       s.spike_value, s.seed if seed is None else seed, s.u_std, s.v_std)


def forward_params(spec: ForwardSpec):
    """Per-channel w (> 0) and u, fp32 [C]."""
    w = exp_uniform(spec.seed, S_W, (spec.C,), spec.w_lo, spec.w_hi)
    u = normal(spec.seed, S_U, (spec.C,), 0.0, spec.u_std)
    return w, u


def forward_inputs(spec: ForwardSpec):
    """(w, u, k, v): w,u fp32 [C]; k,v fp32 [B,T,C] holding exactly representable values
    of the I/O dtype (bf16 workloads are rounded to bf16 here)."""
    w, u = forward_params(spec)
    shape = (spec.B, spec.T, spec.C)
    k = normal(spec.seed, S_K, shape, 0.0, spec.k_std)
    if spec.spike_prob > 0:
        spike(spec.seed, S_KSPIKE, k, spec.spike_prob, spec.spike_value)
    v = normal(spec.seed, S_V, shape, 0.0, spec.v_std)
    if spec.dtype == "bf16":
        k, v = to_bf16_exact(k), to_bf16_exact(v)
    return w, u, k, v


def receptance(spec: ForwardSpec, r_std: float = 2.0, spike_prob: float = 0.01, spike_value: float = -40.0):
    """Receptance r [B,T,C] for the output gate sigma(r) * wkv: N(0, r_std) with a fraction
    of entries set to spike_value (a gate pushed shut, sigma ~ 4e-18); exact in the I/O dtype."""
    r = normal(spec.seed, S_R, (spec.B, spec.T, spec.C), 0.0, r_std)
    if spike_prob > 0:
        spike(spec.seed, S_RSPIKE, r, spike_prob, spike_value)
    if spec.dtype == "bf16":
        r = to_bf16_exact(r)
    return r


def grad_output(spec: ForwardSpec, std: float = 1.0):
    """Upstream gradient gy [B,T,C] for the backward: N(0, std), fp32."""
    return normal(spec.seed, S_GY, (spec.B, spec.T, spec.C), 0.0, std)


def forward_inputs_at(spec: ForwardSpec, b: np.ndarray, c: np.ndarray):
    """k, v of the sampled channels (b[j], c[j]) over all T: arrays [n, T] (fp32)."""
    b = np.asarray(b, np.int64)
    c = np.asarray(c, np.int64)
    t = np.arange(spec.T, dtype=np.int64)
    idx = (b[:, None] * spec.T + t[None, :]) * spec.C + c[:, None]
    k = normal_at(spec.seed, S_K, idx, 0.0, spec.k_std)
    if spec.spike_prob > 0:
        spike_at(spec.seed, S_KSPIKE, idx, k, spec.spike_prob, spec.spike_value)
    v = normal_at(spec.seed, S_V, idx, 0.0, spec.v_std)
    if spec.dtype == "bf16":
        k, v = to_bf16_exact(k), to_bf16_exact(v)
    return k, v


@dataclass(frozen=True)
class DecodeSpec:
    name: str
    N: int          # sessions
    L: int          # layers
    C: int          # channels
    warmup: int     # tokens of oracle warm-up that produce the start state
    steps: int      # decode steps compared / timed
    seed: int
    w_lo: float = -5.0
    w_hi: float = 1.0
    u_std: float = 0.5
    n_sets: int = 4  # full-size runs cycle through this many pre-drawn input sets


DECODE = {
    "decode_256x32x4096": DecodeSpec("decode_256x32x4096", 256, 32, 4096, 512, 128, 1005),
}


def decode_params(spec: DecodeSpec):
    """mu ~ U(0,1), w = exp(U(-5,1)), u ~ N(0,0.5): fp32 [L, C]."""
    shape = (spec.L, spec.C)
    mu = uniform(spec.seed, S_MU, shape, 0.0, 1.0)
    w = exp_uniform(spec.seed, S_W, shape, spec.w_lo, spec.w_hi)
    u = normal(spec.seed, S_U, shape, 0.0, spec.u_std)
    return mu, w, u


def decode_step_inputs(spec: DecodeSpec, step: int):
    """x_t, k, v for decode step ``step``: fp32 [N, L, C] each, N(0,1)."""
    n = spec.N * spec.L * spec.C
    shape = (spec.N, spec.L, spec.C)
    off = step * n
    return (normal(spec.seed, S_DEC_X, shape, offset=off), normal(spec.seed, S_DEC_K, shape, offset=off),
            normal(spec.seed, S_DEC_V, shape, offset=off))


def decode_step_inputs_at(spec: DecodeSpec, step: int, flat: np.ndarray):
    """x_t, k, v of decode step ``step`` at flat row-channel indices ``flat``."""
    n = spec.N * spec.L * spec.C
    idx = step * n + np.asarray(flat, np.int64)
    return (normal_at(spec.seed, S_DEC_X, idx), normal_at(spec.seed, S_DEC_K, idx),
            normal_at(spec.seed, S_DEC_V, idx))


def warmup_inputs_at(spec: DecodeSpec, t: int, flat: np.ndarray):
    """k, v of warm-up token ``t`` at flat row-channel indices ``flat``."""
    n = spec.N * spec.L * spec.C
    idx = t * n + np.asarray(flat, np.int64)
    return normal_at(spec.seed, S_WARM_K, idx), normal_at(spec.seed, S_WARM_V, idx)


def warmup_inputs(spec: DecodeSpec, t: int):
    shape = (spec.N, spec.L, spec.C)
    n = spec.N * spec.L * spec.C
    return (normal(spec.seed, S_WARM_K, shape, offset=t * n), normal(spec.seed, S_WARM_V, shape, offset=t * n))


def warmup_last_x(spec: DecodeSpec, flat: np.ndarray | None = None):
    """The last warm-up token's x (the decode's first x_prev)."""
    n = spec.N * spec.L * spec.C
    t = spec.warmup - 1
    if flat is None:
        return normal(spec.seed, S_WARM_X, (spec.N, spec.L, spec.C), offset=t * n)
    return normal_at(spec.seed, S_WARM_X, t * n + np.asarray(flat, np.int64))


def filler_state(spec: DecodeSpec):
    """A valid but arbitrary fp32 (a, b, p) start state [3, N, L, C] for channels that no
    check reads (full-size runs overwrite the sampled channels with the oracle's warm-up
    state): p ~ N(1, 1), b = 1 + |N(0,1)|, a = b * N(0,1)."""
    shape = (spec.N, spec.L, spec.C)
    st = np.empty((3,) + shape, np.float32)
    normal(spec.seed, S_STATE_P, shape, 1.0, 1.0, out=st[2])
    bn = normal(spec.seed, S_STATE_B, shape)
    np.abs(bn, out=bn)
    bn += 1.0
    st[1] = bn
    an = normal(spec.seed, S_STATE_A, shape)
    np.multiply(an, bn, out=st[0])
    return st


# --------------------------------------------------------------------------
# Eagle (RWKV-5) matrix-state workloads: heads of 64 channels.  The pages give no
# distributions for it; these take the RWKV-4 forward workloads' decay range
# (w = exp(U(-5, 1))) and r, k, v ~ N(0, 1).
# --------------------------------------------------------------------------

@dataclass(frozen=True)
class EagleSpec:
    name: str
    B: int
    T: int
    C: int                # a multiple of 64: C / 64 heads
    seed: int
    w_lo: float = -5.0
    w_hi: float = 1.0


EAGLE = {
    # the headline forward shape read as 12 heads of 64 channels
    "eagle_8x1024x768": EagleSpec("eagle_8x1024x768", 8, 1024, 768, 2001),
    # the long bf16 forward shape's size, fp32, 32 heads
    "eagle_4x4096x2048": EagleSpec("eagle_4x4096x2048", 4, 4096, 2048, 2002),
}


def eagle_spec_like(base: str, B: int, T: int, C: int, seed: int | None = None) -> EagleSpec:
    s = EAGLE[base]
    return EagleSpec(f"{base}@{B}x{T}x{C}", B, T, C, s.seed if seed is None else seed, s.w_lo, s.w_hi)


def eagle_inputs(spec: EagleSpec):
    """(w, r, k, v): w fp32 [C] (> 0), r, k, v fp32 [B, T, C]."""
    w = exp_uniform(spec.seed, S_EAGLE_W, (spec.C,), spec.w_lo, spec.w_hi)
    shape = (spec.B, spec.T, spec.C)
    r = normal(spec.seed, S_EAGLE_R, shape)
    k = normal(spec.seed, S_EAGLE_K, shape)
    v = normal(spec.seed, S_EAGLE_V, shape)
    return w, r, k, v


def eagle_state(spec: EagleSpec, std: float = 1.0):
    """A given starting state [B, C / 64, 64, 64], N(0, std)."""
    return normal(spec.seed, S_EAGLE_STATE, (spec.B, spec.C // 64, 64, 64), 0.0, std)
