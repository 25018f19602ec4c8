// WKV backward: gradients of L = sum(gy * y) with respect to k, v (per element) and w, u
// (per channel, summed over batch and time), for the forward from the empty state.
//
// The pages give no gradient; this is the wkv_t equation ("RWKV" transformer-math page,
// aicassindra.com, section "The WKV operator: attention with a fixed decay"; aiwiki "RWKV",
// eq. 1) differentiated as written.  With D_t the denominator of position t, alpha_t = e^{u+k_t}
// and beta_{t,i} = e^{-(t-1-i) w + k_i}:
//   gv_i = gy_i alpha_i / D_i + e^{k_i} X_i
//   gk_i = gy_i alpha_i (v_i - y_i) / D_i + e^{k_i} (v_i X_i - Y_i)
//   gu   = sum_t gy_t alpha_t (v_t - y_t) / D_t
//   gw   = -sum_i e^{k_i} (v_i X'_i - Y'_i)
// where X_i = sum_{t>i} e^{-(t-1-i) w} gy_t / D_t, Y_i the same with gy_t y_t, and X', Y' the
// same sums weighted by (t-1-i).  They obey the reverse (adjoint) recurrences
//   X_{i-1} = gy_i / D_i + e^{-w} X_i,   X'_{i-1} = e^{-w} (X'_i + X_i)   (likewise Y, Y'),
// so over a span of len positions entered with (X, X') from its right they compose as
//   X_start = X_local + e^{-w len} X,   X'_start = X'_local + e^{-w len} (X' + len X).
//
// Time-parallel in segments of kSeg steps, one thread per (b, c, segment), five launches:
//   A  each segment's forward recurrence from the empty state -> its state record;
//   B  per channel, the records combined in time order -> each segment's starting state;
//   C  each segment's forward from its starting state, keeping per position the output's
//      reference exponent q_t, normalised denominator Dn_t (D_t = Dn_t 2^{q_t}) and y_t, then
//      its adjoint recurrence from zero -> the segment's local (X, Y, X', Y');
//   D  per channel, the local sums composed right to left -> each segment's incoming sums;
//   E  each segment's adjoint recurrence from its incoming sums -> gk, gv, and gw, gu
//      partials added into the zeroed outputs with atomics.
// Numerics: the forward keeps an anchored reference p = anc - n w (no drift from rounding
// p - w); the adjoint sums are held relative to a running reference r (X = x 2^{-r}) chosen so
// every rescaling exponent is <= 0, and e^{k_i} X_i = x 2^{k_i log2 e - r} <= x because k_i
// never exceeds the reference of a later output.
#include "wkv_device.cuh"
#include "wkv_internal.h"

namespace wkvb {
namespace {

constexpr int kSeg = 64;      // time steps per segment
constexpr int kBlk = 8;       // steps whose loads are issued together
constexpr float kRNone = 3.0e38f;  // reference of an empty adjoint sum

struct Adj {
    float x, y, xp, yp, r;  // X, Y, X', Y' relative to 2^{-r}
};

__device__ __forceinline__ Adj adj_empty() { return Adj{0.f, 0.f, 0.f, 0.f, kRNone}; }

// Forward recurrence state: (a, b) relative to 2^{anc - n w2} (base 2), the record convention.
struct FwdState {
    float a, bb, anc, n;
};

// One forward step at position `at`: the output's (q, Dn, y) into the scratch planes, then the
// token folded in (decay by counting, re-anchor on a new maximum).
__device__ __forceinline__ void fwd_step(FwdState& s, float k2, float vt, float u2, float w2, float* q_out,
                                         float* d_out, float* y_out) {
    const float p = fmaf(-s.n, w2, s.anc);
    const float uk = u2 + k2;
    if (q_out) {
        const float e = ex2(-fabsf(p - uk));  // the other weight is exactly 1
        const bool cur = uk > p;
        const float e1 = cur ? e : 1.f, e2 = cur ? 1.f : e;
        const float dn = fmaf(e1, s.bb, e2);
        *q_out = fmaxf(p, uk);
        *d_out = dn;
        *y_out = fmaf(e1, s.a, e2 * vt) * rcp(dn);
    }
    const float pn = fmaf(-(s.n + 1.f), w2, s.anc);
    if (k2 > pn) {
        const float f = ex2(pn - k2);
        s.a = fmaf(f, s.a, vt);
        s.bb = fmaf(f, s.bb, 1.f);
        s.anc = k2;
        s.n = 0.f;
    } else {
        const float f = ex2(k2 - pn);
        s.a = fmaf(f, vt, s.a);
        s.bb += f;
        s.n += 1.f;
    }
}

// One adjoint step at a position (walking right to left): the position's gradients (if asked
// for) from the sums over later outputs, then its own output's terms added and the rest decayed.
template <bool OUT>
__device__ __forceinline__ void adj_step(Adj& s, float k2, float vt, float g, float q, float dn, float yt, float u2,
                                         float w2, float* gk_out, float* gv_out, float& sgw, float& sgu) {
    const float rd = rcp(dn);
    if (OUT) {
        const float cur = ex2(u2 + k2 - q) * rd;  // alpha_t / D_t
        const float ek = ex2(k2 - s.r);           // e^{k_t} 2^{-r} (0 for an empty sum)
        const float gc = g * cur;
        *gv_out = fmaf(ek, s.x, gc);
        *gk_out = fmaf(ek, fmaf(vt, s.x, -s.y), gc * (vt - yt));
        sgu = fmaf(gc, vt - yt, sgu);
        sgw = fmaf(-ek, fmaf(vt, s.xp, -s.yp), sgw);
    }
    const float rn = fminf(q, s.r + w2);
    const float sn = ex2(rn - q) * rd * g;  // gy_t / D_t in the new frame
    const float so = ex2(rn - s.r - w2);    // e^{-w} and the change of frame
    s.xp = (s.xp + s.x) * so;
    s.yp = (s.yp + s.y) * so;
    s.x = fmaf(s.x, so, sn);
    s.y = fmaf(s.y, so, sn * yt);
    s.r = rn;
}

struct BwdArgs {
    int64_t B, T, C, P;  // P segments of kSeg steps (the last may be shorter)
    const float *w, *u, *k, *v, *gy;
    float *gk, *gv, *gw, *gu;
    float *q, *dn, *y;   // [B][T][C] per-position forward values
    float* fs;           // [4][B][P][C] segment records, then starting states
    float* as;           // [5][B][P][C] local adjoint sums, then incoming sums
};

__device__ __forceinline__ int64_t seg_index(const BwdArgs& a, int64_t b, int64_t j, int64_t c) {
    return (b * a.P + j) * a.C + c;
}

// A: each segment's forward from the empty state -> its record
__global__ void __launch_bounds__(128) bwd_seg_forward(BwdArgs a) {
    const int64_t c = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int64_t j = blockIdx.y, b = blockIdx.z;
    if (c >= a.C) return;
    const float w2 = a.w[c] * kLog2e, u2 = a.u[c] * kLog2e;
    const int64_t t0 = j * kSeg, t1 = min64(a.T, t0 + kSeg);
    const int64_t base = b * a.T * a.C + c;
    FwdState s{0.f, 0.f, kPEmpty, 0.f};
    int64_t t = t0;
    for (; t + kBlk <= t1; t += kBlk) {
        float kb[kBlk], vb[kBlk];
#pragma unroll
        for (int i = 0; i < kBlk; ++i) {
            kb[i] = a.k[base + (t + i) * a.C];
            vb[i] = a.v[base + (t + i) * a.C];
        }
#pragma unroll
        for (int i = 0; i < kBlk; ++i) fwd_step(s, kb[i] * kLog2e, vb[i], u2, w2, nullptr, nullptr, nullptr);
    }
    for (; t < t1; ++t) fwd_step(s, a.k[base + t * a.C] * kLog2e, a.v[base + t * a.C], u2, w2, nullptr, nullptr, nullptr);
    const int64_t si = seg_index(a, b, j, c), SP = a.B * a.P * a.C;
    a.fs[si] = s.a;
    a.fs[SP + si] = s.bb;
    a.fs[2 * SP + si] = s.anc;
    a.fs[3 * SP + si] = s.n;
}

// B: per channel, segment records combined left to right -> each segment's starting state
__global__ void __launch_bounds__(128) bwd_seg_carry(BwdArgs a) {
    const int64_t c = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int64_t b = blockIdx.y;
    if (c >= a.C) return;
    const float w2 = a.w[c] * kLog2e;
    const int64_t SP = a.B * a.P * a.C;
    Rec run = rec_identity();
    for (int64_t j = 0; j < a.P; ++j) {
        const int64_t si = seg_index(a, b, j, c);
        const Rec seg{a.fs[si], a.fs[SP + si], a.fs[2 * SP + si], a.fs[3 * SP + si]};
        a.fs[si] = run.a;
        a.fs[SP + si] = run.b;
        a.fs[2 * SP + si] = run.anc;
        a.fs[3 * SP + si] = run.n;
        const float len = (float)(min64(a.T, (j + 1) * kSeg) - j * kSeg);
        run = rec_combine(run, seg, len, w2);
    }
}

// C: each segment's forward from its starting state (per-position values kept), then its
// adjoint recurrence from zero -> the segment's local sums
__global__ void __launch_bounds__(128) bwd_seg_values(BwdArgs a) {
    const int64_t c = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int64_t j = blockIdx.y, b = blockIdx.z;
    if (c >= a.C) return;
    const float w2 = a.w[c] * kLog2e, u2 = a.u[c] * kLog2e;
    const int64_t t0 = j * kSeg, t1 = min64(a.T, t0 + kSeg);
    const int64_t base = b * a.T * a.C + c;
    const int64_t si = seg_index(a, b, j, c), SP = a.B * a.P * a.C;
    FwdState s{a.fs[si], a.fs[SP + si], a.fs[2 * SP + si], a.fs[3 * SP + si]};
    int64_t t = t0;
    for (; t + kBlk <= t1; t += kBlk) {
        float kb[kBlk], vb[kBlk];
#pragma unroll
        for (int i = 0; i < kBlk; ++i) {
            kb[i] = a.k[base + (t + i) * a.C];
            vb[i] = a.v[base + (t + i) * a.C];
        }
#pragma unroll
        for (int i = 0; i < kBlk; ++i) {
            const int64_t at = base + (t + i) * a.C;
            fwd_step(s, kb[i] * kLog2e, vb[i], u2, w2, a.q + at, a.dn + at, a.y + at);
        }
    }
    for (; t < t1; ++t) {
        const int64_t at = base + t * a.C;
        fwd_step(s, a.k[at] * kLog2e, a.v[at], u2, w2, a.q + at, a.dn + at, a.y + at);
    }
    Adj r = adj_empty();
    float dummy_w = 0.f, dummy_u = 0.f;
    for (t = t1; t > t0; --t) {
        const int64_t at = base + (t - 1) * a.C;
        adj_step<false>(r, 0.f, 0.f, a.gy[at], a.q[at], a.dn[at], a.y[at], u2, w2, nullptr, nullptr, dummy_w,
                        dummy_u);
    }
    a.as[si] = r.x;
    a.as[SP + si] = r.y;
    a.as[2 * SP + si] = r.xp;
    a.as[3 * SP + si] = r.yp;
    a.as[4 * SP + si] = r.r;
}

// D: per channel, local sums composed right to left -> each segment's incoming sums
__global__ void __launch_bounds__(128) bwd_seg_adjoint_carry(BwdArgs a) {
    const int64_t c = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int64_t b = blockIdx.y;
    if (c >= a.C) return;
    const float w2 = a.w[c] * kLog2e;
    const int64_t SP = a.B * a.P * a.C;
    Adj in = adj_empty();  // entering the last segment from its right: nothing
    for (int64_t j = a.P - 1; j >= 0; --j) {
        const int64_t si = seg_index(a, b, j, c);
        const Adj loc{a.as[si], a.as[SP + si], a.as[2 * SP + si], a.as[3 * SP + si], a.as[4 * SP + si]};
        a.as[si] = in.x;
        a.as[SP + si] = in.y;
        a.as[2 * SP + si] = in.xp;
        a.as[3 * SP + si] = in.yp;
        a.as[4 * SP + si] = in.r;
        // what leaves this segment to its left: the local sums plus the incoming ones carried
        // across the segment's len steps
        const float len = (float)(min64(a.T, (j + 1) * kSeg) - j * kSeg);
        const float rin = in.r + len * w2;
        const float rn = fminf(loc.r, rin);
        const float fl = ex2(rn - loc.r), fi = ex2(rn - rin);
        Adj out;
        out.x = fmaf(in.x, fi, loc.x * fl);
        out.y = fmaf(in.y, fi, loc.y * fl);
        out.xp = fmaf(fmaf(len, in.x, in.xp), fi, loc.xp * fl);
        out.yp = fmaf(fmaf(len, in.y, in.yp), fi, loc.yp * fl);
        out.r = rn;
        in = out;
    }
}

// E: each segment's adjoint recurrence from its incoming sums -> gradients
__global__ void __launch_bounds__(128) bwd_seg_grads(BwdArgs a) {
    const int64_t c = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int64_t j = blockIdx.y, b = blockIdx.z;
    if (c >= a.C) return;
    const float w2 = a.w[c] * kLog2e, u2 = a.u[c] * kLog2e;
    const int64_t t0 = j * kSeg, t1 = min64(a.T, t0 + kSeg);
    const int64_t base = b * a.T * a.C + c;
    const int64_t si = seg_index(a, b, j, c), SP = a.B * a.P * a.C;
    Adj s{a.as[si], a.as[SP + si], a.as[2 * SP + si], a.as[3 * SP + si], a.as[4 * SP + si]};
    float sgw = 0.f, sgu = 0.f;
    int64_t t = t1;
    for (; t - kBlk >= t0; t -= kBlk) {
        float kb[kBlk], vb[kBlk], gb[kBlk], qb[kBlk], db[kBlk], yb[kBlk];
#pragma unroll
        for (int i = 0; i < kBlk; ++i) {
            const int64_t at = base + (t - 1 - i) * a.C;
            kb[i] = a.k[at];
            vb[i] = a.v[at];
            gb[i] = a.gy[at];
            qb[i] = a.q[at];
            db[i] = a.dn[at];
            yb[i] = a.y[at];
        }
#pragma unroll
        for (int i = 0; i < kBlk; ++i) {
            const int64_t at = base + (t - 1 - i) * a.C;
            adj_step<true>(s, kb[i] * kLog2e, vb[i], gb[i], qb[i], db[i], yb[i], u2, w2, a.gk + at, a.gv + at, sgw,
                           sgu);
        }
    }
    for (; t > t0; --t) {
        const int64_t at = base + (t - 1) * a.C;
        adj_step<true>(s, a.k[at] * kLog2e, a.v[at], a.gy[at], a.q[at], a.dn[at], a.y[at], u2, w2, a.gk + at,
                       a.gv + at, sgw, sgu);
    }
    atomicAdd(&a.gw[c], sgw);
    atomicAdd(&a.gu[c], sgu);
}

}  // namespace

int64_t backward_segments(int64_t T) { return (T + kSeg - 1) / kSeg; }

cudaError_t launch_backward(int64_t B, int64_t T, int64_t C, const float* w, const float* u, const float* k,
                            const float* v, const float* gy, float* gk, float* gv, float* gw, float* gu, void* ws,
                            cudaStream_t s) {
    cudaError_t e = cudaMemsetAsync(gw, 0, (size_t)C * sizeof(float), s);
    if (e != cudaSuccess) return e;
    e = cudaMemsetAsync(gu, 0, (size_t)C * sizeof(float), s);
    if (e != cudaSuccess) return e;
    if (B == 0 || T == 0) return cudaSuccess;
    BwdArgs a;
    a.B = B;
    a.T = T;
    a.C = C;
    a.P = backward_segments(T);
    a.w = w;
    a.u = u;
    a.k = k;
    a.v = v;
    a.gy = gy;
    a.gk = gk;
    a.gv = gv;
    a.gw = gw;
    a.gu = gu;
    float* f = static_cast<float*>(ws);
    const int64_t n = B * T * C, SP = B * a.P * C;
    a.q = f;
    a.dn = f + n;
    a.y = f + 2 * n;
    a.fs = f + 3 * n;
    a.as = a.fs + 4 * SP;
    const unsigned cx = (unsigned)((C + 127) / 128);
    const dim3 seg_grid(cx, (unsigned)a.P, (unsigned)B), chan_grid(cx, (unsigned)B);
    bwd_seg_forward<<<seg_grid, 128, 0, s>>>(a);
    bwd_seg_carry<<<chan_grid, 128, 0, s>>>(a);
    bwd_seg_values<<<seg_grid, 128, 0, s>>>(a);
    bwd_seg_adjoint_carry<<<chan_grid, 128, 0, s>>>(a);
    bwd_seg_grads<<<seg_grid, 128, 0, s>>>(a);
    return cudaGetLastError();
}

}  // namespace wkvb
