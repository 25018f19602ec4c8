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
// same sums weighted by (t-1-i).  They obey the reverse recurrences
//   X_{i-1} = gy_i / D_i + e^{-w} X_i,   X'_{i-1} = e^{-w} (X'_i + X_i)   (likewise Y, Y').
//
// One thread per (b, c) channel, two passes over time:
//   1. forward: the stabilised recurrence (anchored reference, as the serial forward) gives, per
//      position, the output's reference exponent q_t, its normalised denominator Dn_t
//      (D_t = Dn_t 2^{q_t}) and y_t, kept in the caller's workspace;
//   2. reverse: X, Y, X', Y' are held relative to a running reference r (X = x 2^{-r}) chosen
//      so every rescaling exponent is <= 0, and e^{k_i} X_i = x 2^{k_i log2 e - r} <= x since
//      k_i can never exceed the reference of a later output.
// gw, gu are summed per thread and added into the zeroed outputs with atomics.
#include "wkv_device.cuh"
#include "wkv_internal.h"

namespace wkvb {
namespace {

__global__ void __launch_bounds__(128) backward_kernel(int64_t B, int64_t T, int64_t C, const float* __restrict__ w,
                                                        const float* __restrict__ u, const float* __restrict__ k,
                                                        const float* __restrict__ v, const float* __restrict__ gy,
                                                        float* __restrict__ gk, float* __restrict__ gv,
                                                        float* __restrict__ gw, float* __restrict__ gu,
                                                        float* __restrict__ ws) {
    const int64_t c = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int64_t b = blockIdx.y;
    if (c >= C) return;
    const int64_t BTC = B * T * C;
    float* wq = ws;            // [B][T][C] output reference exponents q_t (base 2)
    float* wd = ws + BTC;      // [B][T][C] normalised denominators Dn_t
    float* wy = ws + 2 * BTC;  // [B][T][C] outputs y_t
    const float w2 = w[c] * kLog2e, u2 = u[c] * kLog2e;
    const int64_t base = b * T * C + c;

    // Both passes walk T in blocks of kBlk steps: a block's loads are all issued before its
    // first step is computed, so the recurrence waits for memory once per block, not per step.
    constexpr int kBlk = 8;

    // ---- pass 1: forward, anchored reference p = anc - n w (no drift from rounding p - w)
    float a = 0.f, bb = 0.f, anc = kPEmpty, n = 0.f;
    auto fwd_step = [&](int64_t at, float k2, float vt) {
        const float p = fmaf(-n, w2, anc);
        const float uk = u2 + k2;
        const float q = fmaxf(p, uk);
        const float e = ex2(-fabsf(p - uk));  // the other weight is exactly 1
        const bool cur = uk > p;
        const float e1 = cur ? e : 1.f, e2 = cur ? 1.f : e;
        const float dn = fmaf(e1, bb, e2);
        wq[at] = q;
        wd[at] = dn;
        wy[at] = fmaf(e1, a, e2 * vt) * rcp(dn);
        // fold the token: decay by counting, re-anchor on a new maximum
        const float pn = fmaf(-(n + 1.f), w2, anc);
        if (k2 > pn) {
            const float f = ex2(pn - k2);
            a = fmaf(f, a, vt);
            bb = fmaf(f, bb, 1.f);
            anc = k2;
            n = 0.f;
        } else {
            const float f = ex2(k2 - pn);
            a = fmaf(f, vt, a);
            bb += f;
            n += 1.f;
        }
    };
    int64_t t = 0;
    for (; t + kBlk <= T; t += kBlk) {
        float kb[kBlk], vb[kBlk];
#pragma unroll
        for (int j = 0; j < kBlk; ++j) {
            kb[j] = k[base + (t + j) * C];
            vb[j] = v[base + (t + j) * C];
        }
#pragma unroll
        for (int j = 0; j < kBlk; ++j) fwd_step(base + (t + j) * C, kb[j] * kLog2e, vb[j]);
    }
    for (; t < T; ++t) fwd_step(base + t * C, k[base + t * C] * kLog2e, v[base + t * C]);

    // ---- pass 2: reverse
    float x = 0.f, ya = 0.f, xp = 0.f, yp = 0.f;  // X, Y, X', Y' relative to 2^{-r}
    float r = 3.0e38f;                            // no later output yet
    float sgw = 0.f, sgu = 0.f;
    auto rev_step = [&](int64_t at, float k2, float vt, float g, float q, float dn, float yt) {
        const float rd = rcp(dn);
        const float cur = ex2(u2 + k2 - q) * rd;          // alpha_t / D_t
        const float ek = ex2(k2 - r);                     // e^{k_t} 2^{-r} (0 while r is the sentinel)
        const float gc = g * cur;
        gv[at] = fmaf(ek, x, gc);
        gk[at] = fmaf(ek, fmaf(vt, x, -ya), gc * (vt - yt));
        sgu = fmaf(gc, vt - yt, sgu);
        sgw = fmaf(-ek, fmaf(vt, xp, -yp), sgw);
        // move the accumulators to position t - 1: add this output's terms, decay the rest
        const float rn = fminf(q, r + w2);
        const float sn = ex2(rn - q) * rd * g;            // gy_t / D_t in the new frame
        const float so = ex2(rn - r - w2);                // e^{-w} and the change of frame
        xp = (xp + x) * so;
        yp = (yp + ya) * so;
        x = fmaf(x, so, sn);
        ya = fmaf(ya, so, sn * yt);
        r = rn;
    };
    t = T;
    for (; t - kBlk >= 0; t -= kBlk) {
        float kb[kBlk], vb[kBlk], gb[kBlk], qb[kBlk], db[kBlk], yb[kBlk];
#pragma unroll
        for (int j = 0; j < kBlk; ++j) {
            const int64_t at = base + (t - 1 - j) * C;
            kb[j] = k[at];
            vb[j] = v[at];
            gb[j] = gy[at];
            qb[j] = wq[at];
            db[j] = wd[at];
            yb[j] = wy[at];
        }
#pragma unroll
        for (int j = 0; j < kBlk; ++j)
            rev_step(base + (t - 1 - j) * C, kb[j] * kLog2e, vb[j], gb[j], qb[j], db[j], yb[j]);
    }
    for (; t > 0; --t) {
        const int64_t at = base + (t - 1) * C;
        rev_step(at, k[at] * kLog2e, v[at], gy[at], wq[at], wd[at], wy[at]);
    }
    atomicAdd(&gw[c], sgw);
    atomicAdd(&gu[c], sgu);
}

}  // namespace

cudaError_t launch_backward(int64_t B, int64_t T, int64_t C, const float* w, const float* u, const float* k,
                            const float* v, const float* gy, float* gk, float* gv, float* gw, float* gu, void* ws,
                            cudaStream_t s) {
    cudaError_t e = cudaMemsetAsync(gw, 0, (size_t)C * sizeof(float), s);
    if (e != cudaSuccess) return e;
    e = cudaMemsetAsync(gu, 0, (size_t)C * sizeof(float), s);
    if (e != cudaSuccess) return e;
    if (B == 0 || T == 0) return cudaSuccess;
    const dim3 grid((unsigned)((C + 127) / 128), (unsigned)B);
    backward_kernel<<<grid, 128, 0, s>>>(B, T, C, w, u, k, v, gy, gk, gv, gw, gu, static_cast<float*>(ws));
    return cudaGetLastError();
}

}  // namespace wkvb
