// Decode-step and token-shift kernels (elementwise, HBM-bound).
//
// Decode: for every row (session n, layer l) and channel c, emit wkv for the new
// token from the stored (a, b, p) and fold the token in (aiwiki "RWKV": the
// one-token decode step; transformer-math page, section "Numerical stability:
// carry the exponent").  The fused variant first forms the token-shift lerp
// xbar = mu x_t + (1 - mu) x_prev (transformer-math page, section "Token shift: a
// two-tap causal convolution").  Work is laid out as a 2-D grid: x covers a row's
// channels in 4-wide vectors (one 16-byte access per array per thread), y walks the
// rows, so no per-element division is needed.  States stay in natural units.
#include "wkv_device.cuh"
#include "wkv_internal.h"
#include "wkv_vec.cuh"

namespace wkvb {
namespace {

template <int V>
struct F;
template <>
struct F<4> {
    static __device__ __forceinline__ void ld(const float* p, float (&o)[4]) {
        float4 t = __ldcs(reinterpret_cast<const float4*>(p));
        o[0] = t.x; o[1] = t.y; o[2] = t.z; o[3] = t.w;
    }
    static __device__ __forceinline__ void ld_keep(const float* p, float (&o)[4]) {
        float4 t = __ldg(reinterpret_cast<const float4*>(p));
        o[0] = t.x; o[1] = t.y; o[2] = t.z; o[3] = t.w;
    }
    static __device__ __forceinline__ void st(float* p, const float (&o)[4]) {
        __stcs(reinterpret_cast<float4*>(p), make_float4(o[0], o[1], o[2], o[3]));
    }
};
template <>
struct F<1> {
    static __device__ __forceinline__ void ld(const float* p, float (&o)[1]) { o[0] = __ldcs(p); }
    static __device__ __forceinline__ void ld_keep(const float* p, float (&o)[1]) { o[0] = __ldg(p); }
    static __device__ __forceinline__ void st(float* p, const float (&o)[1]) { __stcs(p, o[0]); }
};

template <bool FUSED, int V>
__global__ void __launch_bounds__(256) decode_kernel(int64_t rows, int64_t L, int64_t C, const float* __restrict__ mu,
                                                     const float* __restrict__ w, const float* __restrict__ u,
                                                     const float* __restrict__ x_t, const float* __restrict__ x_prev,
                                                     float* __restrict__ xbar, const float* __restrict__ k,
                                                     const float* __restrict__ v, float* __restrict__ st,
                                                     float* __restrict__ y) {
    grid_dep_launch_dependents();
    grid_dep_wait();  // before any global memory access
    const int64_t RC = rows * C;
    const int64_t c = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) * V;
    if (c >= C) return;
    for (int64_t row = blockIdx.y; row < rows; row += gridDim.y) {
        const int64_t l = row % L;
        const int64_t i = row * C + c;
        const int64_t pi = l * C + c;
        float kk[V], vv[V], a[V], bb[V], p[V], ww[V], uu[V], yy[V];
        F<V>::ld(k + i, kk);
        F<V>::ld(v + i, vv);
        F<V>::ld(st + i, a);
        F<V>::ld(st + RC + i, bb);
        F<V>::ld(st + 2 * RC + i, p);
        F<V>::ld_keep(w + pi, ww);
        F<V>::ld_keep(u + pi, uu);
        if (FUSED) {
            float m[V], xt[V], xp[V], xb[V];
            F<V>::ld_keep(mu + pi, m);
            F<V>::ld(x_t + i, xt);
            F<V>::ld(x_prev + i, xp);
#pragma unroll
            for (int q = 0; q < V; ++q) xb[q] = fmaf(m[q], xt[q], (1.f - m[q]) * xp[q]);
            F<V>::st(xbar + i, xb);
        }
#pragma unroll
        for (int q = 0; q < V; ++q) {
            yy[q] = wkv_output<true>(a[q], bb[q], p[q], uu[q] + kk[q], vv[q]);
            wkv_fold<true>(a[q], bb[q], p[q], p[q] - ww[q], kk[q], vv[q], ww[q]);
        }
        F<V>::st(y + i, yy);
        F<V>::st(st + i, a);
        F<V>::st(st + RC + i, bb);
        F<V>::st(st + 2 * RC + i, p);
    }
}

template <int V>
__global__ void __launch_bounds__(256) token_shift_kernel(int64_t B, int64_t T, int64_t C, const float* __restrict__ mu,
                                                          const float* __restrict__ x,
                                                          const float* __restrict__ x_last,
                                                          float* __restrict__ xbar) {
    grid_dep_launch_dependents();
    grid_dep_wait();  // before any global memory access
    const int64_t c = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) * V;
    if (c >= C) return;
    float m[V];
    F<V>::ld_keep(mu + c, m);
    const int64_t rows = B * T;
    for (int64_t row = blockIdx.y; row < rows; row += gridDim.y) {
        const int64_t b = row / T, t = row % T;
        float xt[V], xp[V], xb[V];
        F<V>::ld_keep(x + row * C + c, xt);
        if (t > 0) {
            F<V>::ld_keep(x + (row - 1) * C + c, xp);
        } else if (x_last) {
            F<V>::ld_keep(x_last + b * C + c, xp);
        } else {
#pragma unroll
            for (int q = 0; q < V; ++q) xp[q] = 0.f;
        }
#pragma unroll
        for (int q = 0; q < V; ++q) xb[q] = fmaf(m[q], xt[q], (1.f - m[q]) * xp[q]);
        F<V>::st(xbar + row * C + c, xb);
    }
}

// Token shift of the three projections (transformer-math page, section "Token shift": each of
// r, k, v has its own mu): x_t and x_{t-1} are read once and three lerps are written.
template <int V>
__global__ void __launch_bounds__(256) token_shift3_kernel(int64_t B, int64_t T, int64_t C, const float* __restrict__ mu_r,
                                                           const float* __restrict__ mu_k, const float* __restrict__ mu_v,
                                                           const float* __restrict__ x, const float* __restrict__ x_last,
                                                           float* __restrict__ xr, float* __restrict__ xk,
                                                           float* __restrict__ xv) {
    grid_dep_launch_dependents();
    grid_dep_wait();  // before any global memory access
    const int64_t c = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) * V;
    if (c >= C) return;
    float mr[V], mk[V], mv[V];
    F<V>::ld_keep(mu_r + c, mr);
    F<V>::ld_keep(mu_k + c, mk);
    F<V>::ld_keep(mu_v + c, mv);
    const int64_t rows = B * T;
    for (int64_t row = blockIdx.y; row < rows; row += gridDim.y) {
        const int64_t b = row / T, t = row % T;
        float xt[V], xp[V], o[V];
        F<V>::ld_keep(x + row * C + c, xt);
        if (t > 0) {
            F<V>::ld_keep(x + (row - 1) * C + c, xp);
        } else if (x_last) {
            F<V>::ld_keep(x_last + b * C + c, xp);
        } else {
#pragma unroll
            for (int q = 0; q < V; ++q) xp[q] = 0.f;
        }
#pragma unroll
        for (int q = 0; q < V; ++q) o[q] = fmaf(mr[q], xt[q], (1.f - mr[q]) * xp[q]);
        F<V>::st(xr + row * C + c, o);
#pragma unroll
        for (int q = 0; q < V; ++q) o[q] = fmaf(mk[q], xt[q], (1.f - mk[q]) * xp[q]);
        F<V>::st(xk + row * C + c, o);
#pragma unroll
        for (int q = 0; q < V; ++q) o[q] = fmaf(mv[q], xt[q], (1.f - mv[q]) * xp[q]);
        F<V>::st(xv + row * C + c, o);
    }
}

// The receptance gate applied in place, y <- sigma(r) * y (transformer-math page, section
// "Receptance: the gate on the way out"), for paths whose forward kernel does not fuse it.
// sigma(r) = 1 / (1 + 2^(-r log2 e)); for r -> -inf the exponential is +inf and the gate 0.
template <typename TIO, int V>
__global__ void __launch_bounds__(256) gate_kernel(int64_t n, const TIO* __restrict__ r, TIO* __restrict__ y) {
    grid_dep_launch_dependents();
    grid_dep_wait();  // before any global memory access
    const int64_t stride = (int64_t)gridDim.x * blockDim.x * V;
    for (int64_t i = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) * V; i < n; i += stride) {
        float rv[V], yv[V];
        Vec<TIO, V>::load(r + i, rv);
        Vec<TIO, V>::load(y + i, yv);
#pragma unroll
        for (int q = 0; q < V; ++q) yv[q] *= rcp(1.f + ex2(-rv[q] * kLog2e));
        Vec<TIO, V>::store(y + i, yv);
    }
}

__global__ void passthrough_kernel(int64_t BC, const float* in, float* out) {
    grid_dep_launch_dependents();
    grid_dep_wait();  // before any global memory access
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < 3 * BC; i += (int64_t)gridDim.x * blockDim.x)
        out[i] = in ? in[i] : (i < 2 * BC ? 0.f : kPEmpty);
}

dim3 grid2d(int64_t C, int V, int64_t rows) {
    const int64_t per_row = (C + (int64_t)V * 256 - 1) / ((int64_t)V * 256);
    return dim3((unsigned)per_row, (unsigned)(rows < 65535 ? rows : 65535), 1);
}

}  // namespace

cudaError_t launch_decode_step(int64_t N, int64_t L, int64_t C, const float* mu, const float* w, const float* u,
                               const float* x_t, const float* x_prev, float* xbar, const float* k, const float* v,
                               float* state, float* y, cudaStream_t s) {
    const int64_t rows = N * L;
    const bool fused = mu != nullptr;
    const bool vec = (C % 4) == 0;
    const dim3 grid = grid2d(C, vec ? 4 : 1, rows);
    if (fused) {
        if (vec)
            return launch_pdl(decode_kernel<true, 4>, dim3(grid), dim3(256), 0, s,
                              rows, L, C, mu, w, u, x_t, x_prev, xbar, k, v, state, y);
        else
            return launch_pdl(decode_kernel<true, 1>, dim3(grid), dim3(256), 0, s,
                              rows, L, C, mu, w, u, x_t, x_prev, xbar, k, v, state, y);
    } else {
        if (vec)
            return launch_pdl(decode_kernel<false, 4>, dim3(grid), dim3(256), 0, s,
                              rows, L, C, mu, w, u, x_t, x_prev, xbar, k, v, state, y);
        else
            return launch_pdl(decode_kernel<false, 1>, dim3(grid), dim3(256), 0, s,
                              rows, L, C, mu, w, u, x_t, x_prev, xbar, k, v, state, y);
    }
}

cudaError_t launch_token_shift(int64_t B, int64_t T, int64_t C, const float* mu, const float* x, const float* x_last,
                               float* xbar, cudaStream_t s) {
    const bool vec = (C % 4) == 0;
    const dim3 grid = grid2d(C, vec ? 4 : 1, B * T);
    if (vec)
        return launch_pdl(token_shift_kernel<4>, dim3(grid), dim3(256), 0, s, B, T, C, mu, x, x_last, xbar);
    else
        return launch_pdl(token_shift_kernel<1>, dim3(grid), dim3(256), 0, s, B, T, C, mu, x, x_last, xbar);
}

cudaError_t launch_state_passthrough(int64_t BC, const float* state_in, float* state_out, cudaStream_t s) {
    const int64_t n = 3 * BC;
    const int64_t blocks = (n + 255) / 256 < 148 * 16 ? (n + 255) / 256 : 148 * 16;
    return launch_pdl(passthrough_kernel, dim3((unsigned)blocks), dim3(256), 0, s, BC, state_in, state_out);
}

cudaError_t launch_token_shift3(int64_t B, int64_t T, int64_t C, const float* mu_r, const float* mu_k,
                                const float* mu_v, const float* x, const float* x_last, float* xr, float* xk, float* xv,
                                cudaStream_t s) {
    const bool vec = (C % 4) == 0;
    const dim3 grid = grid2d(C, vec ? 4 : 1, B * T);
    if (vec)
        return launch_pdl(token_shift3_kernel<4>, dim3(grid), dim3(256), 0, s,
                          B, T, C, mu_r, mu_k, mu_v, x, x_last, xr, xk, xv);
    else
        return launch_pdl(token_shift3_kernel<1>, dim3(grid), dim3(256), 0, s,
                          B, T, C, mu_r, mu_k, mu_v, x, x_last, xr, xk, xv);
}

cudaError_t launch_gate(int64_t n, int io, const void* r, void* y, cudaStream_t s) {
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    auto blocks = [&](int64_t units) {
        const int64_t b = (units + 255) / 256;
        const int64_t cap = (int64_t)sms * 8;
        return (unsigned)(b < cap ? (b > 0 ? b : 1) : cap);
    };
    if (io == 1) {
        const __nv_bfloat16* rr = static_cast<const __nv_bfloat16*>(r);
        __nv_bfloat16* yy = static_cast<__nv_bfloat16*>(y);
        if (n % 8 == 0)
            return launch_pdl(gate_kernel<__nv_bfloat16, 8>, dim3(blocks(n / 8)), dim3(256), 0, s, n, rr, yy);
        else
            return launch_pdl(gate_kernel<__nv_bfloat16, 1>, dim3(blocks(n)), dim3(256), 0, s, n, rr, yy);
    } else {
        const float* rr = static_cast<const float*>(r);
        float* yy = static_cast<float*>(y);
        if (n % 4 == 0)
            return launch_pdl(gate_kernel<float, 4>, dim3(blocks(n / 4)), dim3(256), 0, s, n, rr, yy);
        else
            return launch_pdl(gate_kernel<float, 1>, dim3(blocks(n)), dim3(256), 0, s, n, rr, yy);
    }
}

}  // namespace wkvb
