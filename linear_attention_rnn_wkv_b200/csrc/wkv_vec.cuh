// Vector loads and stores of V adjacent channels (fp32 or bf16 in memory, fp32 in
// registers), shared by the forward kernels.
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

namespace wkvb {

template <typename TIO, int V>
struct Vec;

template <>
struct Vec<float, 1> {
    static __device__ __forceinline__ void load(const float* p, float (&o)[1]) { o[0] = *p; }
    static __device__ __forceinline__ void store(float* p, const float (&o)[1]) { *p = o[0]; }
};
template <>
struct Vec<float, 2> {
    static __device__ __forceinline__ void load(const float* p, float (&o)[2]) {
        float2 t = *reinterpret_cast<const float2*>(p);
        o[0] = t.x; o[1] = t.y;
    }
    static __device__ __forceinline__ void store(float* p, const float (&o)[2]) {
        *reinterpret_cast<float2*>(p) = make_float2(o[0], o[1]);
    }
};
template <>
struct Vec<float, 4> {
    static __device__ __forceinline__ void load(const float* p, float (&o)[4]) {
        float4 t = *reinterpret_cast<const float4*>(p);
        o[0] = t.x; o[1] = t.y; o[2] = t.z; o[3] = t.w;
    }
    static __device__ __forceinline__ void store(float* p, const float (&o)[4]) {
        *reinterpret_cast<float4*>(p) = make_float4(o[0], o[1], o[2], o[3]);
    }
};

__device__ __forceinline__ float bf_lo(uint32_t x) { return __uint_as_float(x << 16); }
__device__ __forceinline__ float bf_hi(uint32_t x) { return __uint_as_float(x & 0xFFFF0000u); }
__device__ __forceinline__ uint32_t bf_pack(float lo, float hi) {
    __nv_bfloat162 t = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&t);
}

template <>
struct Vec<__nv_bfloat16, 1> {
    static __device__ __forceinline__ void load(const __nv_bfloat16* p, float (&o)[1]) { o[0] = __bfloat162float(*p); }
    static __device__ __forceinline__ void store(__nv_bfloat16* p, const float (&o)[1]) { *p = __float2bfloat16_rn(o[0]); }
};
template <>
struct Vec<__nv_bfloat16, 2> {
    static __device__ __forceinline__ void load(const __nv_bfloat16* p, float (&o)[2]) {
        uint32_t t = *reinterpret_cast<const uint32_t*>(p);
        o[0] = bf_lo(t); o[1] = bf_hi(t);
    }
    static __device__ __forceinline__ void store(__nv_bfloat16* p, const float (&o)[2]) {
        *reinterpret_cast<uint32_t*>(p) = bf_pack(o[0], o[1]);
    }
};
template <>
struct Vec<__nv_bfloat16, 4> {
    static __device__ __forceinline__ void load(const __nv_bfloat16* p, float (&o)[4]) {
        uint2 t = *reinterpret_cast<const uint2*>(p);
        o[0] = bf_lo(t.x); o[1] = bf_hi(t.x); o[2] = bf_lo(t.y); o[3] = bf_hi(t.y);
    }
    static __device__ __forceinline__ void store(__nv_bfloat16* p, const float (&o)[4]) {
        *reinterpret_cast<uint2*>(p) = make_uint2(bf_pack(o[0], o[1]), bf_pack(o[2], o[3]));
    }
};
template <>
struct Vec<__nv_bfloat16, 8> {
    static __device__ __forceinline__ void load(const __nv_bfloat16* p, float (&o)[8]) {
        uint4 t = *reinterpret_cast<const uint4*>(p);
        o[0] = bf_lo(t.x); o[1] = bf_hi(t.x); o[2] = bf_lo(t.y); o[3] = bf_hi(t.y);
        o[4] = bf_lo(t.z); o[5] = bf_hi(t.z); o[6] = bf_lo(t.w); o[7] = bf_hi(t.w);
    }
    static __device__ __forceinline__ void store(__nv_bfloat16* p, const float (&o)[8]) {
        *reinterpret_cast<uint4*>(p) = make_uint4(bf_pack(o[0], o[1]), bf_pack(o[2], o[3]), bf_pack(o[4], o[5]),
                                                  bf_pack(o[6], o[7]));
    }
};

}  // namespace wkvb
