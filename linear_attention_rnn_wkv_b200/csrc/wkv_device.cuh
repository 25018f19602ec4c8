// Device-side numerics shared by the WKV kernels (sm_100a).
//
// Notation follows the RWKV transformer-math page (aicassindra.com, tm_rwkv_math),
// section "Numerical stability: carry the exponent": a channel's state is (a, b, p)
// with true accumulators A = a e^p, B = b e^p, and every exponent handed to exp is
// <= 0 (up to rounding).
//
// Two exponent domains are used:
//  * natural (the ABI's): exp(x) is evaluated as 2^(x * log2 e);
//  * base 2 (inside the forward kernels): k, w, u and p are pre-multiplied by
//    log2 e once, so exp is a single ex2.  States cross the ABI in natural units.
//
// Rounding.  The page's update p' = max(p - w, k), a' = e^{p-w-p'} a + e^{k-p'} v
// rounds p - w at every step, and in fp32 that rounding error repeats (w is constant
// and p stays in one binade), so the true accumulators A = a e^p drift linearly.  Two
// ways of evaluating the same real-number arithmetic avoid it:
//  (1) scans keep (a, b) relative to the exact exponent anc - n w, where anc is the key
//      (or carried exponent) that set the maximum and n counts the steps since: the
//      history then decays by incrementing n, without touching a or b, and rounding
//      enters only through the argument of each exp (once per term).  Used by the
//      forward kernels and the segment records (Rec);
//  (2) the decode step, whose state crosses the ABI as an explicit p, evaluates the
//      history factor's exponent as (p - p') - w -- the exact rounding residual of p'
//      when p' = p - w -- and applies it as a + (e^x - 1) a with a Taylor polynomial
//      for e^x - 1 (wkv_fold).  Over 128 steps that keeps the state within a few 1e-6.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace wkvb {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.69314718055994531f;
// Exponent of the empty state (a = b = 0): finite so p - w never forms inf - inf.
constexpr float kPEmpty = -1e38f;

__host__ __device__ __forceinline__ int64_t min64(int64_t a, int64_t b) { return a < b ? a : b; }

// ---------------------------------------------------------------------------
// Hardware approximations (MUFU): 2^x and 1/x, flush-to-zero.
// ex2.approx of a large negative argument returns +0, which is the intended
// weight of the empty state.
// ---------------------------------------------------------------------------
__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ float rcp(float x) {
    float y;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// exp in the chosen domain
template <bool NAT>
__device__ __forceinline__ float expd(float x) {
    return NAT ? ex2(x * kLog2e) : ex2(x);
}

// e^y - 1 (NAT) or 2^y - 1 (base 2) for |y| well below 1: fourth-order Taylor
// polynomial of e^z - 1 in z = y (or y ln 2); relative error < 1e-8 for |z| < 2^-4.
// The argument is clamped to [-1, 1] so degenerate (empty-state) inputs stay finite.
template <bool NAT>
__device__ __forceinline__ float expm1d_small(float y) {
    float z = fminf(fmaxf(NAT ? y : y * kLn2, -1.f), 1.f);
    return z * fmaf(z, fmaf(z, fmaf(z, 1.f / 24.f, 1.f / 6.f), 0.5f), 1.f);
}

// ---------------------------------------------------------------------------
// Output of the current token from a state:  q = max(p, u + k),
//   y = (e^{p-q} a + e^{u+k-q} v) / (e^{p-q} b + e^{u+k-q}).
// One of the two weights is exactly 1, so a single exp is needed.
// uk = u + k in the domain's units.
// ---------------------------------------------------------------------------
template <bool NAT>
__device__ __forceinline__ float wkv_output(float a, float b, float p, float uk, float v) {
    float d = p - uk;
    float e = expd<NAT>(-fabsf(d));
    bool hist = d >= 0.f;
    float sa = hist ? 1.f : e;
    float sv = hist ? e : 1.f;
    return fmaf(sv, v, sa * a) * rcp(fmaf(sa, b, sv));
}

// ---------------------------------------------------------------------------
// Fold token (k, v) into the state:  p' = max(p - w, k),
//   a' = e^{p-w-p'} a + e^{k-p'} v,  b' = e^{p-w-p'} b + e^{k-p'}.
// pd is the candidate p - w (the caller may compute it from an anchor).
// ---------------------------------------------------------------------------
template <bool NAT>
__device__ __forceinline__ void wkv_fold(float& a, float& b, float& p, float pd, float k, float v, float w) {
    bool keep = pd >= k;                   // history still holds the maximum
    float pn = keep ? pd : k;
    float x = (p - pn) - w;                // keep: rounding residual of pd; else p - k - w
    float f = expd<NAT>(keep ? (k - pn) : x);
    float m = keep ? expm1d_small<NAT>(x) : f;
    float nf = keep ? f : 1.f;
    a = fmaf(nf, v, fmaf(m, a, keep ? a : 0.f));
    b = nf + fmaf(m, b, keep ? b : 0.f);
    p = pn;
}

// ---------------------------------------------------------------------------
// Anchored segment record (base-2 units): accumulators (a, b) relative to the exact
// exponent anc - n w (a real number; rec_p gives its fp32 value with one rounding).
// Decaying a record by `len` steps only adds len to n.  The identity (empty segment)
// is (0, 0, kPEmpty, 0).
// ---------------------------------------------------------------------------
struct Rec {
    float a, b, anc, n;
};

__device__ __forceinline__ Rec rec_identity() { return Rec{0.f, 0.f, kPEmpty, 0.f}; }

__device__ __forceinline__ float rec_p(const Rec& r, float w2) { return fmaf(-r.n, w2, r.anc); }

// left (earlier) then right (later, spanning len steps): the left decays over len
// steps (the telescoping of the decay factor, transformer-math page, section "Why
// it collapses into a recurrence"); the larger exponent stays the reference and the
// other record is scaled onto it with one exp.
__device__ __forceinline__ Rec rec_combine(const Rec& L, const Rec& R, float len, float w2) {
    const float nl = L.n + len;
    const float pl = fmaf(-nl, w2, L.anc);
    const float pr = fmaf(-R.n, w2, R.anc);
    const bool keep = pl >= pr;
    const float f = ex2(-fabsf(pl - pr));
    Rec o;
    if (keep) {
        o.a = fmaf(f, R.a, L.a);
        o.b = fmaf(f, R.b, L.b);
        o.anc = L.anc;
        o.n = nl;
    } else {
        o.a = fmaf(f, L.a, R.a);
        o.b = fmaf(f, L.b, R.b);
        o.anc = R.anc;
        o.n = R.n;
    }
    return o;
}

// One token of a long scan in the anchored form (base-2 units): output from the
// state before the token, then fold the token in.  (a, b) are relative to anc - n w.
__device__ __forceinline__ float scan_step(float& a, float& b, float& anc, float& n, float k2, float v, float u2,
                                           float w2) {
    const float p = fmaf(-n, w2, anc);
    const float y = wkv_output<false>(a, b, p, u2 + k2, v);
    const float n1 = n + 1.f;
    const float pd = fmaf(-n1, w2, anc);   // the history's exponent after decaying one step
    const bool keep = pd >= k2;            // history still holds the maximum
    const float e = ex2(-fabsf(k2 - pd));  // the smaller of the two weights
    const float sa = keep ? 1.f : e;
    const float sv = keep ? e : 1.f;
    a = fmaf(sv, v, sa * a);
    b = fmaf(sa, b, sv);
    anc = keep ? anc : k2;
    n = keep ? n1 : 0.f;
    return y;
}

// ---------------------------------------------------------------------------
// Record packing and the one-exp chunk step used by the chunked forward kernels
// ---------------------------------------------------------------------------
__device__ __forceinline__ float4 rec_pack(const Rec& r) { return make_float4(r.a, r.b, r.anc, r.n); }
__device__ __forceinline__ Rec rec_unpack(const float4& f) { return Rec{f.x, f.y, f.z, f.w}; }

// Natural-units state (a, b, p) -> anchored base-2 record.
__device__ __forceinline__ Rec rec_from_state(const float* st, int64_t bc, int64_t BC) {
    return Rec{st[bc], st[BC + bc], st[2 * BC + bc] * kLog2e, 0.f};
}

// One token within a chunk, one exp for both the output and the update.
// State (a, b) is relative to the reference exponent r = R - n w (base 2, exact real;
// the history decays by counting n), i.e. A = a 2^r.  With D = (u + k) - r, E = 2^-|D|:
//   D <= 0 (history dominates): y = (a + E v)/(b + E); the new token's weight relative to
//          the decayed reference r - w is 2^(k - r + w) = E * c with c = 2^(w - u), so
//          a += E c v, b += E c, n += 1;
//   D > 0  (token dominates):   y = (E a + v)/(E b + 1); re-reference to u + k:
//          a = E a + c v, b = E b + c, R = u + k, n = 1.
// Exact in real arithmetic; valid while c and its reciprocal stay far from the fp32
// range limits (callers check |u|, w <= kLazyLimit).
__device__ __forceinline__ float lazy_step(float& a, float& b, float& R, float& n, float k2, float v, float u2,
                                           float w2, float c) {
    const float r = fmaf(-n, w2, R);
    const float uk = u2 + k2;
    const float d = uk - r;
    const float e = ex2(-fabsf(d));
    const bool cur = d > 0.f;
    const float sa = cur ? e : 1.f;
    const float sv = cur ? 1.f : e;
    const float t = sa * a;
    const float y = fmaf(sv, v, t) * rcp(fmaf(sa, b, sv));
    const float nw = sv * c;
    a = fmaf(nw, v, t);
    b = fmaf(sa, b, nw);
    R = cur ? uk : R;
    n = cur ? 1.f : n + 1.f;
    return y;
}
constexpr float kLazyLimit = 40.f;  // base-2 units: c = 2^(w - u) within 2^(+-80)

// ---------------------------------------------------------------------------
// I/O element conversions
// ---------------------------------------------------------------------------
template <typename T>
struct io;

template <>
struct io<float> {
    static __device__ __forceinline__ float load(const float* p) { return *p; }
    static __device__ __forceinline__ void store(float* p, float x) { *p = x; }
    static __device__ __forceinline__ float to_f(float x) { return x; }
    static __device__ __forceinline__ float from_f(float x) { return x; }
};

template <>
struct io<__nv_bfloat16> {
    static __device__ __forceinline__ float load(const __nv_bfloat16* p) { return __bfloat162float(*p); }
    static __device__ __forceinline__ void store(__nv_bfloat16* p, float x) { *p = __float2bfloat16_rn(x); }
    static __device__ __forceinline__ float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }
    static __device__ __forceinline__ __nv_bfloat16 from_f(float x) { return __float2bfloat16_rn(x); }
};

// ---------------------------------------------------------------------------
// Async bulk copies (TMA engine, non-tensor form) and mbarriers.  No cluster
// multicast is used anywhere.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}

// Returns true once the phase with the given parity has completed.
// As mbar_try_wait, but the thread is suspended (issuing nothing) until the phase
// completes or about `hint_ns` nanoseconds pass.
__device__ __forceinline__ bool mbar_try_wait_hint(uint64_t* bar, uint32_t parity, uint32_t hint_ns) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred P;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 P, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, P;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity), "r"(hint_ns)
        : "memory");
    return ok != 0;
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred P;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 P, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, P;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Non-blocking test: true once the phase with the given parity has completed (the thread is
// never suspended, so a caller that must also watch another condition sees it promptly).
__device__ __forceinline__ bool mbar_test_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred P;\n\t"
        "mbarrier.test_wait.parity.shared::cta.b64 P, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, P;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Global -> shared bulk copy of `bytes` (multiple of 16, both addresses 16-B aligned),
// completion signalled on `bar` as transaction bytes.
__device__ __forceinline__ void bulk_g2s(void* dst_smem, const void* src_gmem, uint32_t bytes, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_u32(dst_smem)),
        "l"(src_gmem), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

// ---------------------------------------------------------------------------
// GPU-scope acquire/release on 32-bit flags (decoupled look-back).
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t ld_acquire_u32(const uint32_t* p) {
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ uint32_t ld_relaxed_u32(const uint32_t* p) {
    uint32_t v;
    asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ uint64_t ld_relaxed_u64(const uint64_t* p) {
    uint64_t v;
    asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ void st_relaxed_u64(uint64_t* p, uint64_t v) {
    asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}

// Two adjacent 64-bit words in one 16-byte access (p 16-byte aligned); each word is its
// own single-copy-atomic element, the pair is not.
__device__ __forceinline__ void ld_relaxed_v2u64(const uint64_t* p, uint64_t& x, uint64_t& y) {
    asm volatile("ld.relaxed.gpu.global.v2.u64 {%0, %1}, [%2];" : "=l"(x), "=l"(y) : "l"(p) : "memory");
}

__device__ __forceinline__ void st_relaxed_v2u64(uint64_t* p, uint64_t x, uint64_t y) {
    asm volatile("st.relaxed.gpu.global.v2.u64 [%0], {%1, %2};" ::"l"(p), "l"(x), "l"(y) : "memory");
}

// Makes earlier relaxed loads acquire: later accesses see what their writers released.
__device__ __forceinline__ void fence_acquire_gpu() { asm volatile("fence.acq_rel.gpu;" ::: "memory"); }

// Programmatic dependent launch: a kernel launched with programmatic stream serialisation may
// be scheduled while the stream's previous kernel is still running; it runs its prologue
// (shared and tensor memory, barriers) and then waits here, before its first access to global
// memory, until that kernel has completed and its writes are visible.  Without the attribute
// the wait returns at once.  launch_dependents lets the next such kernel be scheduled early.
__device__ __forceinline__ void grid_dep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void grid_dep_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

__device__ __forceinline__ void st_release_u32(uint32_t* p, uint32_t v) {
    asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ float4 ld_relaxed_f4(const float4* p) {
    float4 r;
    asm volatile("ld.relaxed.gpu.global.v4.f32 {%0, %1, %2, %3}, [%4];"
                 : "=f"(r.x), "=f"(r.y), "=f"(r.z), "=f"(r.w)
                 : "l"(p)
                 : "memory");
    return r;
}

}  // namespace wkvb
