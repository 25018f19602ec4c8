// Pieces shared by the pipelined chunked forward kernels: bounded mbarrier waits, TMA tile
// loads and their tensor maps, and the fence-free tagged records of the decoupled
// look-back.  Included by one translation unit per kernel (everything here has internal
// linkage).
#pragma once

#include <cuda.h>
#include <cudaTypedefs.h>

#include "wkv_device.cuh"
#include "wkv_internal.h"

// Per-unit event trace (profiling builds only): compiled with -DWKV_TRACE, the kernel
// stamps %globaltimer at each hand-over of every unit into the buffer registered with
// wkv_trace_set_buffer ([units][11] u64: events 0..9 below, slot 10 the SM id).  Normal
// builds define the hooks away.
#ifdef WKV_TRACE
static __device__ unsigned long long* g_wkv_trace = nullptr;
__device__ __forceinline__ void wkv_trace(int64_t unit, int ev) {
    if (!g_wkv_trace) return;
    unsigned long long t;
    asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
    g_wkv_trace[unit * 11 + ev] = t;
    if (ev == 0) {
        unsigned sm;
        asm volatile("mov.u32 %0, %smid;" : "=r"(sm));
        g_wkv_trace[unit * 11 + 10] = sm;
    }
}
#define WKV_TRACE_EVENT(unit, ev) wkv_trace(unit, ev)
// per block, after the units' events: [2] = block start, block end
__device__ __forceinline__ void wkv_trace_block(int64_t units, int ev) {
    if (!g_wkv_trace) return;
    unsigned long long t;
    asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
    g_wkv_trace[units * 11 + blockIdx.x * 2 + ev] = t;
}
#define WKV_TRACE_BLOCK(units, ev) wkv_trace_block(units, ev)
// per block and warp, after the blocks' events: [24] = each warp's role end (warps 0-19), then
// the block's SM id
__device__ __forceinline__ void wkv_trace_warp(int64_t units, int warp) {
    if (!g_wkv_trace) return;
    unsigned long long t;
    asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
    unsigned long long* base = g_wkv_trace + units * 11 + 2 * 148 + blockIdx.x * 24;
    base[warp] = t;
    if (warp == 0) {
        unsigned sm;
        asm volatile("mov.u32 %0, %smid;" : "=r"(sm));
        base[20] = sm;
    }
}
#define WKV_TRACE_WARP(units, warp) wkv_trace_warp(units, warp)
#else
#define WKV_TRACE_WARP(units, warp) ((void)0)
#define WKV_TRACE_EVENT(unit, ev) ((void)0)
#define WKV_TRACE_BLOCK(units, ev) ((void)0)
#endif
// events: 0 ticket, 1 tile loaded, 2 chunks summarised, 3 look-back start, 4 summaries
// scanned, 5 carry known, 6 carry handed over, 7 records published, 8 emit start, 9 emit end

namespace wkvb {
namespace {

// Rows per TMA box (a tile of Ts rows is fetched as Ts / kBoxRows boxes per array).
constexpr int kBoxRows = 32;

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// Suspend-time hint of the mbarrier waits, in nanoseconds.
constexpr uint32_t kWaitHintNs = 250;

// Bounded wait on an mbarrier phase; returns false if it ran out.  With a hint, a waiting
// warp is parked by the hardware instead of spinning, so it takes no issue slots from the
// warps that do the work.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, uint32_t limit) {
    for (uint32_t it = 0;; ++it) {
        if (mbar_try_wait_hint(bar, parity, kWaitHintNs)) return true;
        if (it >= limit) return false;
    }
}

__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* tm, int x, int y, int z, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(
            smem_u32(dst)),
        "l"(tm), "r"(x), "r"(y), "r"(z), "r"(smem_u32(bar))
        : "memory");
}

// Shared -> global tensor copy of one box (the TMA engine clips rows and channels that fall
// outside the tensor), tracked by this thread's bulk async-group.  Coordinates are
// non-negative and x is a multiple of 16 bytes' worth of elements.
__device__ __forceinline__ void tma_store_3d(const CUtensorMap* tm, const void* src, int x, int y, int z) {
    asm volatile("cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%2, %3, %4}], [%1];" ::"l"(tm),
                 "r"(smem_u32(src)), "r"(x), "r"(y), "r"(z)
                 : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// waits until this thread's committed bulk stores have read their shared-memory source
__device__ __forceinline__ void bulk_wait_read() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
// waits until this thread's committed bulk stores are complete
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

struct PipeParams {
    int64_t groups_per_b, G, S, U;
    uint64_t* slot;     // [U][Cg][4] tagged words: a tile's aggregate, later its inclusive prefix
    WsHeader* hdr;
    int64_t drop_unit;  // test hook: this unit never publishes its records (-1: none)
};

// A published record is four 64-bit words, (a | tag), (b | tag), (anc | tag), (n | tag):
// the value's bits in the low half, the launch epoch and the record kind in the high
// half.  Aligned 64-bit accesses are single-copy atomic, so a reader that finds one tag
// in all four words holds one consistent record; nothing else has to be ordered, so
// neither side needs a fence or a separate flag.  The anchored exponent (anc, n) travels
// unrounded.  Each tile has one slot per channel: the tile's aggregate is published there
// first and later overwritten by its inclusive prefix (same thread, so every word takes
// the second value after the first); a reader that catches the overwrite half done sees
// mixed tags and reads again.  A tile's slots are stored word-major, [4][Cg] words, so a
// lane moves the same word of its two channels with one 16-byte access and a warp's
// access is contiguous.
__device__ __forceinline__ uint64_t tagged(uint32_t tag, float x) { return ((uint64_t)tag << 32) | __float_as_uint(x); }

template <int Cg>
__device__ __forceinline__ void publish_pair(uint64_t* tile_slots, int cl, const Rec& r0, const Rec& r1, uint32_t tag) {
    st_relaxed_v2u64(tile_slots + 0 * Cg + cl, tagged(tag, r0.a), tagged(tag, r1.a));
    st_relaxed_v2u64(tile_slots + 1 * Cg + cl, tagged(tag, r0.b), tagged(tag, r1.b));
    st_relaxed_v2u64(tile_slots + 2 * Cg + cl, tagged(tag, r0.anc), tagged(tag, r1.anc));
    st_relaxed_v2u64(tile_slots + 3 * Cg + cl, tagged(tag, r0.n), tagged(tag, r1.n));
}

struct RawPair {
    uint64_t w[4][2];  // word i of channel cl + c
};

template <int Cg>
__device__ __forceinline__ RawPair load_pair(const uint64_t* tile_slots, int cl) {
    RawPair r;
#pragma unroll
    for (int i = 0; i < 4; ++i) ld_relaxed_v2u64(tile_slots + i * Cg + cl, r.w[i][0], r.w[i][1]);
    return r;
}

// 2: both channels hold an inclusive prefix, 1: both an aggregate, 0: nothing usable yet
// (stale, half written, or the two channels caught at different kinds).
__device__ __forceinline__ int pair_kind(const RawPair& r, uint32_t tag_agg, uint32_t tag_incl, Rec& o0, Rec& o1) {
    const uint32_t t0 = (uint32_t)(r.w[0][0] >> 32);
    bool same = true;
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int c = 0; c < 2; ++c) same = same && (uint32_t)(r.w[i][c] >> 32) == t0;
    if (!same || (t0 != tag_agg && t0 != tag_incl)) return 0;
    o0 = Rec{__uint_as_float((uint32_t)r.w[0][0]), __uint_as_float((uint32_t)r.w[1][0]),
             __uint_as_float((uint32_t)r.w[2][0]), __uint_as_float((uint32_t)r.w[3][0])};
    o1 = Rec{__uint_as_float((uint32_t)r.w[0][1]), __uint_as_float((uint32_t)r.w[1][1]),
             __uint_as_float((uint32_t)r.w[2][1]), __uint_as_float((uint32_t)r.w[3][1])};
    return t0 == tag_incl ? 2 : 1;
}

constexpr size_t align128(size_t x) { return (x + 127) / 128 * 128; }

// Tensor maps for k and v viewed as [B][T][C] (3-D, channels innermost), box = one tile.
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }
    return fn;
}

bool make_tile_map(CUtensorMap* tm, const void* base, int64_t B, int64_t T, int64_t C, int io, int Cg, int Ts,
                   bool swizzle128 = false) {
    auto fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t es = io == 1 ? 2 : 4;
    cuuint64_t dims[3] = {(cuuint64_t)C, (cuuint64_t)T, (cuuint64_t)B};
    cuuint64_t strides[2] = {(cuuint64_t)C * es, (cuuint64_t)T * (cuuint64_t)C * es};
    cuuint32_t box[3] = {(cuuint32_t)Cg, (cuuint32_t)Ts, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    const CUresult r = fn(tm, io == 1 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3,
                          const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                          swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

}  // namespace
}  // namespace wkvb
