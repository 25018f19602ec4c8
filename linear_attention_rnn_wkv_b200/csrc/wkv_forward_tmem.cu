// Persistent, warp-specialised chunked WKV forward that parks each tile in tensor memory
// (the default chunked path when rows are 16-byte multiples).
//
// A unit is a tile of Ts = 8 * LC time steps by 64 channels; units are taken by an atomic
// ticket in time-segment-major order; each unit's chunk summaries fold into a tile
// aggregate, a decoupled look-back over earlier segments of the same channel group yields
// the carry, and each chunk is re-scanned from its carry to write y (the decay telescopes:
// RWKV transformer-math page, aicassindra.com, section "Why it collapses into a
// recurrence").
//
// Where a tile waits for its carry matters most.  A unit's k and v rows are needed
// twice, by the summaries and, after the look-back, by the re-scan; in between the tile
// sits idle for several microseconds.  Here the TMA lands a tile in a shared-memory stage,
// each summarising warp copies its chunk into its quadrant of the SM's tensor memory
// (tcgen05.st, 512 columns x 128 lanes x 32 bits) while it reads it, and the stage is
// free again as soon as the summaries are done.  The emitting warp of the same quadrant
// reads the chunk back (tcgen05.ld) once the carry is known.  Tensor memory holds 4
// (fp32, 16-step chunks) or 5 (bf16) units, so that many units per SM wait for carries at
// once while only 2-4 shared-memory stages are needed for the loads.
//
// Roles (20 warps):
//   warp 0          producer: a ticket once a stage and a unit slot are free, handed at once
//                   to the look-back warps (a ring of tickets), the unit's TMA box copies
//                   (`full`, one barrier per box of rows); also allocates and frees the
//                   tensor memory;
//   warps 1-3       look-back, round robin over units: from the ticket on, fold the
//                   predecessors' records into the carry while the unit's rows load; scan the
//                   chunk summaries once they are in (publishing the aggregate if the carry
//                   is still open), publish the inclusive prefix, hand the carry over (`carry`);
//   warps 4-11      summarise chunk c = warp - 4: summary record, rows into tensor memory
//                   (`chunks`; the stage is released, `dempty`);
//   warps 12-19     emit chunk c = warp - 12 (same quadrant as its summariser): rows back
//                   from tensor memory, re-scan in a fixed frame, y to HBM (`uempty`).
// All waits are bounded (error word on expiry, then the pipeline keeps moving), and the
// tensor memory is freed on every path before the CTA exits.  Deadlock freedom: a ticket
// is taken only when its stage and slot are free, roles handle a CTA's units in ticket
// order, every cross-CTA wait is on a smaller ticket, and the ticket ring's producer waits
// only for look-back warps that are working on older units.
#include <type_traits>

#include "wkv_device.cuh"
#include "wkv_internal.h"
#include "wkv_vec.cuh"
#include "wkv_pipe_common.cuh"

#ifdef WKV_TRACE
extern "C" cudaError_t wkv_trace_set_buffer(void* p) { return cudaMemcpyToSymbol(g_wkv_trace, &p, sizeof(p)); }
#endif

namespace wkvb {
namespace {

// ---------------------------------------------------------------------------
// Tensor memory (tcgen05) helpers.  A warp reaches the 32 lanes of its quadrant
// (warp index mod 4); the 32x32b shape gives thread i lane (quadrant * 32 + i) and N
// consecutive 32-bit columns.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
                 "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

template <int N>
struct TmemIO;

template <>
struct TmemIO<8> {
    static __device__ __forceinline__ void st(uint32_t taddr, const uint32_t (&r)[8]) {
        asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
                     : "memory");
    }
    static __device__ __forceinline__ void ld(uint32_t taddr, uint32_t (&r)[8]) {
        asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];" : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]) : "r"(taddr)
                     : "memory");
    }
    // completes this thread's earlier loads; the operands tie r's later uses to it
    static __device__ __forceinline__ void wait_ld(uint32_t (&r)[8]) {
        asm volatile("tcgen05.wait::ld.sync.aligned;" : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7])::"memory");
    }
    // completes this thread's earlier stores before r's registers are reused
    static __device__ __forceinline__ void wait_st(uint32_t (&r)[8]) {
        asm volatile("tcgen05.wait::st.sync.aligned;" : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7])::"memory");
    }
};

template <>
struct TmemIO<16> {
    static __device__ __forceinline__ void st(uint32_t taddr, const uint32_t (&r)[16]) {
        asm volatile("tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16};" ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
                     : "memory");
    }
    static __device__ __forceinline__ void ld(uint32_t taddr, uint32_t (&r)[16]) {
        asm volatile("tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];" : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]) : "r"(taddr)
                     : "memory");
    }
    // completes this thread's earlier loads; the operands tie r's later uses to it
    static __device__ __forceinline__ void wait_ld(uint32_t (&r)[16]) {
        asm volatile("tcgen05.wait::ld.sync.aligned;" : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]), "+r"(r[15])::"memory");
    }
    // completes this thread's earlier stores before r's registers are reused
    static __device__ __forceinline__ void wait_st(uint32_t (&r)[16]) {
        asm volatile("tcgen05.wait::st.sync.aligned;" : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]), "+r"(r[15])::"memory");
    }
};


// A lane's two channels of one row as 32-bit words: two fp32 words, or one bf16 pair.
template <typename TIO>
struct Pk;
template <>
struct Pk<float> {
    static constexpr int W = 2;
    static __device__ __forceinline__ void load(const float* p, uint32_t* w) {
        const float2 f = *reinterpret_cast<const float2*>(p);
        w[0] = __float_as_uint(f.x);
        w[1] = __float_as_uint(f.y);
    }
    static __device__ __forceinline__ float2 unpack(const uint32_t* w) {
        return make_float2(__uint_as_float(w[0]), __uint_as_float(w[1]));
    }
};
template <>
struct Pk<__nv_bfloat16> {
    static constexpr int W = 1;
    static __device__ __forceinline__ void load(const __nv_bfloat16* p, uint32_t* w) {
        w[0] = *reinterpret_cast<const uint32_t*>(p);
    }
    static __device__ __forceinline__ float2 unpack(const uint32_t* w) { return make_float2(bf_lo(w[0]), bf_hi(w[0])); }
};

// The receptance gate on one output pair (transformer-math page, section "Receptance: the
// gate on the way out"): y <- sigma(r) * y with sigma(r) = 1 / (1 + 2^(-r log2 e)).
__device__ __forceinline__ void gate_pair(float (&y)[2], const float (&r)[2]) {
#pragma unroll
    for (int c = 0; c < 2; ++c) y[c] *= rcp(1.f + ex2(-r[c] * kLog2e));
}

constexpr int kNWS = 8;   // chunks per tile (summarising warps, emitting warps)
constexpr int kNL = 3;    // look-back warps
constexpr int kCg = 64;   // channels per tile (a lane owns a pair)
// Beside the values, the summarising warps park in tensor memory each key's exponent as
// seen from the chunk's last row, x_i = k_i log2 e - (L - 1 - i) w log2 e, exactly as the
// summary used it, so the emitters need not recompute it.
constexpr int kThreads = (1 + kNL + 2 * kNWS) * 32;
// The producer hands each unit's ticket to the look-back warps through a ring of this many
// entries as soon as it has it, so a unit's look-back over its predecessors runs while its rows
// are still loading and being summarised.
constexpr int kRing = 16;

// What every role needs to know about a unit, worked out once by the producer (per
// shared-memory stage) and copied with the unit into its tensor-memory slot: the tile's
// geometry, and the channels' w and u (bulk-copied; entries past the last channel are
// left from an earlier unit and only feed lanes whose results are discarded).
struct UnitInfo {
    int64_t row0;  // element offset of (b, t0, c0) in [B][T][C]
    int64_t bc0;   // b * C + c0: the state index of the tile's first channel
    int32_t unit;  // ticket, or -1 past the end
    int32_t j;     // time segment
    int32_t g;     // channel group
    int32_t len;   // rows in the tile
    int32_t nch;   // channels in the tile (even)
    int32_t b, c0, t0;  // sequence, first channel, first row (tensor-map coordinates)
};
struct UnitBlock {
    UnitInfo info;
    float w[kCg];
    float u[kCg];
};
static_assert(sizeof(UnitBlock) % 16 == 0, "unit blocks are copied as 16-byte words");

template <typename TIO, int LC, int NS, int NT, bool GATE = false>
struct TmLayout {
    static constexpr int Cg = kCg;
    static constexpr int Ts = kNWS * LC;
    static constexpr size_t tile = sizeof(TIO) * Ts * Cg;  // one array (k or v)
    static constexpr size_t stage = align128(2 * tile);     // shared-memory stage: k tile, v tile
    // unit slot: chunk records [NWS][Cg], carries [Cg], chunk maxima [NWS][Cg], the unit's block
    static constexpr size_t recs_off = 0;
    static constexpr size_t carry_off = recs_off + sizeof(Rec) * kNWS * Cg;
    static constexpr size_t mx_off = carry_off + sizeof(Rec) * Cg;
    static constexpr size_t ub_off = mx_off + sizeof(float) * kNWS * Cg;
    static constexpr size_t slot = align128(ub_off + sizeof(UnitBlock));
    static constexpr int BR = kBoxRows < Ts ? kBoxRows : Ts;  // rows per TMA box
    static constexpr int NB = Ts / BR;
    static constexpr size_t slots_off = NS * stage;
    static constexpr size_t bars_off = slots_off + NT * slot;
    // per stage: NB full + 1 empty + 1 unit block; per slot: chunks, carry, empty
    static constexpr int NBARS = NS * (NB + 2) + NT * 3;
    static constexpr size_t misc_off = bars_off + NBARS * 8;  // end index, epoch, tensor memory base
    // the ticket ring: kRing tickets, then a full and an empty barrier per entry
    static constexpr size_t ring_off = align128(misc_off + 16);
    static constexpr size_t stage_ub_off = align128(ring_off + kRing * (4 + 16));  // the stages' unit blocks [NS]
    // gated forward: each emitting warp's chunk of r (TMA box of LC rows x Cg) and its barrier
    static constexpr size_t rbuf_bytes = align128(sizeof(TIO) * LC * Cg);
    static constexpr size_t rbuf_off = align128(stage_ub_off + NS * sizeof(UnitBlock));
    static constexpr size_t rbar_off = rbuf_off + (GATE ? kNWS * rbuf_bytes : 0);
    // each emitting warp's chunk of y, written row by row and stored by one TMA copy; the gated
    // forward writes each output over its own receptance in the r buffer
    static constexpr size_t ybuf_bytes = align128(sizeof(TIO) * LC * Cg);
    static constexpr size_t ybuf_off = GATE ? rbuf_off : align128(rbar_off);
    static constexpr size_t total = GATE ? rbar_off + kNWS * 8 : ybuf_off + kNWS * ybuf_bytes;
    // tensor memory: words per row per lane, columns per chunk array, per chunk, per unit and quadrant
    static constexpr int W = Pk<TIO>::W;
    // words per row of the first array: the key's exponent as an fp32 pair
    static constexpr int WK = 2;
    static constexpr int CPAK = LC * WK;  // columns of a chunk's first array (exponents)
    static constexpr int CPAV = LC * W;   // columns of a chunk's values
    static constexpr int CPC = CPAK + CPAV;
    static constexpr int CPU = (kNWS / 4) * CPC;
    static constexpr int SR = 8 / W;     // rows per tensor-memory slice (two slices of each array
    static constexpr int SWK = SR * WK;  // stay in registers while the next pair is read)
    static constexpr int SW = SR * W;
    static_assert(NT * CPU <= 512, "unit slots exceed the tensor memory");
    static_assert(LC % SR == 0, "slices must tile a chunk");
};

template <typename TIO, int LC, int NS, int NT, bool GATE>
__global__ void __launch_bounds__(kThreads, 1)
    tmem_kernel(ForwardArgs args, PipeParams pp, const __grid_constant__ CUtensorMap tmk,
                const __grid_constant__ CUtensorMap tmv, const __grid_constant__ CUtensorMap tmr,
                const __grid_constant__ CUtensorMap tmy) {
    using Lay = TmLayout<TIO, LC, NS, NT, GATE>;
    constexpr int V = 2;
    constexpr int Cg = Lay::Cg, Ts = Lay::Ts, NB = Lay::NB, BR = Lay::BR, W = Lay::W, SR = Lay::SR, SW = Lay::SW,
                  SWK = Lay::SWK;
    constexpr int W_L0 = 1, W_S0 = 1 + kNL, W_E0 = 1 + kNL + kNWS;
    // Where a unit takes its slot.  With few slots (fp32: 4) they are the scarce resource and
    // the summarisers take one only once the rows have landed; with more (bf16: 8) the
    // producer takes it with the ticket, so no ticketed unit waits for a slot and holds up its
    // successors in other CTAs.
    constexpr bool kLateSlot = NT <= 4;
    static_assert(W_S0 % 4 == 0 && W_E0 % 4 == 0, "a chunk's summariser and emitter must share a quadrant");
    extern __shared__ __align__(128) unsigned char smem[];
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Lay::bars_off);
    volatile int64_t* s_iend = reinterpret_cast<volatile int64_t*>(smem + Lay::misc_off);
    uint32_t* s_epoch = reinterpret_cast<uint32_t*>(smem + Lay::misc_off + 8);
    uint32_t* s_tmem = s_epoch + 1;
    auto dfull = [&](int s, int b) { return &bars[s * (NB + 2) + b]; };
    auto dempty = [&](int s) { return &bars[s * (NB + 2) + NB]; };
    auto dunit = [&](int s) { return &bars[s * (NB + 2) + NB + 1]; };  // the stage's unit block is written
    auto chunks_bar = [&](int t) { return &bars[NS * (NB + 2) + t * 3 + 0]; };
    auto carry_bar = [&](int t) { return &bars[NS * (NB + 2) + t * 3 + 1]; };
    auto uempty = [&](int t) { return &bars[NS * (NB + 2) + t * 3 + 2]; };
    auto ktile = [&](int s) { return reinterpret_cast<TIO*>(smem + s * Lay::stage); };
    auto vtile = [&](int s) { return reinterpret_cast<TIO*>(smem + s * Lay::stage + Lay::tile); };
    auto slotp = [&](int t) { return smem + Lay::slots_off + t * Lay::slot; };
    auto recs = [&](int t) { return reinterpret_cast<Rec*>(slotp(t) + Lay::recs_off); };
    auto carries = [&](int t) { return reinterpret_cast<Rec*>(slotp(t) + Lay::carry_off); };
    auto chunk_max = [&](int t) { return reinterpret_cast<float*>(slotp(t) + Lay::mx_off); };
    auto slot_ub = [&](int t) { return reinterpret_cast<UnitBlock*>(slotp(t) + Lay::ub_off); };
    auto stage_ub = [&](int s) { return reinterpret_cast<UnitBlock*>(smem + Lay::stage_ub_off) + s; };
    volatile uint32_t* ring_tk = reinterpret_cast<volatile uint32_t*>(smem + Lay::ring_off);
    auto ring_full = [&](int e) { return reinterpret_cast<uint64_t*>(smem + Lay::ring_off + kRing * 4) + 2 * e; };
    auto ring_empty = [&](int e) { return reinterpret_cast<uint64_t*>(smem + Lay::ring_off + kRing * 4) + 2 * e + 1; };

    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;
    const int64_t T = args.T, C = args.C, BC = args.B * args.C;
    const uint32_t lim = args.spin_limit;

    grid_dep_launch_dependents();
    if (warp == 0) {
        tmem_alloc(s_tmem, 512);
        tmem_relinquish();
    }
    uint32_t first_ticket = 0;
    if (tid == 0) {
        *s_iend = INT64_MAX;
        for (int s = 0; s < NS; ++s) {
            for (int b = 0; b < NB; ++b) mbar_init(dfull(s, b), 1);
            mbar_init(dempty(s), kNWS);
            mbar_init(dunit(s), 1);
        }
        if (GATE)
            for (int e = 0; e < kNWS; ++e) mbar_init(reinterpret_cast<uint64_t*>(smem + Lay::rbar_off) + e, 1);
        for (int t = 0; t < NT; ++t) {
            mbar_init(chunks_bar(t), kNWS);
            mbar_init(carry_bar(t), 1);
            mbar_init(uempty(t), kNWS);
        }
        for (int e = 0; e < kRing; ++e) {
            mbar_init(ring_full(e), 1);
            mbar_init(ring_empty(e), 1);
        }
        fence_mbar_init();
    }
    // global memory only from here: the stream's previous kernel may still be running
    grid_dep_wait();
    if (tid == 0) {
        WKV_TRACE_BLOCK(pp.U, 0);
        // the producer's first ticket and the launch's epoch (two round trips in flight at once)
        first_ticket = atomicAdd(&pp.hdr->ticket, 1u);
        *s_epoch = (*reinterpret_cast<volatile uint32_t*>(&pp.hdr->epoch) + 1u) & 0x3FFFFFFFu;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *s_tmem;
    const uint32_t epoch30 = *s_epoch;
    const uint32_t tag_agg = (epoch30 << 2) | 1u, tag_incl = (epoch30 << 2) | 2u;
    auto report = [&](uint32_t code) {
        atomicCAS(&pp.hdr->error, kDevOk, code);
        atomicCAS(args.dev_err, kDevOk, code);
    };
    // this warp's quadrant; the columns of chunk c's array a (0 k, 1 v) in unit slot t
    const uint32_t tq = tmem + ((uint32_t)((warp & 3) * 32) << 16);
    auto tcol = [&](int t, int c, int a) { return (uint32_t)(t * Lay::CPU + (c >> 2) * Lay::CPC + a * Lay::CPAK); };

    if (warp == 0) {
        // ------------------------------- producer -------------------------------
        // Lane 0 takes the tickets, works out each unit's geometry once for every other role
        // and issues the copies: the k and v boxes (`full`) and the tile's w and u (`unit`, with
        // the geometry).  The next ticket is requested as soon as the current unit's copies are
        // issued, so its round trip overlaps the wait for the next free stage (safe: the
        // block handles its units in ticket order whatever it has taken, and every
        // cross-block wait is on a smaller ticket).
        if (lane == 0) {
            uint32_t tk_next = first_ticket;
            for (int64_t i = 0;; ++i) {
                const int s = (int)(i % NS);
                if (i >= NS && !mbar_wait(dempty(s), (uint32_t)((i / NS - 1) & 1), lim)) report(kDevTimeoutCopy);
                const int t = (int)(i % NT);
                if (!kLateSlot && i >= NT && !mbar_wait(uempty(t), (uint32_t)((i / NT - 1) & 1), lim))
                    report(kDevTimeoutCopy);
                const uint32_t tk = tk_next;
                if (tk >= (uint32_t)pp.U + gridDim.x) report(kDevBadWorkspace);
                {
                    // the ticket to the unit's look-back warp, which starts on it at once (the
                    // sentinel past the end too)
                    const int e = (int)(i % kRing);
                    if (i >= kRing && !mbar_wait(ring_empty(e), (uint32_t)((i / kRing - 1) & 1), lim))
                        report(kDevTimeoutCopy);
                    ring_tk[e] = tk;
                    mbar_arrive(ring_full(e));
                }
                UnitBlock* ub = stage_ub(s);
                if (tk >= (uint32_t)pp.U) {
                    *s_iend = i;
                    ub->info.unit = -1;
                    for (int b = 0; b < NB; ++b) mbar_arrive(dfull(s, b));
                    mbar_arrive(dunit(s));
                    break;
                }
                // the unit's geometry: 32-bit divisions (tickets, G and groups per row are all
                // below 2^31: the host checks U)
                const uint32_t G32 = (uint32_t)pp.G, gpb32 = (uint32_t)pp.groups_per_b;
                const uint32_t j32 = tk / G32, g32 = tk - j32 * G32;
                const uint32_t b32 = g32 / gpb32, cg32 = g32 - b32 * gpb32;
                const int64_t unit = tk, j = j32, g = g32, b = b32;
                const int64_t c0 = (int64_t)cg32 * Cg, t0 = j * Ts;
                const int nch = (int)min64(Cg, C - c0);
                WKV_TRACE_EVENT(unit, 0);
#pragma unroll
                for (int bx = 0; bx < NB; ++bx) {
                    uint64_t* fb = dfull(s, bx);
                    mbar_arrive_expect_tx(fb, 2u * (uint32_t)(BR * Cg * sizeof(TIO)));
                    tma_load_3d(ktile(s) + bx * BR * Cg, &tmk, (int)c0, (int)(t0 + bx * BR), (int)b, fb);
                    tma_load_3d(vtile(s) + bx * BR * Cg, &tmv, (int)c0, (int)(t0 + bx * BR), (int)b, fb);
                }
                UnitInfo& q = ub->info;
                q.row0 = (b * T + t0) * C + c0;
                q.bc0 = b * C + c0;
                q.unit = (int32_t)unit;
                q.j = (int32_t)j;
                q.g = (int32_t)g;
                q.len = (int)min64(Ts, T - t0);
                q.nch = nch;
                q.b = (int32_t)b;
                q.c0 = (int32_t)c0;
                q.t0 = (int32_t)t0;
                // w and u of the tile's channels (nch is a multiple of 4: 16-byte rows); the
                // barrier's one arrival comes after the geometry above is written
                const uint32_t wbytes = (uint32_t)nch * (uint32_t)sizeof(float);
                mbar_arrive_expect_tx(dunit(s), 2u * wbytes);
                bulk_g2s(ub->w, args.w + c0, wbytes, dunit(s));
                bulk_g2s(ub->u, args.u + c0, wbytes, dunit(s));
                tk_next = atomicAdd(&pp.hdr->ticket, 1u);
            }
        }
        __syncwarp();
    } else if (warp < W_S0) {
        // ------------------------------- look-back ------------------------------
        // Warp l takes units l, l + kNL, ...  It learns a unit's ticket from the producer's
        // ring as soon as the producer has it and folds the records of the unit's predecessors
        // (a decoupled look-back) while the unit's rows are still loading and being
        // summarised.  Once the summaries are in it scans them (exclusive prefixes for the
        // emitters); if by then the carry is not yet known, it first publishes the tile's
        // aggregate for later segments.  Then the inclusive prefix is published and the carry
        // handed to the emitters.
        const int l = warp - W_L0;
        const uint32_t G32 = (uint32_t)pp.G, gpb32 = (uint32_t)pp.groups_per_b;
        for (int64_t i = l;; i += kNL) {
            const int t = (int)(i % NT);
            const uint32_t ph = (uint32_t)((i / NT) & 1);
            const int e = (int)(i % kRing);
            // the unit's ticket; polled without suspending, so a warp whose unit lies past the
            // end sees the producer's end index at once
            bool got = false, gone = false;
            for (uint32_t it = 0; it <= lim; ++it) {
                if (mbar_test_wait(ring_full(e), (uint32_t)((i / kRing) & 1))) {
                    got = true;
                    break;
                }
                if (*s_iend < i) {  // past the end (the sentinel unit itself still arrives)
                    gone = true;
                    break;
                }
                __nanosleep(it < 256 ? 64 : 512);  // the bound stays ~0.1 s of waiting
            }
            if (gone) break;
            if (!got) {  // gave up: release the unit's emitters and stop
                if (lane == 0) {
                    report(kDevTimeoutCarry);
                    mbar_arrive(carry_bar(t));
                }
                break;
            }
            const uint32_t tk = ring_tk[e];
            __syncwarp();
            if (lane == 0) mbar_arrive(ring_empty(e));
            if (tk >= (uint32_t)pp.U) {
                // the sentinel: its emitters learn of the end from a hand-over, once the
                // summarisers have passed it into the slot
                if (!mbar_wait(chunks_bar(t), ph, lim) && lane == 0) report(kDevTimeoutCarry);
                __syncwarp();
                if (lane == 0) mbar_arrive(carry_bar(t));
                break;
            }
            // the unit's geometry (as the producer works it out)
            const uint32_t j32 = tk / G32, g32 = tk - j32 * G32;
            const uint32_t b32 = g32 / gpb32, cg32 = g32 - b32 * gpb32;
            const int64_t unit = tk, j = j32, g = g32;
            const int64_t c0 = (int64_t)cg32 * Cg, t0 = j * Ts;
            const int nch = (int)min64(Cg, C - c0);
            const int len = (int)min64(Ts, T - t0);
            const int64_t bc0 = (int64_t)b32 * C + c0;
            if (lane == 0) WKV_TRACE_EVENT(unit, 3);
            const int cl = lane * V;
            const bool lane_active = cl < nch;  // (nch is even: a lane's two channels are both in or both out)
            float w2[V] = {0.f, 0.f};
            if (lane_active) {
                const float2 wp = *reinterpret_cast<const float2*>(args.w + c0 + cl);
                w2[0] = wp.x * kLog2e;
                w2[1] = wp.y * kLog2e;
            }
            // the chunk summaries scanned: exclusive prefixes for the emitters, the tile aggregate
            Rec agg[V] = {rec_identity(), rec_identity()};
            bool scanned = false;
            auto scan = [&]() {
                if (lane_active) {
                    Rec* rc = recs(t);
#pragma unroll
                    for (int w = 0; w < kNWS; ++w) {
                        const int lw = max(0, min(LC, len - w * LC));
#pragma unroll
                        for (int c = 0; c < V; ++c) {
                            const Rec r = rc[w * Cg + cl + c];
                            rc[w * Cg + cl + c] = agg[c];  // exclusive prefix of chunk w
                            if (lw > 0) agg[c] = rec_combine(agg[c], r, (float)lw, w2[c]);
                        }
                    }
                }
                scanned = true;
                if (lane == 0) WKV_TRACE_EVENT(unit, 4);
            };
            Rec run[V];
            if (j == 0) {
#pragma unroll
                for (int c = 0; c < V; ++c)
                    run[c] = (args.state_in && lane_active) ? rec_from_state(args.state_in, bc0 + cl + c, BC)
                                                            : rec_identity();
            } else {
#pragma unroll
                for (int c = 0; c < V; ++c) run[c] = rec_identity();
                // Each lane looks back for its channel pair: it folds aggregates from the newest
                // predecessor backwards and stops at the first inclusive prefix (the carry is then
                // known); a slot not yet published is read again after a short sleep.
                float span = 0.f;
                int64_t hi = j - 1;
                bool done = !lane_active;
                uint32_t nap = 64;
                bool all_done = false;
                for (uint32_t it = 0; it <= lim && !all_done; ++it) {
                    RawPair raw;
                    if (!done) raw = load_pair<Cg>(pp.slot + (hi * pp.G + g) * 4 * Cg, cl);
                    // while the read travels: the summaries are in before the carry, so the
                    // aggregate goes out now and later segments need not wait for this carry
                    if (!scanned && __any_sync(0xffffffffu, mbar_test_wait(chunks_bar(t), ph))) {
                        if (!mbar_wait(chunks_bar(t), ph, lim) && lane == 0) report(kDevTimeoutCarry);
                        scan();
                        if (lane_active && unit != pp.drop_unit)
                            publish_pair<Cg>(pp.slot + unit * 4 * Cg, cl, agg[0], agg[1], tag_agg);
                    }
                    if (!done) {
                        Rec r0, r1;
                        const int kind = pair_kind(raw, tag_agg, tag_incl, r0, r1);
                        if (kind != 0) {
                            run[0] = rec_combine(r0, run[0], span, w2[0]);
                            run[1] = rec_combine(r1, run[1], span, w2[1]);
                            if (kind == 2) {
                                done = true;
                            } else {
                                span += (float)Ts;
                                if (--hi < 0) done = true;
                            }
                            nap = 64;
                        } else {
                            __nanosleep(nap);
                            nap = nap < 256 ? nap * 2 : 256;
                        }
                    }
                    all_done = __all_sync(0xffffffffu, done);
                }
                if (!all_done) {
                    report(kDevTimeoutCarry);
                    pp.hdr->error_unit = (uint32_t)unit;
                }
            }
            if (lane == 0) WKV_TRACE_EVENT(unit, 5);
            if (!scanned) {
                if (!mbar_wait(chunks_bar(t), ph, lim) && lane == 0) report(kDevTimeoutCarry);
                scan();
            }
            // publish the inclusive prefix (over the aggregate, if that went out), then hand the
            // carry to the emitters
            Rec inc[V];
            if (lane_active) {
#pragma unroll
                for (int c = 0; c < V; ++c) inc[c] = rec_combine(run[c], agg[c], (float)len, w2[c]);
                if (unit != pp.drop_unit) publish_pair<Cg>(pp.slot + unit * 4 * Cg, cl, inc[0], inc[1], tag_incl);
                Rec* cs = carries(t);
#pragma unroll
                for (int c = 0; c < V; ++c) cs[cl + c] = run[c];
            }
            if (lane == 0) WKV_TRACE_EVENT(unit, 7);
            __syncwarp();
            if (lane == 0) {
                WKV_TRACE_EVENT(unit, 6);
                mbar_arrive(carry_bar(t));
            }
            if (lane_active && j == pp.S - 1 && args.state_out) {
#pragma unroll
                for (int c = 0; c < V; ++c) {
                    const int64_t bc = bc0 + cl + c;
                    args.state_out[bc] = inc[c].a;
                    args.state_out[BC + bc] = inc[c].b;
                    args.state_out[2 * BC + bc] = rec_p(inc[c], w2[c]) * kLn2;
                }
            }
        }
    } else if (warp < W_E0) {
        // ------------------------------- summarise ------------------------------
        // Warp c summarises chunk c of each tile and moves its rows into tensor memory.
        const int sw = warp - W_S0;
        for (int64_t i = 0;; ++i) {
            const int s = (int)(i % NS);
            const int t = (int)(i % NT);
            const uint32_t ph = (uint32_t)((i / NS) & 1);
            if (!mbar_wait(dunit(s), ph, lim) && lane == 0) report(kDevTimeoutCopy);
            if (!mbar_wait(dfull(s, sw * LC / BR), ph, lim) && lane == 0) report(kDevTimeoutCopy);
            const UnitBlock* sub = stage_ub(s);
            const UnitInfo q = sub->info;
            const int64_t unit = q.unit;
            // with late slots, the unit slot (tensor-memory columns and records) is taken only
            // now that the rows are here, so a slot is held from the summaries to the re-scan's end
            if (kLateSlot && i >= NT && !mbar_wait(uempty(t), (uint32_t)((i / NT - 1) & 1), lim) && lane == 0)
                report(kDevTimeoutCopy);
            if (sw == 0) {
                // the unit block goes with the unit into its slot (the stage is reused first)
                const uint4* src = reinterpret_cast<const uint4*>(sub);
                uint4* dst = reinterpret_cast<uint4*>(slot_ub(t));
                for (int x = lane; x < (int)(sizeof(UnitBlock) / 16); x += 32) dst[x] = src[x];
            }
            if (unit < 0) {
                __syncwarp();
                if (lane == 0) mbar_arrive(chunks_bar(t));
                break;
            }
            tc_fence_after();
            if (sw == 0 && lane == 0) WKV_TRACE_EVENT(unit, 1);
            const int cl = lane * V;
            const bool lane_active = cl < q.nch;
            const int r_begin = sw * LC;
            const int r_cnt = max(0, min(LC, q.len - r_begin));
            if (r_cnt > 0) {
                const float2 wraw = *reinterpret_cast<const float2*>(sub->w + cl);
                const float2 w2p = make_float2(wraw.x * kLog2e, wraw.y * kLog2e);
                const float2 L2 = make_float2(kLog2e, kLog2e);
                const TIO* kt = ktile(s);
                const TIO* vt = vtile(s);
                // The TMA fills rows past T and channels past C with zeros, so every row of the
                // chunk is read unconditionally; only the maxima and sums skip rows past the
                // end.  A full chunk (the usual case) runs with no per-row test at all, so the
                // rows' arithmetic interleaves freely.
                float M0 = kPEmpty, M1 = kPEmpty;
                float2 sa = make_float2(0.f, 0.f), sb = make_float2(0.f, 0.f);
                auto summarise = [&](auto full_c) {
                    constexpr bool FULL = decltype(full_c)::value;
                    float2 gx[LC];
                    // pass 1: k rows -> exponents at the chunk's last row, their maximum; rows to
                    // tensor memory
#pragma unroll
                    for (int h = 0; h < LC / SR; ++h) {
                        uint32_t kw[SWK];
#pragma unroll
                        for (int rr = 0; rr < SR; ++rr) {
                            const int r = h * SR + rr;
                            uint32_t raw[W];
                            Pk<TIO>::load(kt + (r_begin + r) * Cg + cl, raw);
                            const float back = FULL ? -(float)(LC - 1 - r) : -(float)(r_cnt - 1 - r);
                            gx[r] = __ffma2_rn(make_float2(back, back), w2p, __fmul2_rn(Pk<TIO>::unpack(raw), L2));
                            if (FULL || r < r_cnt) {
                                M0 = fmaxf(M0, gx[r].x);
                                M1 = fmaxf(M1, gx[r].y);
                            }
                            kw[rr * 2] = __float_as_uint(gx[r].x);
                            kw[rr * 2 + 1] = __float_as_uint(gx[r].y);
                        }
                        TmemIO<SWK>::st(tq + tcol(t, sw, 0) + h * SWK, kw);
                        TmemIO<SWK>::wait_st(kw);
                    }
                    // pass 2: v rows -> the chunk's sums relative to its maximum; rows to tensor
                    // memory
                    const float2 nM = make_float2(-M0, -M1);
#pragma unroll
                    for (int h = 0; h < LC / SR; ++h) {
                        uint32_t vw[SW];
#pragma unroll
                        for (int rr = 0; rr < SR; ++rr) {
                            const int r = h * SR + rr;
                            Pk<TIO>::load(vt + (r_begin + r) * Cg + cl, &vw[rr * W]);
                            if (FULL || r < r_cnt) {
                                const float2 x = __fadd2_rn(gx[r], nM);
                                const float2 e = make_float2(ex2(x.x), ex2(x.y));
                                sa = __ffma2_rn(e, Pk<TIO>::unpack(&vw[rr * W]), sa);
                                sb = __fadd2_rn(sb, e);
                            }
                        }
                        TmemIO<SW>::st(tq + tcol(t, sw, 1) + h * SW, vw);
                        TmemIO<SW>::wait_st(vw);
                    }
                };
                if (r_cnt == LC)
                    summarise(std::true_type{});
                else
                    summarise(std::false_type{});
                if (lane_active) {
                    Rec* rc = recs(t);
                    rc[sw * Cg + cl] = Rec{sa.x, sb.x, M0, 0.f};
                    rc[sw * Cg + cl + 1] = Rec{sa.y, sb.y, M1, 0.f};
                    *reinterpret_cast<float2*>(chunk_max(t) + sw * Cg + cl) = make_float2(M0, M1);
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(dempty(s));  // the stage's rows of this chunk are no longer needed
                mbar_arrive(chunks_bar(t));
            }
            if (sw == 0 && lane == 0) WKV_TRACE_EVENT(unit, 2);
        }
    } else {
        // --------------------------------- emit ---------------------------------
        const int ew = warp - W_E0;  // chunk index (the same quadrant as its summariser)
        // gated forward: this warp's chunk of r arrives by TMA in its own buffer
        uint64_t* rbar = reinterpret_cast<uint64_t*>(smem + Lay::rbar_off) + ew;
        const TIO* rbuf = reinterpret_cast<const TIO*>(smem + Lay::rbuf_off + ew * Lay::rbuf_bytes);
        // this warp's chunk of y: written row by row, then stored by one TMA tensor copy (rows past
        // T and channels past C are clipped by the copy)
        TIO* ybuf = reinterpret_cast<TIO*>(smem + Lay::ybuf_off + ew * Lay::ybuf_bytes);
        uint32_t rphase = 0;
        for (int64_t i = 0;; ++i) {
            const int t = (int)(i % NT);
            const uint32_t ph = (uint32_t)((i / NT) & 1);
            bool got = false, gone = false;
            bool r_pending = false;
            if (GATE) {
                // The unit is known once its summaries are in, well before its carry: fetch
                // this chunk's r rows now (one TMA box), so they are waiting when the rows are
                // emitted.  The buffer is free: the previous unit's rows were read before.
                for (uint32_t it = 0; it <= lim; ++it) {
                    if (mbar_try_wait_hint(chunks_bar(t), ph, kWaitHintNs)) {
                        got = true;
                        break;
                    }
                    if (*s_iend < i) {
                        gone = true;
                        break;
                    }
                }
                if (gone) break;
                const UnitInfo q0 = slot_ub(t)->info;
                if (got && q0.unit >= 0) {
                    if (q0.len > ew * LC) {
                        r_pending = true;
                        if (lane == 0) {
                            bulk_wait_read();  // the previous chunk's outputs have left the buffer
                            mbar_arrive_expect_tx(rbar, (uint32_t)(LC * Cg * sizeof(TIO)));
                            tma_load_3d(const_cast<TIO*>(rbuf), &tmr, (int)q0.c0, (int)(q0.t0 + ew * LC), (int)q0.b, rbar);
                        }
                    }
                }
                got = false;
            }
            for (uint32_t it = 0; it <= lim; ++it) {
                if (mbar_try_wait_hint(carry_bar(t), ph, kWaitHintNs)) {
                    got = true;
                    break;
                }
                // past the end (the producer has recorded the last unit)
                if (*s_iend < i) {
                    gone = true;
                    break;
                }
            }
            if (gone) break;
            if (!got && lane == 0) report(kDevTimeoutCarry);
            const UnitInfo q = slot_ub(t)->info;
            const int64_t unit = q.unit;
            if (unit < 0) break;
            tc_fence_after();
            if (ew == 0 && lane == 0) WKV_TRACE_EVENT(unit, 8);
            const int cl = lane * V;
            const bool lane_active = cl < q.nch;
            const int r_begin = ew * LC;
            const int r_cnt = max(0, min(LC, q.len - r_begin));
            if (r_cnt > 0) {
                // the first slice's rows are read while the carry is combined below
                uint32_t kw[SWK], vw[SW];
                TmemIO<SWK>::ld(tq + tcol(t, ew, 0), kw);
                TmemIO<SW>::ld(tq + tcol(t, ew, 1), vw);
                float w2[V], u2[V], a[V], bb[V], R[V], nn[V];
                bool lazy_ok = true;
                const float2 wv = *reinterpret_cast<const float2*>(slot_ub(t)->w + cl);
                const float2 uv = *reinterpret_cast<const float2*>(slot_ub(t)->u + cl);
                w2[0] = wv.x * kLog2e;
                w2[1] = wv.y * kLog2e;
                u2[0] = uv.x * kLog2e;
                u2[1] = uv.y * kLog2e;
#pragma unroll
                for (int c = 0; c < V; ++c) {
                    const Rec cr = lane_active
                                       ? rec_combine(carries(t)[cl + c], recs(t)[ew * Cg + cl + c], (float)r_begin, w2[c])
                                       : rec_identity();
                    a[c] = cr.a;
                    bb[c] = cr.b;
                    R[c] = cr.anc;
                    nn[c] = cr.n;
                    lazy_ok = lazy_ok && fabsf(u2[c]) <= kLazyLimit && w2[c] <= kLazyLimit;
                }
                TIO* yg = static_cast<TIO*>(args.y) + q.row0;
                TmemIO<SWK>::wait_ld(kw);
                TmemIO<SW>::wait_ld(vw);
                if (GATE && r_pending) {
                    if (!mbar_wait(rbar, rphase, lim) && lane == 0) report(kDevTimeoutCopy);
                    rphase ^= 1u;
                    r_pending = false;
                }
                // Fixed-frame re-scan.  Seen from the chunk's last row, each token's weight
                // e_i = 2^(k_i - (L-1-i) w - G) and the carried-in history K do not change from
                // row to row (everything decays at the same rate), so with running sums S of
                // K + e_i v_i and K + e_i over earlier rows and c = 2^(w - u)
                //   y_r = (S^a + e_r v_r / c) / (S^b + e_r / c):
                // no re-referencing and no selects, and only S is carried from row to row (the
                // first row of a sequence without history returns v itself, as the
                // recurrence does).  The frame G lies at most 100 above the larger of the
                // history and the first token (so no term that matters can be flushed), at
                // most 64 below the history (so K stays finite) and high enough that no later
                // token's term can overflow; a chunk whose range leaves no such G takes the
                // token-by-token step (one exp per token against a moving reference), and
                // parameters outside that step's range take the page's two-exp step.
                int mode = lazy_ok ? 1 : 2;
                float2 fSa = make_float2(0.f, 0.f), fSb = fSa, fnG = fSa, fic = fSa;
                if (lazy_ok) {
                    // the first token's exponent at the chunk's last row
                    const float h0v[2] = {__uint_as_float(kw[0]), __uint_as_float(kw[1])};
                    float fa[V], fb[V], fg[V], fi[V];
                    bool ok = true;
                    const float fc = (float)r_cnt;
#pragma unroll
                    for (int c = 0; c < V; ++c) {
                        const float M = lane_active ? chunk_max(t)[ew * Cg + cl + c] : 0.f;
                        const float hK = fmaf(-fc, w2[c], fmaf(-nn[c], w2[c], R[c]));  // history, at the last row
                        const float h0 = h0v[c];
                        const float bonus = u2[c] - w2[c];
                        const float dom = fminf(fmaxf(hK, h0), fmaxf(hK, h0 + bonus));
                        const float G = fmaxf(fminf(M, dom + 100.f), hK - 64.f);
                        ok = ok && (M - G + fmaxf(bonus, 0.f) <= 100.f);
                        const float sc = ex2(hK - G);
                        fa[c] = a[c] * sc;
                        fb[c] = bb[c] * sc;
                        fg[c] = -G;
                        fi[c] = ex2(bonus);
                    }
                    if (ok) {
                        mode = 0;
                        fSa = make_float2(fa[0], fa[1]);
                        fSb = make_float2(fb[0], fb[1]);
                        fnG = make_float2(fg[0], fg[1]);
                        fic = make_float2(fi[0], fi[1]);
                    }
                }
                if (__all_sync(0xffffffffu, mode == 0 || !lane_active)) {
                    // every lane in the fixed frame: one branch-free loop, the next slice's rows
                    // read from tensor memory while this slice is computed
                    // the previous chunk's copy must have read the buffer before it is overwritten
                    if (lane == 0) bulk_wait_read();
                    __syncwarp();
                    TIO* yrow = ybuf + cl;
                    {
#pragma unroll
                        for (int h = 0; h < LC / SR; ++h) {
                            uint32_t kn[SWK], vn[SW];
                            if (h + 1 < LC / SR) {
                                TmemIO<SWK>::ld(tq + tcol(t, ew, 0) + (h + 1) * SWK, kn);
                                TmemIO<SW>::ld(tq + tcol(t, ew, 1) + (h + 1) * SW, vn);
                            }

#pragma unroll
                            for (int rr = 0; rr < SR; ++rr) {
                                const int r = h * SR + rr;
                                const float2 vp = Pk<TIO>::unpack(&vw[rr * W]);
                                // the summary's own exponent, moved into the frame
                                const float2 x = __fadd2_rn(
                                    make_float2(__uint_as_float(kw[rr * 2]), __uint_as_float(kw[rr * 2 + 1])), fnG);
                                const float2 e = make_float2(ex2(x.x), ex2(x.y));
                                const float2 ec = __fmul2_rn(e, fic);
                                const float2 num = __ffma2_rn(ec, vp, fSa);
                                float2 den = __fadd2_rn(fSb, ec);
                                float2 er = make_float2(0.f, 0.f);
                                if (GATE) {
                                    // sigma(r) folded into the one reciprocal: y = num / (den (1 + 2^(-r log2 e)));
                                    // for r -> -inf the product overflows and y is the limit 0
                                    float rv[V];
                                    Vec<TIO, V>::load(rbuf + r * Cg + cl, rv);
                                    er = make_float2(ex2(-rv[0] * kLog2e), ex2(-rv[1] * kLog2e));
                                    den = __ffma2_rn(den, er, den);
                                }
                                const float2 yv = __fmul2_rn(num, make_float2(rcp(den.x), rcp(den.y)));
                                float yy[V] = {yv.x, yv.y};
                                if (r == 0) {
                                    // no history: the recurrence returns v itself (times the gate)
                                    if (fSb.x == 0.f) yy[0] = GATE ? vp.x * rcp(1.f + er.x) : vp.x;
                                    if (fSb.y == 0.f) yy[1] = GATE ? vp.y * rcp(1.f + er.y) : vp.y;
                                }
                                fSa = __ffma2_rn(e, vp, fSa);
                                fSb = __fadd2_rn(fSb, e);
                                Vec<TIO, V>::store(yrow + r * Cg, yy);
                            }
                            if (h + 1 < LC / SR) {
                                TmemIO<SWK>::wait_ld(kn);
                                TmemIO<SW>::wait_ld(vn);
#pragma unroll
                                for (int x = 0; x < SWK; ++x) kw[x] = kn[x];
#pragma unroll
                                for (int x = 0; x < SW; ++x) vw[x] = vn[x];
                            }
                        }
                    }
                    fence_proxy_async_smem();  // the rows written by the lanes, read by the TMA engine
                    __syncwarp();
                    if (lane == 0) {
                        tma_store_3d(&tmy, ybuf, q.c0, q.t0 + r_begin, q.b);
                        bulk_commit();
                    }
                } else {
                const float2 L2 = make_float2(kLog2e, kLog2e), nL2 = make_float2(-kLog2e, -kLog2e);
                const float2 w2p = make_float2(w2[0], w2[1]), u2p = make_float2(u2[0], u2[1]);
                const float2 nu2p = make_float2(-u2[0], -u2[1]);
                const float2 cwp = make_float2(ex2(w2[0] - u2[0]), ex2(w2[1] - u2[1]));
                const float2 one = make_float2(1.f, 1.f);
                float2 ap = make_float2(a[0], a[1]), bp = make_float2(bb[0], bb[1]);
                float2 nRp = make_float2(-R[0], -R[1]), np = make_float2(nn[0], nn[1]);
                float pp2[V] = {fmaf(-nn[0], w2[0], R[0]), fmaf(-nn[1], w2[1], R[1])};
#pragma unroll
                for (int h = 0; h < LC / SR; ++h) {
                    if (h > 0) {
                        TmemIO<SWK>::ld(tq + tcol(t, ew, 0) + h * SWK, kw);
                        TmemIO<SW>::ld(tq + tcol(t, ew, 1) + h * SW, vw);
                        TmemIO<SWK>::wait_ld(kw);
                        TmemIO<SW>::wait_ld(vw);
                    }
#pragma unroll
                    for (int rr = 0; rr < SR; ++rr) {
                        const int r = h * SR + rr;
                        if (!lane_active || r >= r_cnt) continue;
                        const int row = r_begin + r;
                        const float2 vp = Pk<TIO>::unpack(&vw[rr * W]);
                        float2 kp;
                        if (mode != 0) {
                            // the steps below need the keys themselves, which tensor memory does
                            // not hold: this rare lane reads them again
                            float kv2[V];
                            Vec<TIO, V>::load(static_cast<const TIO*>(args.k) + q.row0 + (int64_t)row * C + cl, kv2);
                            kp = make_float2(kv2[0], kv2[1]);
                        }
                        float yy[V];
                        if (mode == 0) {
                            const float2 x =
                                __fadd2_rn(make_float2(__uint_as_float(kw[rr * 2]), __uint_as_float(kw[rr * 2 + 1])), fnG);
                            const float2 e = make_float2(ex2(x.x), ex2(x.y));
                            const float2 ec = __fmul2_rn(e, fic);
                            const float2 num = __ffma2_rn(ec, vp, fSa);
                            const float2 den = __fadd2_rn(fSb, ec);
                            const float2 yv = __fmul2_rn(num, make_float2(rcp(den.x), rcp(den.y)));
                            yy[0] = (r == 0 && fSb.x == 0.f) ? vp.x : yv.x;
                            yy[1] = (r == 0 && fSb.y == 0.f) ? vp.y : yv.y;
                            fSa = __ffma2_rn(e, vp, fSa);
                            fSb = __fadd2_rn(fSb, e);
                        } else if (mode == 1) {
                            // lazy_step on the pair; the reference is kept negated (nR = -R)
                            const float2 uk = __ffma2_rn(kp, L2, u2p);
                            const float2 nuk = __ffma2_rn(kp, nL2, nu2p);
                            const float2 d = __ffma2_rn(np, w2p, __fadd2_rn(nRp, uk));  // (u + k) - (R - n w)
                            const bool c0 = d.x > 0.f, c1 = d.y > 0.f;
                            const float e0 = ex2(-fabsf(d.x)), e1 = ex2(-fabsf(d.y));
                            const float2 sa = make_float2(c0 ? e0 : 1.f, c1 ? e1 : 1.f);
                            const float2 sv = make_float2(c0 ? 1.f : e0, c1 ? 1.f : e1);
                            const float2 tt = __fmul2_rn(sa, ap);
                            const float2 num = __ffma2_rn(sv, vp, tt);
                            const float2 den = __ffma2_rn(sa, bp, sv);
                            const float2 yv = __fmul2_rn(num, make_float2(rcp(den.x), rcp(den.y)));
                            const float2 nw = __fmul2_rn(sv, cwp);
                            ap = __ffma2_rn(nw, vp, tt);
                            bp = __ffma2_rn(sa, bp, nw);
                            nRp = make_float2(c0 ? nuk.x : nRp.x, c1 ? nuk.y : nRp.y);
                            const float2 n1 = __fadd2_rn(np, one);
                            np = make_float2(c0 ? 1.f : n1.x, c1 ? 1.f : n1.y);
                            yy[0] = yv.x;
                            yy[1] = yv.y;
                        } else {
                            const float kv[2] = {kp.x, kp.y}, vv[2] = {vp.x, vp.y};
#pragma unroll
                            for (int c = 0; c < V; ++c) {
                                const float k2 = kv[c] * kLog2e;
                                yy[c] = wkv_output<false>(a[c], bb[c], pp2[c], u2[c] + k2, vv[c]);
                                wkv_fold<false>(a[c], bb[c], pp2[c], pp2[c] - w2[c], k2, vv[c], w2[c]);
                            }
                        }
                        if (GATE) {
                            float rv[V];
                            Vec<TIO, V>::load(rbuf + r * Cg + cl, rv);
                            gate_pair(yy, rv);
                        }
                        Vec<TIO, V>::store(yg + (int64_t)row * C + cl, yy);
                    }
                }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (ew == 0 && lane == 0) WKV_TRACE_EVENT(unit, 9);
            if (lane == 0) mbar_arrive(uempty(t));
        }
        // the chunks' stores must have read their rows before the block's shared memory goes
        // away (their writes complete on their own; the kernel's end orders them for later work)
        if (lane == 0) bulk_wait_read();
        __syncwarp();
    }
    if (lane == 0) WKV_TRACE_WARP(pp.U, warp);

    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
    if (tid == 0) {
        WKV_TRACE_BLOCK(pp.U, 1);
        __threadfence();
        const uint32_t finished = atomicAdd(&pp.hdr->done, 1u) + 1u;
        if (finished == gridDim.x) {
            atomicExch(&pp.hdr->ticket, 0u);
            atomicExch(&pp.hdr->done, 0u);
            atomicExch(&pp.hdr->epoch, epoch30);
        }
    }
}

// Unit slots: as many as the tensor memory holds (at most 8); stages: as many as the rest
// of the 227 KB of shared memory holds (at most 4).
template <typename TIO, int LC, bool GATE>
struct TmConfig {
    static constexpr int NT0 = 512 / TmLayout<TIO, LC, 1, 1>::CPU;
    static constexpr int NT = NT0 > 8 ? 8 : NT0;
    static constexpr size_t fixed = TmLayout<TIO, LC, 0, NT, GATE>::total;  // everything but the stages
    static constexpr size_t per_stage =
        TmLayout<TIO, LC, 1, NT>::stage + (TmLayout<TIO, LC, 1, NT>::NB + 2) * 8 + sizeof(UnitBlock);
    static constexpr int NS0 = (int)((232448 - fixed) / per_stage);
    static constexpr int NS = NS0 > 4 ? 4 : NS0;
};

template <typename TIO, int LC, bool GATE>
cudaError_t launch_tmem_g(const ForwardArgs& a, const ChunkGeom& g, const PipeParams& pp, cudaStream_t s) {
    constexpr int NT = TmConfig<TIO, LC, GATE>::NT;
    constexpr int NS = TmConfig<TIO, LC, GATE>::NS;
    static_assert(NS >= 2, "fewer than two shared-memory stages");
    // a look-back warp waits on unit i's slot only after finishing unit i - kNL, so the
    // slot's previous phase (unit i - NT) is complete whenever NT >= kNL
    static_assert(NT >= kNL, "fewer unit slots than look-back warps");
    using Lay = TmLayout<TIO, LC, NS, NT, GATE>;
    static_assert(Lay::total <= 232448, "shared memory layout over the per-CTA limit");
    static_assert(Lay::Ts % Lay::BR == 0, "tile rows must be a multiple of the box rows");
    static_assert(LC <= Lay::BR && Lay::BR % LC == 0, "a chunk must lie inside one box");
    auto kern = tmem_kernel<TIO, LC, NS, NT, GATE>;
    CUtensorMap tmk, tmv, tmr, tmy;
    if (!make_tile_map(&tmk, a.k, a.B, a.T, a.C, a.io, Lay::Cg, Lay::BR) ||
        !make_tile_map(&tmv, a.v, a.B, a.T, a.C, a.io, Lay::Cg, Lay::BR) ||
        !make_tile_map(&tmy, a.y, a.B, a.T, a.C, a.io, Lay::Cg, LC))
        return cudaErrorInvalidValue;
    if (GATE ? !make_tile_map(&tmr, a.r, a.B, a.T, a.C, a.io, Lay::Cg, LC) : false) return cudaErrorInvalidValue;
    if (!GATE) tmr = tmk;  // unused
    static uint64_t attr_done = 0;  // per device; set once so captured launches issue no attribute call
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    static int sms[64] = {0};
    if (dev >= 64 || !(attr_done & (1ull << dev))) {
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)Lay::total);
        if (e != cudaSuccess) return e;
        int n = 0;
        e = cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
        if (e != cudaSuccess) return e;
        if (dev < 64) {
            sms[dev] = n;
            attr_done |= 1ull << dev;
        }
    }
    const int64_t nsm = dev < 64 ? sms[dev] : 148;
    const int64_t grid = g.U < nsm ? g.U : nsm;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = Lay::total;
    cfg.stream = s;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[0].val.programmaticStreamSerializationAllowed = kProgrammaticLaunch ? 1 : 0;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, a, pp, tmk, tmv, tmr, tmy);
}

template <typename TIO, int LC>
cudaError_t launch_tmem_t(const ForwardArgs& a, const ChunkGeom& g, const PipeParams& pp, cudaStream_t s) {
    return a.r ? launch_tmem_g<TIO, LC, true>(a, g, pp, s) : launch_tmem_g<TIO, LC, false>(a, g, pp, s);
}

}  // namespace

cudaError_t launch_forward_tmem(const ForwardArgs& a, const ChunkGeom& g, void* ws, int64_t drop_unit,
                                cudaStream_t s) {
    unsigned char* base = static_cast<unsigned char*>(ws);
    PipeParams pp;
    pp.groups_per_b = g.groups_per_b;
    pp.G = g.G;
    pp.S = g.S;
    pp.U = g.U;
    pp.hdr = reinterpret_cast<WsHeader*>(base);
    pp.slot = reinterpret_cast<uint64_t*>(base + kWsHeaderBytes);
    pp.drop_unit = drop_unit;
    if (g.V != 2 || g.NW != kNWS) return cudaErrorInvalidValue;
    if (a.io == 1) {
        if (g.LC == 8) return launch_tmem_t<__nv_bfloat16, 8>(a, g, pp, s);
        if (g.LC == 16) return launch_tmem_t<__nv_bfloat16, 16>(a, g, pp, s);
        return cudaErrorInvalidValue;
    }
    if (g.LC == 8) return launch_tmem_t<float, 8>(a, g, pp, s);
    if (g.LC == 16) return launch_tmem_t<float, 16>(a, g, pp, s);
    return cudaErrorInvalidValue;
}

}  // namespace wkvb
