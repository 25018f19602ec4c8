// Chunked, time-parallel WKV forward in a single pass (12 B/element for fp32 I/O).
//
// The decay factor telescopes (RWKV transformer-math page, aicassindra.com, section
// "Why it collapses into a recurrence"), so the state after a span of tokens is an
// associative fold: a segment is summarised by (a, b, p) relative to its own running
// maximum, and two adjacent segments combine by decaying the earlier one over the
// later one's length and re-referencing to the larger exponent.  The summaries use
// the anchored record of wkv_device.cuh (p = anc - n w) so that exponents carry one
// rounding, not one per step.
//
// Work decomposition.  A unit is a tile of Ts = NW * LC time steps by Cg = 32 * V
// channels of one sequence.  Units are handed out by an atomic ticket in
// segment-major order (all channel groups of time segment j before segment j + 1),
// so a unit's predecessors in time always hold smaller tickets and are already
// running or finished: the look-back below cannot deadlock, whatever the CTA
// residency.  Inside a CTA, warp w owns chunk w (LC steps) and lane l owns V
// adjacent channels.
//
//   1. the tile of k and v lands in shared memory (TMA bulk copies, one per row,
//      completion on an mbarrier; per-element loads when rows are not 16-byte
//      multiples);
//   2. each warp summarises its chunk from the empty state: the exact maximum
//      exponent max_i (k_i - (LC-1-i) w) first, then one exp per element;
//   3. one thread per channel scans the NW chunk summaries (exclusive prefixes stay
//      in shared memory; the inclusive one is the tile aggregate);
//   4. warp 0 publishes the aggregate, then looks back over the predecessor tiles of
//      the same channel group (decoupled look-back, Merrill & Garland 2016): it
//      combines aggregates until it meets an inclusive prefix, and publishes its own
//      inclusive prefix.  Every wait is bounded; on expiry the error word is set and
//      the missing carry is taken as empty, so no successor can hang;
//   5. every warp combines the tile carry with its chunk's exclusive prefix and
//      re-scans its chunk from shared memory, writing y.
// The last time segment's inclusive prefix is the final state (state_out).
#include "wkv_device.cuh"
#include "wkv_internal.h"

namespace wkvb {
namespace {

// ---- vector I/O of V adjacent channels ----
template <typename TIO, int V>
struct Vec;

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

template <>
struct Vec<float, 1> {
    static __device__ __forceinline__ void load(const float* p, float (&o)[1]) { o[0] = *p; }
    static __device__ __forceinline__ void store(float* p, const float (&o)[1]) { *p = o[0]; }
};

template <>
struct Vec<__nv_bfloat16, 4> {
    static __device__ __forceinline__ void load(const __nv_bfloat16* p, float (&o)[4]) {
        uint2 t = *reinterpret_cast<const uint2*>(p);
        o[0] = __uint_as_float(t.x << 16);
        o[1] = __uint_as_float(t.x & 0xFFFF0000u);
        o[2] = __uint_as_float(t.y << 16);
        o[3] = __uint_as_float(t.y & 0xFFFF0000u);
    }
    static __device__ __forceinline__ void store(__nv_bfloat16* p, const float (&o)[4]) {
        __nv_bfloat162 lo = __floats2bfloat162_rn(o[0], o[1]);
        __nv_bfloat162 hi = __floats2bfloat162_rn(o[2], o[3]);
        uint2 t;
        t.x = *reinterpret_cast<uint32_t*>(&lo);
        t.y = *reinterpret_cast<uint32_t*>(&hi);
        *reinterpret_cast<uint2*>(p) = t;
    }
};

template <>
struct Vec<__nv_bfloat16, 1> {
    static __device__ __forceinline__ void load(const __nv_bfloat16* p, float (&o)[1]) {
        o[0] = __bfloat162float(*p);
    }
    static __device__ __forceinline__ void store(__nv_bfloat16* p, const float (&o)[1]) {
        *p = __float2bfloat16_rn(o[0]);
    }
};

struct ChunkParams {
    int64_t groups_per_b, G, S;
    uint32_t* flags;  // [U]
    float4* agg;      // [U][Cg]
    float4* incl;     // [U][Cg]
    WsHeader* hdr;
    int64_t drop_unit;
};

__device__ __forceinline__ float4 rec_pack(const Rec& r) { return make_float4(r.a, r.b, r.anc, r.n); }
__device__ __forceinline__ Rec rec_unpack(const float4& f) { return Rec{f.x, f.y, f.z, f.w}; }

// Natural-units state (a, b, p) -> anchored base-2 record.
__device__ __forceinline__ Rec rec_from_state(const float* st, int64_t bc, int64_t BC) {
    return Rec{st[bc], st[BC + bc], st[2 * BC + bc] * kLog2e, 0.f};
}

template <typename TIO, int V, int NW, int LC, bool BULK>
__global__ void __launch_bounds__(NW * 32) chunked_kernel(ForwardArgs args, ChunkParams cp) {
    constexpr int NT = NW * 32;
    constexpr int Cg = 32 * V;
    constexpr int Ts = NW * LC;
    extern __shared__ __align__(128) unsigned char smem[];
    TIO* ks = reinterpret_cast<TIO*>(smem);
    TIO* vs = ks + Ts * Cg;
    Rec* recs = reinterpret_cast<Rec*>(smem + sizeof(TIO) * 2 * Ts * Cg);  // [NW][Cg]
    Rec* carry_s = recs + NW * Cg;                                          // [Cg]
    Rec* aggs = carry_s + Cg;                                               // [Cg]
    uint64_t* bar = reinterpret_cast<uint64_t*>(aggs + Cg);
    int64_t* s_ticket = reinterpret_cast<int64_t*>(bar + 1);
    uint32_t* s_epoch = reinterpret_cast<uint32_t*>(s_ticket + 1);

    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;
    const int64_t T = args.T, C = args.C, BC = args.B * args.C;

    if (tid == 0) {
        uint32_t ticket = atomicAdd(&cp.hdr->ticket, 1u);
        if (ticket >= gridDim.x) {
            // the workspace was not zero-filled (or is in use by an overlapping launch):
            // stay in bounds, report it; the waits below are bounded
            atomicCAS(&cp.hdr->error, kDevOk, kDevBadWorkspace);
            ticket %= gridDim.x;
        }
        *s_ticket = (int64_t)ticket;
        // This launch's epoch: the previous launch's last CTA advanced the header
        // before this launch began, and it is advanced again only after every CTA
        // of this launch has finished, so all CTAs read the same value.
        *s_epoch = (*reinterpret_cast<volatile uint32_t*>(&cp.hdr->epoch) + 1u) & 0x3FFFFFFFu;
        if (BULK) {
            mbar_init(bar, 1);
            fence_mbar_init();
        }
    }
    __syncthreads();
    const int64_t unit = *s_ticket;
    const uint32_t epoch30 = *s_epoch;
    const int64_t j = unit / cp.G;  // time segment
    const int64_t g = unit % cp.G;  // channel group
    const int64_t b = g / cp.groups_per_b;
    const int64_t c0 = (g % cp.groups_per_b) * Cg;
    const int64_t t0 = j * Ts;
    const int len = (int)min64(Ts, T - t0);
    const int nch = (int)min64(Cg, C - c0);
    const TIO* kg = static_cast<const TIO*>(args.k) + (b * T + t0) * C + c0;
    const TIO* vg = static_cast<const TIO*>(args.v) + (b * T + t0) * C + c0;
    TIO* yg = static_cast<TIO*>(args.y) + (b * T + t0) * C + c0;

    // ---- 1. tile -> shared memory ----
    bool copy_failed = false;
    if (BULK) {
        const uint32_t row_bytes = (uint32_t)nch * sizeof(TIO);
        if (warp == 0) {
            if (lane == 0) mbar_arrive_expect_tx(bar, 2u * (uint32_t)len * row_bytes);
            __syncwarp();
            for (int r = lane; r < len; r += 32) {
                bulk_g2s(ks + r * Cg, kg + (int64_t)r * C, row_bytes, bar);
                bulk_g2s(vs + r * Cg, vg + (int64_t)r * C, row_bytes, bar);
            }
        }
        bool timed_out = false;
        for (uint32_t it = 0; !mbar_try_wait(bar, 0); ++it) {
            if (it >= args.spin_limit) {
                timed_out = true;
                break;
            }
            __nanosleep(64);
        }
        copy_failed = __syncthreads_or(timed_out);
        if (copy_failed && tid == 0) {
            atomicCAS(&cp.hdr->error, kDevOk, kDevTimeoutCopy);
            cp.hdr->error_unit = (uint32_t)unit;
        }
    } else {
        for (int idx = tid; idx < len * Cg; idx += NT) {
            const int r = idx / Cg, cc = idx % Cg;
            if (cc < nch) {
                ks[idx] = kg[(int64_t)r * C + cc];
                vs[idx] = vg[(int64_t)r * C + cc];
            }
        }
        __syncthreads();
    }

    // per-thread channels and parameters (base-2 units)
    const int cl = lane * V;  // first channel of this lane within the tile
    const bool lane_active = cl < nch;
    float w2[V], u2[V];
#pragma unroll
    for (int q = 0; q < V; ++q) {
        const int64_t c = c0 + cl + q;
        const bool ok = lane_active && (cl + q < nch);
        w2[q] = ok ? args.w[c] * kLog2e : 0.f;
        u2[q] = ok ? args.u[c] * kLog2e : 0.f;
    }

    // ---- 2. chunk summaries from the empty state ----
    const int r_begin = warp * LC;
    const int r_cnt = max(0, min(LC, len - r_begin));
    if (lane_active) {
        float M[V], anc[V], nn[V];
#pragma unroll
        for (int q = 0; q < V; ++q) {
            M[q] = kPEmpty;
            anc[q] = kPEmpty;
            nn[q] = 0.f;
        }
        for (int i = 0; i < r_cnt; ++i) {
            float kk[V];
            Vec<TIO, V>::load(ks + (r_begin + i) * Cg + cl, kk);
            const float back = (float)(r_cnt - 1 - i);
#pragma unroll
            for (int q = 0; q < V; ++q) {
                const float k2 = kk[q] * kLog2e;
                const float gq = fmaf(-back, w2[q], k2);
                if (gq > M[q]) {
                    M[q] = gq;
                    anc[q] = k2;
                    nn[q] = back;
                }
            }
        }
        float sa[V], sb[V];
#pragma unroll
        for (int q = 0; q < V; ++q) sa[q] = sb[q] = 0.f;
        for (int i = 0; i < r_cnt; ++i) {
            float kk[V], vv[V];
            Vec<TIO, V>::load(ks + (r_begin + i) * Cg + cl, kk);
            Vec<TIO, V>::load(vs + (r_begin + i) * Cg + cl, vv);
            const float back = (float)(r_cnt - 1 - i);
#pragma unroll
            for (int q = 0; q < V; ++q) {
                const float e = ex2(fmaf(-back, w2[q], kk[q] * kLog2e) - M[q]);
                sa[q] = fmaf(e, vv[q], sa[q]);
                sb[q] += e;
            }
        }
#pragma unroll
        for (int q = 0; q < V; ++q) recs[warp * Cg + cl + q] = Rec{sa[q], sb[q], anc[q], nn[q]};
    }
    __syncthreads();

    // ---- 3. scan of the chunk summaries (one thread per channel) ----
    for (int cc = tid; cc < nch; cc += NT) {
        const float w2c = args.w[c0 + cc] * kLog2e;
        Rec run = rec_identity();
        for (int w = 0; w < NW; ++w) {
            const int lw = max(0, min(LC, len - w * LC));
            Rec r = recs[w * Cg + cc];
            recs[w * Cg + cc] = run;  // exclusive prefix of chunk w
            if (lw > 0) run = rec_combine(run, r, (float)lw, w2c);
        }
        aggs[cc] = run;
    }
    __syncthreads();

    // ---- 4. decoupled look-back across time segments (warp 0) ----
    if (warp == 0) {
        const int64_t uidx = unit;
        const bool publish = uidx != cp.drop_unit;
        Rec carry[V], inc[V];
        if (j == 0) {
#pragma unroll
            for (int q = 0; q < V; ++q) {
                const int cc = cl + q;
                carry[q] = (args.state_in && cc < nch) ? rec_from_state(args.state_in, b * C + c0 + cc, BC)
                                                       : rec_identity();
            }
        } else {
            // publish the aggregate
            if (lane_active) {
#pragma unroll
                for (int q = 0; q < V; ++q)
                    if (cl + q < nch) cp.agg[uidx * Cg + cl + q] = rec_pack(aggs[cl + q]);
            }
            __threadfence();
            __syncwarp();
            if (lane == 0 && publish) st_release_u32(&cp.flags[uidx], (epoch30 << 2) | 1u);
            // look back
            Rec run[V];
#pragma unroll
            for (int q = 0; q < V; ++q) run[q] = rec_identity();
            float span = 0.f;
            int64_t pred = j - 1;
            while (true) {
                const int64_t pu = pred * cp.G + g;
                // lane 0 polls; then every lane acquires the flag itself (at least the state lane 0
                // saw: flags only move AGG -> INCL within a launch) before reading the record
                uint32_t f = 0;
                bool ready = false;
                if (lane == 0) {
                    for (uint32_t it = 0; it <= args.spin_limit; ++it) {
                        f = ld_acquire_u32(&cp.flags[pu]);
                        if ((f >> 2) == epoch30 && (f & 3u) != 0u) {
                            ready = true;
                            break;
                        }
                        __nanosleep(64);
                    }
                }
                ready = __shfl_sync(0xffffffffu, ready, 0);
                if (!ready) {
                    // the predecessor never published: record it, take its carry as empty
                    if (lane == 0) {
                        atomicCAS(&cp.hdr->error, kDevOk, kDevTimeoutCarry);
                        cp.hdr->error_unit = (uint32_t)uidx;
                    }
                    break;
                }
                f = __shfl_sync(0xffffffffu, f, 0);
                if (lane != 0) {
                    for (uint32_t it = 0; it <= args.spin_limit; ++it) {
                        const uint32_t mine = ld_acquire_u32(&cp.flags[pu]);
                        if ((mine >> 2) == epoch30 && (mine & 3u) >= (f & 3u)) break;
                        __nanosleep(64);
                    }
                }
                const bool inclusive = (f & 3u) == 2u;
                const float4* src = inclusive ? cp.incl : cp.agg;
                if (lane_active) {
#pragma unroll
                    for (int q = 0; q < V; ++q) {
                        if (cl + q < nch) {
                            Rec r = rec_unpack(ld_relaxed_f4(src + pu * Cg + cl + q));
                            run[q] = rec_combine(r, run[q], span, w2[q]);
                        }
                    }
                }
                if (inclusive || pred == 0) break;
                span += (float)Ts;
                --pred;
            }
#pragma unroll
            for (int q = 0; q < V; ++q) carry[q] = run[q];
        }
        // inclusive prefix of this unit
#pragma unroll
        for (int q = 0; q < V; ++q)
            inc[q] = (cl + q < nch) ? rec_combine(carry[q], aggs[cl + q], (float)len, w2[q]) : rec_identity();
        if (lane_active) {
#pragma unroll
            for (int q = 0; q < V; ++q)
                if (cl + q < nch) cp.incl[uidx * Cg + cl + q] = rec_pack(inc[q]);
        }
        __threadfence();
        __syncwarp();
        if (lane == 0 && publish) st_release_u32(&cp.flags[uidx], (epoch30 << 2) | 2u);
        if (lane_active) {
#pragma unroll
            for (int q = 0; q < V; ++q) carry_s[cl + q] = carry[q];
            if (j == cp.S - 1 && args.state_out) {
#pragma unroll
                for (int q = 0; q < V; ++q) {
                    if (cl + q < nch) {
                        const int64_t bc = b * C + c0 + cl + q;
                        args.state_out[bc] = inc[q].a;
                        args.state_out[BC + bc] = inc[q].b;
                        args.state_out[2 * BC + bc] = rec_p(inc[q], w2[q]) * kLn2;
                    }
                }
            }
        }
    }
    __syncthreads();

    // ---- 5. re-scan each chunk from its carry, emitting y ----
    if (lane_active && r_cnt > 0) {
        float a[V], bb[V], p[V];
#pragma unroll
        for (int q = 0; q < V; ++q) {
            const Rec cr = rec_combine(carry_s[cl + q], recs[warp * Cg + cl + q], (float)r_begin, w2[q]);
            a[q] = cr.a;
            bb[q] = cr.b;
            p[q] = rec_p(cr, w2[q]);
        }
        for (int i = 0; i < r_cnt; ++i) {
            const int r = r_begin + i;
            float kk[V], vv[V], yy[V];
            Vec<TIO, V>::load(ks + r * Cg + cl, kk);
            Vec<TIO, V>::load(vs + r * Cg + cl, vv);
#pragma unroll
            for (int q = 0; q < V; ++q) {
                const float k2 = kk[q] * kLog2e;
                yy[q] = wkv_output<false>(a[q], bb[q], p[q], u2[q] + k2, vv[q]);
                wkv_fold<false>(a[q], bb[q], p[q], p[q] - w2[q], k2, vv[q], w2[q]);
            }
            if (V == 1 || cl + V <= nch) {
                Vec<TIO, V>::store(yg + (int64_t)r * C + cl, yy);
            } else {
#pragma unroll
                for (int q = 0; q < V; ++q)
                    if (cl + q < nch) io<TIO>::store(yg + (int64_t)r * C + cl + q, yy[q]);
            }
        }
    }

    // ---- bookkeeping: let in-flight copies land, reset the ticket after the last CTA ----
    if (BULK && copy_failed) {
        for (uint32_t it = 0; it < args.spin_limit && !mbar_try_wait(bar, 0); ++it) __nanosleep(64);
    }
    __syncthreads();
    if (tid == 0) {
        __threadfence();
        const uint32_t finished = atomicAdd(&cp.hdr->done, 1u) + 1u;
        if (finished == gridDim.x) {
            atomicExch(&cp.hdr->ticket, 0u);
            atomicExch(&cp.hdr->done, 0u);
            atomicExch(&cp.hdr->epoch, epoch30);
        }
    }
}

template <typename TIO, int V, int NW, int LC, bool BULK>
cudaError_t launch_t(const ForwardArgs& a, const ChunkGeom& g, const ChunkParams& cp, cudaStream_t s) {
    constexpr int Cg = 32 * V, Ts = NW * LC;
    const size_t smem = sizeof(TIO) * 2 * Ts * Cg + sizeof(Rec) * (NW + 2) * Cg + 16 + 16;
    auto kern = chunked_kernel<TIO, V, NW, LC, BULK>;
    static uint64_t attr_done = 0;  // per device; set once so a launch inside stream capture issues no attribute call
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev >= 64 || !(attr_done & (1ull << dev))) {
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        if (dev < 64) attr_done |= 1ull << dev;
    }
    kern<<<(unsigned)g.U, NW * 32, smem, s>>>(a, cp);
    return cudaGetLastError();
}

template <typename TIO, int V, bool BULK>
cudaError_t launch_lc(const ForwardArgs& a, const ChunkGeom& g, const ChunkParams& cp, cudaStream_t s) {
    constexpr int NW = 4;
    switch (g.LC) {
        case 4: return launch_t<TIO, V, NW, 4, BULK>(a, g, cp, s);
        case 8: return launch_t<TIO, V, NW, 8, BULK>(a, g, cp, s);
        case 16: return launch_t<TIO, V, NW, 16, BULK>(a, g, cp, s);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace

bool chunk_geometry(int64_t B, int64_t T, int64_t C, int io, int chunk, ChunkGeom* g) {
    const int esize = io == 1 ? 2 : 4;
    const bool bulk = ((C * esize) % 16) == 0;
    const int LC = chunk == 0 ? 8 : chunk;
    if (LC != 4 && LC != 8 && LC != 16) return false;
    g->V = bulk ? 4 : 1;
    g->NW = 4;
    g->LC = LC;
    g->bulk = bulk;
    g->Cg = 32 * g->V;
    g->Ts = (int64_t)g->NW * LC;
    g->groups_per_b = (C + g->Cg - 1) / g->Cg;
    g->G = B * g->groups_per_b;
    g->S = (T + g->Ts - 1) / g->Ts;
    g->U = g->G * g->S;
    const size_t flags = ((size_t)g->U * 4 + 15) / 16 * 16;
    g->ws_bytes = kWsHeaderBytes + flags + 2 * (size_t)g->U * (size_t)g->Cg * 16;
    return true;
}

cudaError_t launch_forward_chunked(const ForwardArgs& a, const ChunkGeom& g, void* ws, int64_t drop_unit,
                                   cudaStream_t s) {
    unsigned char* base = static_cast<unsigned char*>(ws);
    const size_t flags_bytes = ((size_t)g.U * 4 + 15) / 16 * 16;
    ChunkParams cp;
    cp.groups_per_b = g.groups_per_b;
    cp.G = g.G;
    cp.S = g.S;
    cp.hdr = reinterpret_cast<WsHeader*>(base);
    cp.flags = reinterpret_cast<uint32_t*>(base + kWsHeaderBytes);
    cp.agg = reinterpret_cast<float4*>(base + kWsHeaderBytes + flags_bytes);
    cp.incl = cp.agg + (size_t)g.U * (size_t)g.Cg;
    cp.drop_unit = drop_unit;
    if (a.io == 1) {
        return g.bulk ? launch_lc<__nv_bfloat16, 4, true>(a, g, cp, s) : launch_lc<__nv_bfloat16, 1, false>(a, g, cp, s);
    }
    return g.bulk ? launch_lc<float, 4, true>(a, g, cp, s) : launch_lc<float, 1, false>(a, g, cp, s);
}

}  // namespace wkvb
