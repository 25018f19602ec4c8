// Chunked, time-parallel WKV forward in a single pass (12 B/element for fp32 I/O).
//
// The decay factor telescopes (RWKV transformer-math page, aicassindra.com, section
// "Why it collapses into a recurrence"), so the state after a span of tokens is an
// associative fold: a segment is summarised by (a, b, p) relative to its own running
// maximum, and two adjacent segments combine by decaying the earlier one over the
// later one's length and re-referencing to the larger exponent (rec_combine).
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
//      exponent M = max_i (k_i - (LC-1-i) w) first (kept as the record's exponent, a
//      single rounding), then one exp per element;
//   3. one thread per channel scans the NW chunk summaries (exclusive prefixes stay
//      in shared memory; the inclusive one is the tile aggregate);
//   4. warp 0 publishes the aggregate and looks back over the predecessor tiles of
//      the same channel group (decoupled look-back, Merrill & Garland 2016).  The 32
//      lanes poll the flags of 32 predecessors at once and stop at the nearest one
//      holding an inclusive prefix; the records in between are then loaded together
//      and folded, so a look-back costs a few L2 round trips whatever its depth.
//      Every wait is bounded; on expiry the error word is set and the missing carry
//      is taken as empty, so no successor can hang;
//   5. every warp combines the tile carry with its chunk's exclusive prefix and
//      re-scans its chunk from shared memory, writing y.  Within a chunk the output
//      and the state update share one exp: the state is kept relative to a reference
//      exponent r that decays with the history, so the new token's weight relative to
//      it is the output's weight times the per-channel constant 2^(w - u); r moves to
//      the current token only when that token dominates (see lazy_step).  Channels
//      with |u| or w too large for that constant fall back to the page's form.
// The last time segment's inclusive prefix is the final state (state_out).
#include "wkv_device.cuh"
#include "wkv_internal.h"
#include "wkv_vec.cuh"

// Tile shape per I/O type: V channels per lane (32 V per tile) and NW warps (chunks).
#ifndef WKV_F32_V
#define WKV_F32_V 2
#endif
#ifndef WKV_F32_NW
#define WKV_F32_NW 8
#endif
#ifndef WKV_BF16_V
#define WKV_BF16_V 4
#endif
#ifndef WKV_BF16_NW
#define WKV_BF16_NW 4
#endif

namespace wkvb {
namespace {

struct ChunkParams {
    int64_t groups_per_b, G, S;
    uint32_t* flags;  // [U]
    float4* agg;      // [U][Cg]
    float4* incl;     // [U][Cg]
    WsHeader* hdr;
    int64_t drop_unit;
};

template <typename TIO, int V, int NW, int LC, bool BULK>
__global__ void __launch_bounds__(NW * 32) chunked_kernel(ForwardArgs args, ChunkParams cp) {
    grid_dep_launch_dependents();
    grid_dep_wait();  // before any global memory access
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
            atomicCAS(args.dev_err, kDevOk, kDevBadWorkspace);
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
    }

    // per-thread channels and parameters (base-2 units), while the copies fly
    const int cl = lane * V;  // first channel of this lane within the tile
    const bool lane_active = cl < nch;
    float w2[V], u2[V];
#pragma unroll
    for (int q = 0; q < V; ++q) {
        const bool ok = lane_active && (cl + q < nch);
        w2[q] = ok ? args.w[c0 + cl + q] * kLog2e : 0.f;
        u2[q] = ok ? args.u[c0 + cl + q] * kLog2e : 0.f;
    }

    if (BULK) {
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
            atomicCAS(args.dev_err, kDevOk, kDevTimeoutCopy);
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

    // ---- 2. chunk summaries from the empty state ----
    const int r_begin = warp * LC;
    const int r_cnt = max(0, min(LC, len - r_begin));
    if (lane_active) {
        float gx[LC][V], M[V];
#pragma unroll
        for (int q = 0; q < V; ++q) M[q] = kPEmpty;
#pragma unroll
        for (int i = 0; i < LC; ++i) {
            if (i < r_cnt) {
                float kk[V];
                Vec<TIO, V>::load(ks + (r_begin + i) * Cg + cl, kk);
                const float back = (float)(r_cnt - 1 - i);
#pragma unroll
                for (int q = 0; q < V; ++q) {
                    gx[i][q] = fmaf(-back, w2[q], kk[q] * kLog2e);
                    M[q] = fmaxf(M[q], gx[i][q]);
                }
            }
        }
        float sa[V], sb[V];
#pragma unroll
        for (int q = 0; q < V; ++q) sa[q] = sb[q] = 0.f;
#pragma unroll
        for (int i = 0; i < LC; ++i) {
            if (i < r_cnt) {
                float vv[V];
                Vec<TIO, V>::load(vs + (r_begin + i) * Cg + cl, vv);
#pragma unroll
                for (int q = 0; q < V; ++q) {
                    const float e = ex2(gx[i][q] - M[q]);
                    sa[q] = fmaf(e, vv[q], sa[q]);
                    sb[q] += e;
                }
            }
        }
        // the record's exponent is M itself (anchor M, zero steps since)
#pragma unroll
        for (int q = 0; q < V; ++q) recs[warp * Cg + cl + q] = Rec{sa[q], sb[q], M[q], 0.f};
    }
    __syncthreads();

    // ---- 3. scan of the chunk summaries (one thread per channel) ----
    for (int cc = tid; cc < nch; cc += NT) {
        const float w2c = args.w[c0 + cc] * kLog2e;
        Rec run = rec_identity();
#pragma unroll
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
        const bool publish = unit != cp.drop_unit;
        Rec carry[V];
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
                    if (cl + q < nch) cp.agg[unit * Cg + cl + q] = rec_pack(aggs[cl + q]);
            }
            __threadfence();
            __syncwarp();
            if (lane == 0 && publish) st_release_u32(&cp.flags[unit], (epoch30 << 2) | 1u);

            Rec run[V];
#pragma unroll
            for (int q = 0; q < V; ++q) run[q] = rec_identity();
            float span = 0.f;
            int64_t hi = j - 1;  // newest predecessor not folded yet
            while (true) {
                // lane i watches predecessor hi - i
                const int64_t mine = hi - lane;
                const bool valid = mine >= 0;
                const uint32_t* myflag = &cp.flags[(valid ? mine : 0) * cp.G + g];
                uint32_t st = valid ? 0u : 3u;  // invalid lanes never block
                int m = -1;                     // lanes 0..m get folded
                bool found_incl = false;
                for (uint32_t it = 0; it <= args.spin_limit; ++it) {
                    if (st == 0u) {
                        const uint32_t f = ld_acquire_u32(myflag);
                        if ((f >> 2) == epoch30 && (f & 3u) != 0u) st = f & 3u;
                    }
                    const unsigned incl = __ballot_sync(0xffffffffu, valid && st == 2u);
                    const unsigned ready = __ballot_sync(0xffffffffu, st != 0u);
                    const int last = (int)min64(31, hi);  // last valid lane
                    const int stop = incl ? (__ffs(incl) - 1) : last;
                    const unsigned need = stop >= 31 ? 0xffffffffu : ((2u << stop) - 1u);
                    if ((ready & need) == need) {
                        m = stop;
                        found_incl = incl != 0;
                        break;
                    }
                    __nanosleep(64);
                }
                if (m < 0) {
                    // a predecessor never published: record it, take the rest of the carry as empty
                    if (lane == 0) {
                        atomicCAS(&cp.hdr->error, kDevOk, kDevTimeoutCarry);
                        atomicCAS(args.dev_err, kDevOk, kDevTimeoutCarry);
                        cp.hdr->error_unit = (uint32_t)unit;
                    }
                    break;
                }
                // Lane i acquired predecessor hi - i's flag; after the warp barrier every
                // lane reads the records behind the flags with L1-bypassing loads (the
                // producer wrote them before its fence and release).  Fold predecessors
                // hi .. hi - m, newest first, loading four at a time.
                __syncwarp();
                for (int i0 = 0; i0 <= m; i0 += 4) {
                    float4 buf[4][V];
                    uint32_t sts[4];
#pragma unroll
                    for (int ii = 0; ii < 4; ++ii) {
                        const int i = i0 + ii;
                        sts[ii] = __shfl_sync(0xffffffffu, st, i & 31);
                        if (i <= m && lane_active) {
                            const float4* src = (sts[ii] == 2u) ? cp.incl : cp.agg;
                            const int64_t pu = (hi - i) * cp.G + g;
#pragma unroll
                            for (int q = 0; q < V; ++q)
                                if (cl + q < nch) buf[ii][q] = ld_relaxed_f4(src + pu * Cg + cl + q);
                        }
                    }
#pragma unroll
                    for (int ii = 0; ii < 4; ++ii) {
                        if (i0 + ii <= m && lane_active) {
#pragma unroll
                            for (int q = 0; q < V; ++q)
                                if (cl + q < nch) run[q] = rec_combine(rec_unpack(buf[ii][q]), run[q], span, w2[q]);
                        }
                        if (i0 + ii <= m) span += (float)Ts;
                    }
                }
                if (found_incl) break;
                hi -= (int64_t)(m + 1);
                if (hi < 0) break;
            }
#pragma unroll
            for (int q = 0; q < V; ++q) carry[q] = run[q];
        }
        // inclusive prefix of this unit
        Rec inc[V];
#pragma unroll
        for (int q = 0; q < V; ++q)
            inc[q] = (cl + q < nch) ? rec_combine(carry[q], aggs[cl + q], (float)len, w2[q]) : rec_identity();
        if (lane_active) {
#pragma unroll
            for (int q = 0; q < V; ++q)
                if (cl + q < nch) cp.incl[unit * Cg + cl + q] = rec_pack(inc[q]);
        }
        __threadfence();
        __syncwarp();
        if (lane == 0 && publish) st_release_u32(&cp.flags[unit], (epoch30 << 2) | 2u);
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
        float a[V], bb[V], R[V], nn[V];
#pragma unroll
        for (int q = 0; q < V; ++q) {
            const Rec cr = rec_combine(carry_s[cl + q], recs[warp * Cg + cl + q], (float)r_begin, w2[q]);
            a[q] = cr.a;
            bb[q] = cr.b;
            R[q] = cr.anc;
            nn[q] = cr.n;
        }
        bool lazy_ok = true;
#pragma unroll
        for (int q = 0; q < V; ++q) lazy_ok = lazy_ok && fabsf(u2[q]) <= kLazyLimit && w2[q] <= kLazyLimit;
        if (lazy_ok) {
            float c[V];
#pragma unroll
            for (int q = 0; q < V; ++q) c[q] = ex2(w2[q] - u2[q]);
#pragma unroll
            for (int i = 0; i < LC; ++i) {
                if (i < r_cnt) {
                    const int r = r_begin + i;
                    float kk[V], vv[V], yy[V];
                    Vec<TIO, V>::load(ks + r * Cg + cl, kk);
                    Vec<TIO, V>::load(vs + r * Cg + cl, vv);
#pragma unroll
                    for (int q = 0; q < V; ++q)
                        yy[q] = lazy_step(a[q], bb[q], R[q], nn[q], kk[q] * kLog2e, vv[q], u2[q], w2[q], c[q]);
                    if (V == 1 || cl + V <= nch) {
                        Vec<TIO, V>::store(yg + (int64_t)r * C + cl, yy);
                    } else {
#pragma unroll
                        for (int q = 0; q < V; ++q)
                            if (cl + q < nch) io<TIO>::store(yg + (int64_t)r * C + cl + q, yy[q]);
                    }
                }
            }
        } else {
            float p[V];
#pragma unroll
            for (int q = 0; q < V; ++q) p[q] = fmaf(-nn[q], w2[q], R[q]);
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
    return launch_pdl(kern, dim3((unsigned)g.U), dim3(NW * 32), smem, s, a, cp);
}

template <typename TIO, int V, int NW, bool BULK>
cudaError_t launch_lc(const ForwardArgs& a, const ChunkGeom& g, const ChunkParams& cp, cudaStream_t s) {
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
    if (chunk != 0 && chunk != 4 && chunk != 8 && chunk != 16) return false;
    // bulk rows run the pipelined kernel (default 16 steps per chunk); chunk 4 and ragged
    // rows run the one-unit-per-CTA kernel above
    g->pipe = bulk && chunk != 4;
    const int LC = chunk != 0 ? chunk : 16;
    if (g->pipe) {
        g->V = 2;  // a lane owns a channel pair: 64 channels per tile (256-byte fp32 / 128-byte bf16 rows)
        g->NW = 8;
    } else {
        g->V = bulk ? (io == 1 ? WKV_BF16_V : WKV_F32_V) : 1;
        g->NW = bulk ? (io == 1 ? WKV_BF16_NW : WKV_F32_NW) : 4;
    }
    g->LC = LC;
    g->bulk = bulk;
    g->Cg = 32 * g->V;
    g->Ts = (int64_t)g->NW * LC;
    g->groups_per_b = (C + g->Cg - 1) / g->Cg;
    g->G = B * g->groups_per_b;
    g->S = (T + g->Ts - 1) / g->Ts;
    g->U = g->G * g->S;
    if (g->pipe) {
        // one slot of four tagged words per tile-channel (aggregate, then inclusive prefix)
        g->ws_bytes = kWsHeaderBytes + (size_t)g->U * (size_t)g->Cg * 32;
    } else {
        // flag per tile, 16-byte aggregate and inclusive records per tile-channel
        const size_t flags = ((size_t)g->U * 4 + 15) / 16 * 16;
        g->ws_bytes = kWsHeaderBytes + flags + 2 * (size_t)g->U * (size_t)g->Cg * 16;
    }
    return true;
}

bool chunked_path_fuses_gate(const ChunkGeom& g) { return g.pipe; }

cudaError_t launch_forward_chunked(const ForwardArgs& a, const ChunkGeom& g, void* ws, int64_t drop_unit,
                                   cudaStream_t s) {
    if (g.pipe) return launch_forward_tmem(a, g, ws, drop_unit, s);
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
        return g.bulk ? launch_lc<__nv_bfloat16, WKV_BF16_V, WKV_BF16_NW, true>(a, g, cp, s)
                      : launch_lc<__nv_bfloat16, 1, 4, false>(a, g, cp, s);
    }
    return g.bulk ? launch_lc<float, WKV_F32_V, WKV_F32_NW, true>(a, g, cp, s)
                  : launch_lc<float, 1, 4, false>(a, g, cp, s);
}

}  // namespace wkvb
