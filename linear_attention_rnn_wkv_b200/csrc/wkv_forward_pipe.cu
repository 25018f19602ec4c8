// Persistent, warp-specialised chunked WKV forward (the default chunked path when
// rows are 16-byte multiples).
//
// Same arithmetic and the same inter-CTA protocol as chunked_kernel (wkv_forward_
// chunked.cu): a unit is a tile of Ts = NWS * LC time steps by Cg = 32 * V channels;
// units are taken by an atomic ticket in time-segment-major order; each unit's chunk
// summaries fold into a tile aggregate, a decoupled look-back over earlier segments of
// the same channel group yields the carry, and the chunks are re-scanned from the
// carry to write y (the decay telescopes: RWKV transformer-math page, aicassindra.com,
// section "Why it collapses into a recurrence").
//
// What changes is the schedule.  One CTA per SM runs for the whole launch and keeps
// NS units in flight in a shared-memory ring; each role is a set of warps that moves
// from unit to unit on its own, handing over through mbarriers:
//   producer  (1 warp)   announces the unit of its (prefetched) ticket (`tick`), and
//                        issues the TMA copies of its k and v rows and of its channels'
//                        w and u (`full`);
//   summarise (NWS warps) one chunk summary each (`chunks`);
//   look-back (NS warps, one per ring stage) starts as soon as the unit is announced,
//                        while its rows are still loading: folds the predecessors'
//                        records into the carry; once the summaries are in, scans them
//                        and publishes the tile aggregate (or, if the carry is already
//                        known, the inclusive prefix); hands the carry over (`carry`);
//   emit      (NWS warps) re-scan each chunk from its carry and write y, then free the
//                        stage (`empty`) for the producer.
// So a unit's load, its look-back and the arithmetic of neighbouring units overlap,
// and no warp waits at a CTA-wide barrier.  All waits are bounded (error word on
// expiry, then the pipeline keeps moving).  Deadlock freedom: roles handle a CTA's units
// in ticket order and every cross-CTA wait is on a smaller ticket, so the oldest
// unfinished unit in the whole grid can always complete.
#include "wkv_device.cuh"
#include "wkv_internal.h"
#include "wkv_vec.cuh"
#include "wkv_pipe_common.cuh"

namespace wkvb {
namespace {

template <typename TIO, int V, int NWS, int LC, int NS>
struct PipeLayout {
    static constexpr int Cg = 32 * V;
    static constexpr int Ts = NWS * LC;
    static constexpr size_t tile = sizeof(TIO) * Ts * Cg;  // one array (k or v)
    static constexpr size_t recs_off = 2 * tile;           // Rec [NWS][Cg]
    static constexpr size_t carry_off = recs_off + sizeof(Rec) * NWS * Cg;
    static constexpr size_t mx_off = carry_off + sizeof(Rec) * Cg;  // float [NWS][Cg]: each chunk's max exponent
    static constexpr size_t stage = align128(mx_off + sizeof(float) * NWS * Cg);
    static constexpr int BR = kBoxRows < Ts ? kBoxRows : Ts;  // rows per TMA box
    static constexpr int NB = Ts / BR;                           // boxes per array
    static constexpr int NBAR = 4 + NB;                          // mbarriers per stage
    static constexpr size_t bars_off = NS * stage;
    static constexpr size_t misc_off = bars_off + NS * NBAR * 8;  // stage unit ids, epoch, end index
    static constexpr size_t total = misc_off + NS * 8 + 24;
    static constexpr size_t per_stage = stage + NBAR * 8 + 8;  // what one more stage costs
};

// per stage: kTick, kChunks, kCarry, kEmpty, then one `full` barrier per TMA box of rows
enum { kTick = 0, kChunks = 1, kCarry = 2, kEmpty = 3, kFull0 = 4 };

template <typename TIO, int V, int NWS, int LC, int NS>
__global__ void __launch_bounds__((1 + 2 * NWS + NS) * 32, 1)
    pipe_kernel(ForwardArgs args, PipeParams pp, const __grid_constant__ CUtensorMap tmk,
                const __grid_constant__ CUtensorMap tmv) {
    using Lay = PipeLayout<TIO, V, NWS, LC, NS>;
    static_assert(V == 2, "a lane owns one channel pair (records move as pairs)");
    constexpr int Cg = Lay::Cg;
    constexpr int Ts = Lay::Ts;
    constexpr int W_S0 = 1, W_L0 = 1 + NWS, W_E0 = 1 + NWS + NS;
    extern __shared__ __align__(128) unsigned char smem[];
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Lay::bars_off);
    int64_t* stage_unit = reinterpret_cast<int64_t*>(smem + Lay::misc_off);
    uint32_t* s_epoch = reinterpret_cast<uint32_t*>(stage_unit + NS);
    volatile int64_t* s_iend = reinterpret_cast<volatile int64_t*>(stage_unit + NS + 1);
    constexpr int NB = Lay::NB, BR = Lay::BR;
    auto bar = [&](int s, int kind) { return &bars[s * Lay::NBAR + kind]; };
    auto ktile = [&](int s) { return reinterpret_cast<TIO*>(smem + s * Lay::stage); };
    auto vtile = [&](int s) { return reinterpret_cast<TIO*>(smem + s * Lay::stage + Lay::tile); };
    auto recs = [&](int s) { return reinterpret_cast<Rec*>(smem + s * Lay::stage + Lay::recs_off); };
    auto carries = [&](int s) { return reinterpret_cast<Rec*>(smem + s * Lay::stage + Lay::carry_off); };
    auto chunk_max = [&](int s) { return reinterpret_cast<float*>(smem + s * Lay::stage + Lay::mx_off); };

    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;
    const int64_t T = args.T, C = args.C, BC = args.B * args.C;
    const uint32_t lim = args.spin_limit;

    if (tid == 0) {
        *s_epoch = (*reinterpret_cast<volatile uint32_t*>(&pp.hdr->epoch) + 1u) & 0x3FFFFFFFu;
        *s_iend = INT64_MAX;
        for (int s = 0; s < NS; ++s) {
            for (int b = 0; b < NB; ++b) mbar_init(bar(s, kFull0 + b), 1);
            mbar_init(bar(s, kTick), 1);
            mbar_init(bar(s, kChunks), NWS);
            mbar_init(bar(s, kCarry), 1);
            mbar_init(bar(s, kEmpty), NWS);
        }
        fence_mbar_init();
    }
    __syncthreads();
    const uint32_t epoch30 = *s_epoch;
    const uint32_t tag_agg = (epoch30 << 2) | 1u, tag_incl = (epoch30 << 2) | 2u;
    auto report = [&](uint32_t code) {
        atomicCAS(&pp.hdr->error, kDevOk, code);
        atomicCAS(args.dev_err, kDevOk, code);
    };

    struct Geo {
        int64_t j, g, b, c0, t0;
        int len, nch;
    };
    auto geo = [&](int64_t unit) {
        Geo q;
        q.j = unit / pp.G;
        q.g = unit % pp.G;
        q.b = q.g / pp.groups_per_b;
        q.c0 = (q.g % pp.groups_per_b) * Cg;
        q.t0 = q.j * Ts;
        q.len = (int)min64(Ts, T - q.t0);
        q.nch = (int)min64(Cg, C - q.c0);
        return q;
    };

    if (warp == 0) {
        // ------------------------------- producer -------------------------------
        if (lane == 0) {
            // A ticket is taken only once a stage is free: a unit that holds a ticket starts
            // at once, so no later unit ever waits on one that sits idle.
            for (int64_t i = 0;; ++i) {
                const int s = (int)(i % NS);
                if (i >= NS && !mbar_wait(bar(s, kEmpty), (uint32_t)((i / NS - 1) & 1), lim)) report(kDevTimeoutCopy);
                const uint32_t t = atomicAdd(&pp.hdr->ticket, 1u);
                if (t >= (uint32_t)pp.U + gridDim.x) report(kDevBadWorkspace);
                if (t >= (uint32_t)pp.U) {
                    *s_iend = i;
                    stage_unit[s] = -1;
                    mbar_arrive(bar(s, kTick));
                    for (int b = 0; b < NB; ++b) mbar_arrive(bar(s, kFull0 + b));
                    break;
                }
                const int64_t unit = t;
                WKV_TRACE_EVENT(unit, 0);
                stage_unit[s] = unit;
                mbar_arrive(bar(s, kTick));
                const Geo q = geo(unit);
                // each box of BR rows (k and v) completes its own barrier, so the summarisers
                // of the first chunks start while later rows are still in flight
#pragma unroll
                for (int b = 0; b < NB; ++b) {
                    uint64_t* fb = bar(s, kFull0 + b);
                    mbar_arrive_expect_tx(fb, 2u * (uint32_t)(BR * Cg * sizeof(TIO)));
                    tma_load_3d(ktile(s) + b * BR * Cg, &tmk, (int)q.c0, (int)(q.t0 + b * BR), (int)q.b, fb);
                    tma_load_3d(vtile(s) + b * BR * Cg, &tmv, (int)q.c0, (int)(q.t0 + b * BR), (int)q.b, fb);
                }
            }
        }
        __syncwarp();
    } else if (warp < W_L0) {
        // ------------------------------- summarise ------------------------------
        // Every warp summarises its own chunk of the tile and signals the stage.
        const int sw = warp - W_S0;
        for (int64_t i = 0;; ++i) {
            const int s = (int)(i % NS);
            const uint32_t ph = (uint32_t)((i / NS) & 1);
            if (!mbar_wait(bar(s, kFull0 + sw * LC / BR), ph, lim) && lane == 0) report(kDevTimeoutCopy);
            const int64_t unit = stage_unit[s];
            if (unit < 0) break;
            if (sw == 0 && lane == 0) WKV_TRACE_EVENT(unit, 1);
            const Geo q = geo(unit);
            const int cl = lane * V;
            const bool lane_active = cl < q.nch;
            const int r_begin = sw * LC;
            const int r_cnt = max(0, min(LC, q.len - r_begin));
            float w2[V];
#pragma unroll
            for (int c = 0; c < V; ++c)
                w2[c] = (lane_active && cl + c < q.nch)
                            ? args.w[q.c0 + cl + c] * kLog2e
                            : 0.f;
            if (lane_active && WKV_PIPE_PACKED) {
                // the same arithmetic as below on the lane's channel pair with f32x2 ops
                const TIO* kt = ktile(s);
                const TIO* vt = vtile(s);
                const float2 w2p = make_float2(w2[0], w2[1]);
                const float2 L2 = make_float2(kLog2e, kLog2e);
                float2 gx[LC];
                float M0 = kPEmpty, M1 = kPEmpty;
#pragma unroll
                for (int r = 0; r < LC; ++r) {
                    if (r < r_cnt) {
                        float kk[V];
                        Vec<TIO, V>::load(kt + (r_begin + r) * Cg + cl, kk);
                        const float back = -(float)(r_cnt - 1 - r);
                        gx[r] = __ffma2_rn(make_float2(back, back), w2p, __fmul2_rn(make_float2(kk[0], kk[1]), L2));
                        M0 = fmaxf(M0, gx[r].x);
                        M1 = fmaxf(M1, gx[r].y);
                    }
                }
                const float2 nM = make_float2(-M0, -M1);
                float2 sa = make_float2(0.f, 0.f), sb = make_float2(0.f, 0.f);
#pragma unroll
                for (int r = 0; r < LC; ++r) {
                    if (r < r_cnt) {
                        float vv[V];
                        Vec<TIO, V>::load(vt + (r_begin + r) * Cg + cl, vv);
                        const float2 x = __fadd2_rn(gx[r], nM);
                        const float2 e = make_float2(ex2(x.x), ex2(x.y));
                        sa = __ffma2_rn(e, make_float2(vv[0], vv[1]), sa);
                        sb = __fadd2_rn(sb, e);
                    }
                }
                Rec* rc = recs(s);
                rc[sw * Cg + cl] = Rec{sa.x, sb.x, M0, 0.f};
                rc[sw * Cg + cl + 1] = Rec{sa.y, sb.y, M1, 0.f};
                *reinterpret_cast<float2*>(chunk_max(s) + sw * Cg + cl) = make_float2(M0, M1);
            } else if (lane_active) {
                float gx[LC][V], M[V], sa[V], sb[V];
#pragma unroll
                for (int c = 0; c < V; ++c) {
                    M[c] = kPEmpty;
                    sa[c] = sb[c] = 0.f;
                }
                const TIO* kt = ktile(s);
                const TIO* vt = vtile(s);
#pragma unroll
                for (int r = 0; r < LC; ++r) {
                    if (r < r_cnt) {
                        float kk[V];
                        Vec<TIO, V>::load(kt + (r_begin + r) * Cg + cl, kk);
                        const float back = (float)(r_cnt - 1 - r);
#pragma unroll
                        for (int c = 0; c < V; ++c) {
                            gx[r][c] = fmaf(-back, w2[c], kk[c] * kLog2e);
                            M[c] = fmaxf(M[c], gx[r][c]);
                        }
                    }
                }
#pragma unroll
                for (int r = 0; r < LC; ++r) {
                    if (r < r_cnt) {
                        float vv[V];
                        Vec<TIO, V>::load(vt + (r_begin + r) * Cg + cl, vv);
#pragma unroll
                        for (int c = 0; c < V; ++c) {
                            const float e = ex2(gx[r][c] - M[c]);
                            sa[c] = fmaf(e, vv[c], sa[c]);
                            sb[c] += e;
                        }
                    }
                }
                Rec* rc = recs(s);
#pragma unroll
                for (int c = 0; c < V; ++c) {
                    rc[sw * Cg + cl + c] = Rec{sa[c], sb[c], M[c], 0.f};
                    chunk_max(s)[sw * Cg + cl + c] = M[c];
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(bar(s, kChunks));
            if (sw == 0 && lane == 0) WKV_TRACE_EVENT(unit, 2);
        }
    } else if (warp < W_E0) {
        // ------------------------------- look-back ------------------------------
        // Look-back warp l owns ring stage l: units i = l, l + NS, ...
        const int s = warp - W_L0;
        for (int64_t i = s;; i += NS) {
            const uint32_t ph = (uint32_t)((i / NS) & 1);
            bool got = false, gone = false;
            for (uint32_t it = 0; it <= lim; ++it) {
                if (WKV_WAIT_HINT ? mbar_try_wait_hint(bar(s, kTick), ph, WKV_WAIT_HINT) : mbar_try_wait(bar(s, kTick), ph)) {
                    got = true;
                    break;
                }
                if (*s_iend < i) {  // past the end (the sentinel unit itself still arrives)
                    gone = true;
                    break;
                }
                if (!WKV_WAIT_HINT) __nanosleep(32);
            }
            if (gone) break;
            if (!got && lane == 0) report(kDevTimeoutCopy);
            const int64_t unit = stage_unit[s];
            if (unit < 0) {
                if (lane == 0) mbar_arrive(bar(s, kCarry));
                break;
            }
            const Geo q = geo(unit);
            const int cl = lane * V;
            const bool lane_active = cl < q.nch;
            float w2[V];
#pragma unroll
            for (int c = 0; c < V; ++c) w2[c] = (lane_active && cl + c < q.nch) ? args.w[q.c0 + cl + c] * kLog2e : 0.f;
            // scan the chunk summaries (exclusive prefixes for the emitters) and publish the
            // tile aggregate for later segments before looking back; the first read of the
            // newest predecessor's slot is issued first, so its round trip overlaps the scan
            if (!mbar_wait(bar(s, kChunks), ph, lim) && lane == 0) report(kDevTimeoutCarry);
            if (lane == 0) WKV_TRACE_EVENT(unit, 3);
            RawPair first;
            if (q.j > 0 && lane_active) first = load_pair<Cg>(pp.slot + ((q.j - 1) * pp.G + q.g) * 4 * Cg, cl);
            Rec agg[V];
            if (lane_active) {
                Rec* rc = recs(s);
#pragma unroll
                for (int c = 0; c < V; ++c) agg[c] = rec_identity();
#pragma unroll
                for (int w = 0; w < NWS; ++w) {
                    const int lw = max(0, min(LC, q.len - w * LC));
#pragma unroll
                    for (int c = 0; c < V; ++c) {
                        const Rec r = rc[w * Cg + cl + c];
                        rc[w * Cg + cl + c] = agg[c];  // exclusive prefix of chunk w
                        if (lw > 0) agg[c] = rec_combine(agg[c], r, (float)lw, w2[c]);
                    }
                }
                // (nch is even, so a lane's two channels are both in range or both out)
                if (q.j > 0 && unit != pp.drop_unit) publish_pair<Cg>(pp.slot + unit * 4 * Cg, cl, agg[0], agg[1], tag_agg);
            }
            if (lane == 0) WKV_TRACE_EVENT(unit, 4);
            Rec run[V];
            if (q.j == 0) {
#pragma unroll
                for (int c = 0; c < V; ++c) {
                    const int cc = cl + c;
                    run[c] = (args.state_in && cc < q.nch) ? rec_from_state(args.state_in, q.b * C + q.c0 + cc, BC)
                                                           : rec_identity();
                }
            } else {
#pragma unroll
                for (int c = 0; c < V; ++c) run[c] = rec_identity();
                // Each lane looks back for its channel pair, reading the slots of the kLook
                // newest unfolded predecessors in one round trip: it folds aggregates from the
                // newest backwards and stops at the first inclusive prefix (the carry is then
                // known) or at the first slot that is not yet published.
                float span = 0.f;
                int64_t hi = q.j - 1;
                bool done = !lane_active;
                uint32_t nap = 64;
                bool all_done = false;
                for (uint32_t it = 0; it <= lim && !all_done; ++it) {
                    if (!done) {
                        RawPair raw[kLook];
#pragma unroll
                        for (int d = 0; d < kLook; ++d)
                            if (hi - d >= 0)
                                raw[d] = (it == 0 && d == 0)
                                             ? first
                                             : load_pair<Cg>(pp.slot + ((hi - d) * pp.G + q.g) * 4 * Cg, cl);
                        bool progressed = false;
#pragma unroll
                        for (int d = 0; d < kLook; ++d) {
                            if (done) break;
                            Rec r0, r1;
                            const int kind = pair_kind(raw[d], tag_agg, tag_incl, r0, r1);
                            if (kind == 0) break;
                            run[0] = rec_combine(r0, run[0], span, w2[0]);
                            run[1] = rec_combine(r1, run[1], span, w2[1]);
                            progressed = true;
                            if (kind == 2) {
                                done = true;
                            } else {
                                span += (float)Ts;
                                if (--hi < 0) done = true;
                            }
                        }
                        if (!done && !progressed) {
                            __nanosleep(nap);
                            nap = nap < 1024 ? nap * 2 : 1024;
                        } else if (progressed) {
                            nap = 64;
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
            // publish the inclusive prefix (it overwrites the aggregate), then hand the carry
            // to the emitters
            Rec inc[V];
            if (lane_active) {
#pragma unroll
                for (int c = 0; c < V; ++c) inc[c] = rec_combine(run[c], agg[c], (float)q.len, w2[c]);
                if (unit != pp.drop_unit) publish_pair<Cg>(pp.slot + unit * 4 * Cg, cl, inc[0], inc[1], tag_incl);
            }
            if (lane == 0) WKV_TRACE_EVENT(unit, 7);
            if (lane_active) {
                Rec* cs = carries(s);
#pragma unroll
                for (int c = 0; c < V; ++c) cs[cl + c] = run[c];
            }
            __syncwarp();
            if (lane == 0) {
                WKV_TRACE_EVENT(unit, 6);
                mbar_arrive(bar(s, kCarry));
            }
            if (lane_active && q.j == pp.S - 1 && args.state_out) {
#pragma unroll
                for (int c = 0; c < V; ++c) {
                    if (cl + c >= q.nch) continue;
                    const int64_t bc = q.b * C + q.c0 + cl + c;
                    args.state_out[bc] = inc[c].a;
                    args.state_out[BC + bc] = inc[c].b;
                    args.state_out[2 * BC + bc] = rec_p(inc[c], w2[c]) * kLn2;
                }
            }
        }
    } else {
        // --------------------------------- emit ---------------------------------
        const int ew = warp - W_E0;  // chunk index
        for (int64_t i = 0;; ++i) {
            const int s = (int)(i % NS);
            const uint32_t ph = (uint32_t)((i / NS) & 1);
            if (!mbar_wait(bar(s, kCarry), ph, lim) && lane == 0) report(kDevTimeoutCarry);
            (void)mbar_wait(bar(s, kFull0 + ew * LC / BR), ph, lim);  // already complete; orders the tile reads
            const int64_t unit = stage_unit[s];
            if (unit < 0) break;
            if (ew == 0 && lane == 0) WKV_TRACE_EVENT(unit, 8);
            const Geo q = geo(unit);
            const int cl = lane * V;
            const int r_begin = ew * LC;
            const int r_cnt = max(0, min(LC, q.len - r_begin));
            if (cl < q.nch && r_cnt > 0) {
                float w2[V], u2[V], a[V], bb[V], R[V], nn[V];
                bool lazy_ok = true;
#pragma unroll
                for (int c = 0; c < V; ++c) {
                    const bool ok = cl + c < q.nch;
                    w2[c] = ok ? args.w[q.c0 + cl + c] * kLog2e : 0.f;
                    u2[c] = ok ? args.u[q.c0 + cl + c] * kLog2e : 0.f;
                    const Rec cr = rec_combine(carries(s)[cl + c], recs(s)[ew * Cg + cl + c], (float)r_begin, w2[c]);
                    a[c] = cr.a;
                    bb[c] = cr.b;
                    R[c] = cr.anc;
                    nn[c] = cr.n;
                    lazy_ok = lazy_ok && fabsf(u2[c]) <= kLazyLimit && w2[c] <= kLazyLimit;
                }
                const TIO* kt = ktile(s);
                const TIO* vt = vtile(s);
                TIO* yg = static_cast<TIO*>(args.y) + (q.b * T + q.t0) * C + q.c0;
                // Fixed-frame re-scan.  Seen from the chunk's last row, each token's weight
                // e_i = 2^(k_i - (L-1-i) w - G) and the carried-in history K do not change from
                // row to row (everything decays at the same rate), so with running sums S of
                // K + e_i v_i and K + e_i over earlier rows and c = 2^(w - u)
                //   y_r = (S^a + e_r v_r / c) / (S^b + e_r / c):
                // no re-referencing and no selects, and only S is carried from row to row (the
                // first row of a sequence without history returns v itself, as the
                // recurrence does; the rearranged form v + (S^a - S^b v) / (...) would do that
                // by itself but cancels badly when the history dominates).  The frame G lies
                // at most 100 above the larger of the history and the first token (so no term
                // that matters can be flushed), at most 64 below the history (so K stays finite)
                // and high enough that no later token's term can overflow; a chunk whose range
                // leaves no such G takes the token-by-token path below.
                bool frame_ok = false;
                float2 fSa, fSb, fnG, fic;
                if (WKV_PIPE_FRAME && lazy_ok) {
                    float k0[V];
                    Vec<TIO, V>::load(kt + r_begin * Cg + cl, k0);
                    float fa[V], fb[V], fg[V], fi[V];
                    bool ok = true;
                    const float fc = (float)r_cnt;
#pragma unroll
                    for (int c = 0; c < V; ++c) {
                        const float M = chunk_max(s)[ew * Cg + cl + c];
                        const float hK = fmaf(-fc, w2[c], fmaf(-nn[c], w2[c], R[c]));  // history, at the last row
                        const float h0 = fmaf(-(fc - 1.f), w2[c], k0[c] * kLog2e);        // first token, same
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
                    frame_ok = ok;
                    fSa = make_float2(fa[0], fa[1]);
                    fSb = make_float2(fb[0], fb[1]);
                    fnG = make_float2(fg[0], fg[1]);
                    fic = make_float2(fi[0], fi[1]);
                }
                if (frame_ok) {
                    const float2 L2 = make_float2(kLog2e, kLog2e);
                    const float2 w2p = make_float2(w2[0], w2[1]);
                    const float back0 = 1.f - (float)r_cnt;  // -(steps from row 0 to the last row)
#pragma unroll
                    for (int r = 0; r < LC; ++r) {
                        if (r < r_cnt) {
                            const int row = r_begin + r;
                            float kk[V], vv[V], yy[V];
                            Vec<TIO, V>::load(kt + row * Cg + cl, kk);
                            Vec<TIO, V>::load(vt + row * Cg + cl, vv);
                            const float2 vp = make_float2(vv[0], vv[1]);
                            // k - G first: the large cancellation happens inside one rounding
                            const float back = back0 + (float)r;
                            const float2 x = __ffma2_rn(make_float2(back, back), w2p,
                                                        __ffma2_rn(make_float2(kk[0], kk[1]), L2, fnG));
                            const float2 e = make_float2(ex2(x.x), ex2(x.y));
                            const float2 ec = __fmul2_rn(e, fic);
                            const float2 num = __ffma2_rn(ec, vp, fSa);
                            const float2 den = __fadd2_rn(fSb, ec);
                            const float2 yv = __fmul2_rn(num, make_float2(rcp(den.x), rcp(den.y)));
                            yy[0] = yv.x;
                            yy[1] = yv.y;
                            if (r == 0) {
                                if (fSb.x == 0.f) yy[0] = vv[0];
                                if (fSb.y == 0.f) yy[1] = vv[1];
                            }
                            fSa = __ffma2_rn(e, vp, fSa);
                            fSb = __fadd2_rn(fSb, e);
                            Vec<TIO, V>::store(yg + (int64_t)row * C + cl, yy);
                        }
                    }
                } else if (lazy_ok && WKV_PIPE_PACKED) {
                    // lazy_step on the lane's channel pair with f32x2 ops; the reference is
                    // kept negated (nR = -R) and u + k formed with one FMA, so no negation
                    // is needed inside the loop
                    const float2 L2 = make_float2(kLog2e, kLog2e), nL2 = make_float2(-kLog2e, -kLog2e);
                    const float2 u2p = make_float2(u2[0], u2[1]), nu2p = make_float2(-u2[0], -u2[1]);
                    const float2 w2p = make_float2(w2[0], w2[1]);
                    const float2 cwp = make_float2(ex2(w2[0] - u2[0]), ex2(w2[1] - u2[1]));
                    const float2 one = make_float2(1.f, 1.f);
                    float2 ap = make_float2(a[0], a[1]), bp = make_float2(bb[0], bb[1]);
                    float2 nRp = make_float2(-R[0], -R[1]), np = make_float2(nn[0], nn[1]);
#pragma unroll
                    for (int r = 0; r < LC; ++r) {
                        if (r < r_cnt) {
                            const int row = r_begin + r;
                            float kk[V], vv[V], yy[V];
                            Vec<TIO, V>::load(kt + row * Cg + cl, kk);
                            Vec<TIO, V>::load(vt + row * Cg + cl, vv);
                            const float2 kp = make_float2(kk[0], kk[1]), vp = make_float2(vv[0], vv[1]);
                            const float2 uk = __ffma2_rn(kp, L2, u2p);
                            const float2 nuk = __ffma2_rn(kp, nL2, nu2p);
                            const float2 d = __ffma2_rn(np, w2p, __fadd2_rn(nRp, uk));  // (u + k) - (R - n w)
                            const bool c0 = d.x > 0.f, c1 = d.y > 0.f;
                            const float e0 = ex2(-fabsf(d.x)), e1 = ex2(-fabsf(d.y));
                            const float2 sa = make_float2(c0 ? e0 : 1.f, c1 ? e1 : 1.f);
                            const float2 sv = make_float2(c0 ? 1.f : e0, c1 ? 1.f : e1);
                            const float2 t = __fmul2_rn(sa, ap);
                            const float2 num = __ffma2_rn(sv, vp, t);
                            const float2 den = __ffma2_rn(sa, bp, sv);
                            const float2 yv = __fmul2_rn(num, make_float2(rcp(den.x), rcp(den.y)));
                            const float2 nw = __fmul2_rn(sv, cwp);
                            ap = __ffma2_rn(nw, vp, t);
                            bp = __ffma2_rn(sa, bp, nw);
                            nRp = make_float2(c0 ? nuk.x : nRp.x, c1 ? nuk.y : nRp.y);
                            const float2 n1 = __fadd2_rn(np, one);
                            np = make_float2(c0 ? 1.f : n1.x, c1 ? 1.f : n1.y);
                            yy[0] = yv.x;
                            yy[1] = yv.y;
                            Vec<TIO, V>::store(yg + (int64_t)row * C + cl, yy);
                        }
                    }
                } else if (lazy_ok) {
                    float cw[V];
#pragma unroll
                    for (int c = 0; c < V; ++c) cw[c] = ex2(w2[c] - u2[c]);
#pragma unroll
                    for (int r = 0; r < LC; ++r) {
                        if (r < r_cnt) {
                            const int row = r_begin + r;
                            float kk[V], vv[V], yy[V];
                            Vec<TIO, V>::load(kt + row * Cg + cl, kk);
                            Vec<TIO, V>::load(vt + row * Cg + cl, vv);
#pragma unroll
                            for (int c = 0; c < V; ++c)
                                yy[c] = lazy_step(a[c], bb[c], R[c], nn[c], kk[c] * kLog2e, vv[c], u2[c], w2[c], cw[c]);
                            Vec<TIO, V>::store(yg + (int64_t)row * C + cl, yy);
                        }
                    }
                } else {
                    float p[V];
#pragma unroll
                    for (int c = 0; c < V; ++c) p[c] = fmaf(-nn[c], w2[c], R[c]);
                    for (int r = 0; r < r_cnt; ++r) {
                        const int row = r_begin + r;
                        float kk[V], vv[V], yy[V];
                        Vec<TIO, V>::load(kt + row * Cg + cl, kk);
                        Vec<TIO, V>::load(vt + row * Cg + cl, vv);
#pragma unroll
                        for (int c = 0; c < V; ++c) {
                            const float k2 = kk[c] * kLog2e;
                            yy[c] = wkv_output<false>(a[c], bb[c], p[c], u2[c] + k2, vv[c]);
                            wkv_fold<false>(a[c], bb[c], p[c], p[c] - w2[c], k2, vv[c], w2[c]);
                        }
                        Vec<TIO, V>::store(yg + (int64_t)row * C + cl, yy);
                    }
                }
            }
            __syncwarp();
            if (ew == 0 && lane == 0) WKV_TRACE_EVENT(unit, 9);
            if (lane == 0) mbar_arrive(bar(s, kEmpty));
        }
    }

    __syncthreads();
    if (tid == 0) {
        __threadfence();
        const uint32_t finished = atomicAdd(&pp.hdr->done, 1u) + 1u;
        if (finished == gridDim.x) {
            atomicExch(&pp.hdr->ticket, 0u);
            atomicExch(&pp.hdr->done, 0u);
            atomicExch(&pp.hdr->epoch, epoch30);
        }
    }
}

template <typename TIO, int V, int NWS, int LC>
cudaError_t launch_pipe_t(const ForwardArgs& a, const ChunkGeom& g, const PipeParams& pp, cudaStream_t s) {
    // as many stages as fit in the 227 KB a CTA may use (at most 5)
    constexpr size_t per_stage = PipeLayout<TIO, V, NWS, LC, 1>::per_stage;
    constexpr size_t budget = 232448 - 24;  // the most dynamic shared memory a CTA may use, minus the misc words
    constexpr int NS = (int)(budget / per_stage > 5 ? 5 : budget / per_stage);
    static_assert(NS >= 3, "tile too large for a three-stage ring");
    using Lay = PipeLayout<TIO, V, NWS, LC, NS>;
    static_assert(Lay::total <= 232448, "shared memory layout over the per-CTA limit");
    auto kern = pipe_kernel<TIO, V, NWS, LC, NS>;
    CUtensorMap tmk, tmv;
    static_assert(Lay::Ts % Lay::BR == 0, "tile rows must be a multiple of the box rows");
    static_assert(LC <= Lay::BR && Lay::BR % LC == 0, "a chunk must lie inside one box");
    if (!make_tile_map(&tmk, a.k, a.B, a.T, a.C, a.io, Lay::Cg, Lay::BR) ||
        !make_tile_map(&tmv, a.v, a.B, a.T, a.C, a.io, Lay::Cg, Lay::BR))
        return cudaErrorInvalidValue;
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
    kern<<<(unsigned)grid, (1 + 2 * NWS + NS) * 32, Lay::total, s>>>(a, pp, tmk, tmv);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_forward_pipe(const ForwardArgs& a, const ChunkGeom& g, void* ws, int64_t drop_unit,
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
    if (a.io == 1) {
        if (g.V == 2 && g.NW == 8 && g.LC == 8) return launch_pipe_t<__nv_bfloat16, 2, 8, 8>(a, g, pp, s);
        if (g.V == 2 && g.NW == 8 && g.LC == 16) return launch_pipe_t<__nv_bfloat16, 2, 8, 16>(a, g, pp, s);
        return cudaErrorInvalidValue;
    }
    if (g.V == 2 && g.NW == 8 && g.LC == 8) return launch_pipe_t<float, 2, 8, 8>(a, g, pp, s);
    if (g.V == 2 && g.NW == 8 && g.LC == 16) return launch_pipe_t<float, 2, 8, 16>(a, g, pp, s);
    return cudaErrorInvalidValue;
}

}  // namespace wkvb
