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
//   X_start = X_local + e^{-w len} X,   X'_start = X'_local + e^{-w len} (X' + len X),
// and a span's local sums at its left edge t0 - 1 are the plain weighted sums
//   X_local = sum_{t in span} e^{-(t-t0) w} gy_t / D_t,  X'_local = the same weighted by (t - t0),
// which can be accumulated walking left to right.
//
// Time-parallel in segments of kSeg steps, one thread per (b, c, segment), two launches, each
// handing its units out by an atomic ticket so that every wait is on a smaller ticket:
//   A  the segments in time order: each segment's forward recurrence from the empty state
//      gives its record, a decoupled look-back over the earlier segments of its channel folds
//      their published records into its starting state (written for R), and the state at its
//      end is published for the later segments; gw, gu are zeroed for R's atomics;
//   R  the segments in reverse time order: each runs its forward from its starting state,
//      keeping per position the output's reference exponent q_t, 1 / Dn_t (D_t = Dn_t 2^{q_t})
//      and y_t in shared memory while it accumulates its local (X, Y, X', Y') left to right;
//      publishes them; folds in the published sums of the later segments of its channel (a
//      decoupled look-back towards the end of the sequence) to get its incoming sums; publishes
//      what leaves it to the left; then runs its adjoint recurrence from the incoming sums ->
//      gk, gv, and gw, gu partials added with atomics.
// k, v are read once by A and once by R, gy once, and gk, gv written once (28 B per element);
// R's adjoint pass reads its segment's k, v, gy again straight after its forward pass, from
// the L2.  Nothing per position is stored in global memory.
// Numerics: the forward keeps an anchored reference p = anc - n w (no drift from rounding
// p - w); the adjoint sums are held relative to a reference r (X = x 2^{-r}) chosen so every
// rescaling exponent is <= 0, and e^{k_i} X_i = x 2^{k_i log2 e - r} <= x because k_i never
// exceeds the reference of a later output.
#include "wkv_device.cuh"
#include "wkv_internal.h"

namespace wkvb {
namespace {

constexpr int kSeg = 32;           // time steps per segment
constexpr int kBlk = 16;           // steps whose loads are issued together
constexpr int kThreads = 128;      // threads per block (channels of one (b, segment))
constexpr float kRNone = 3.0e38f;  // reference of an empty adjoint sum
// Segments per block: their records and adjoint sums are combined in shared memory, and the
// look-backs walk over groups of this many segments.
constexpr int kGroupSegs = 4;
constexpr int kGroupThreads = kGroupSegs * kThreads;
// R's per-position values: [kGroupSegs][kSeg][3][kThreads] floats, each thread its own column
constexpr size_t kGradSmem = (size_t)kGroupSegs * kSeg * 3 * kThreads * sizeof(float);

struct Adj {
    float x, y, xp, yp, r;  // X, Y, X', Y' relative to 2^{-r}
};

__device__ __forceinline__ Adj adj_empty() { return Adj{0.f, 0.f, 0.f, 0.f, kRNone}; }

// Forward recurrence state: (a, b) relative to 2^{anc - n w2} (base 2), the record convention.
struct FwdState {
    float a, bb, anc, n;
};

// What the adjoint needs of one output: its reference exponent q (base 2), 1 / Dn with
// D = Dn 2^q, and y.
struct FwdOut {
    float q, rd, y;
};

// One forward step: the output (when OUT) from the state before the token, then the token
// folded in (decay by counting, re-anchor on a new maximum).
template <bool OUT>
__device__ __forceinline__ void fwd_step(FwdState& s, float k2, float vt, float u2, float w2, FwdOut& o) {
    if (OUT) {
        const float p = fmaf(-s.n, w2, s.anc);
        const float uk = u2 + k2;
        const float e = ex2(-fabsf(p - uk));  // the other weight is exactly 1
        const bool cur = uk > p;
        const float e1 = cur ? e : 1.f, e2 = cur ? 1.f : e;
        o.q = fmaxf(p, uk);
        o.rd = rcp(fmaf(e1, s.bb, e2));
        o.y = fmaf(e1, s.a, e2 * vt) * o.rd;
    }
    // fold the token in without a branch (the loads of later steps stay ahead of this):
    // a new maximum re-anchors on k2 and scales the history, else the token is scaled
    const float pn = fmaf(-(s.n + 1.f), w2, s.anc);
    const bool nw = k2 > pn;
    const float f = ex2(-fabsf(pn - k2));
    s.a = fmaf(f, nw ? s.a : vt, nw ? vt : s.a);
    s.bb = fmaf(f, nw ? s.bb : 1.f, nw ? 1.f : s.bb);
    s.anc = nw ? k2 : s.anc;
    s.n = nw ? 0.f : s.n + 1.f;
}

// One adjoint step at a position (walking right to left): the position's gradients from the
// sums over later outputs, then its own output's terms added and the rest decayed.
__device__ __forceinline__ void adj_step(Adj& s, float k2, float vt, float g, const FwdOut& o, float u2, float w2,
                                         float& gk_out, float& gv_out, float& sgw, float& sgu) {
    const float cur = ex2(u2 + k2 - o.q) * o.rd;  // alpha_t / D_t
    const float ek = ex2(k2 - s.r);               // e^{k_t} 2^{-r} (0 for an empty sum)
    const float gc = g * cur;
    gv_out = fmaf(ek, s.x, gc);
    gk_out = fmaf(ek, fmaf(vt, s.x, -s.y), gc * (vt - o.y));
    sgu = fmaf(gc, vt - o.y, sgu);
    sgw = fmaf(-ek, fmaf(vt, s.xp, -s.yp), sgw);
    const float rn = fminf(o.q, s.r + w2);
    const float sn = ex2(rn - o.q) * o.rd * g;  // gy_t / D_t in the new frame
    const float so = ex2(rn - s.r - w2);        // e^{-w} and the change of frame
    s.xp = (s.xp + s.x) * so;
    s.yp = (s.yp + s.y) * so;
    s.x = fmaf(s.x, so, sn);
    s.y = fmaf(s.y, so, sn * o.y);
    s.r = rn;
}

// A segment's local adjoint sums at its left edge, accumulated left to right.  Term j (the
// segment's j-th output) is gy/D e^{-j w} = (g rd) 2^{-(q + j w2)}; the sums are held relative
// to 2^{-R} with R = Rq + Rj w2 the smallest term exponent so far, so each rescaling factor
// is <= 1 and the exponent difference is formed without the large j w2 rounded on its own.
struct LocalSums {
    float x, y, xp, yp, Rq, Rj;
    __device__ __forceinline__ void add(float jf, float g, const FwdOut& o, float w2) {
        const float d = fmaf(jf - Rj, w2, o.q - Rq);  // this term's exponent minus R
        const float e = ex2(-fabsf(d));
        const bool lower = d < 0.f;                   // the new term is the larger: new frame
        const float fo = lower ? e : 1.f, fn = lower ? 1.f : e;
        Rq = lower ? o.q : Rq;
        Rj = lower ? jf : Rj;
        const float m = g * o.rd * fn;
        const float my = m * o.y;
        x = fmaf(x, fo, m);
        y = fmaf(y, fo, my);
        xp = fmaf(xp, fo, jf * m);
        yp = fmaf(yp, fo, jf * my);
    }
};

// A block's loads are volatile asm (kept in program order) and each loaded value passes through
// an empty volatile asm after the last of them, so all of a block's loads are in flight before
// its first step is computed.  The inputs are read-only for the whole launch.
__device__ __forceinline__ float ld_in(const float* p) {
    float x;
    asm volatile("ld.global.nc.f32 %0, [%1];" : "=f"(x) : "l"(p));
    return x;
}
__device__ __forceinline__ void hold(float& x) { asm volatile("" : "+f"(x)); }

// Workspace header of the backward: the reverse pass's ticket and completion counters and the
// launch epoch that tags its published sums (advanced by each launch's last block).
struct BwdHeader {
    uint32_t ticket, done, epoch;        // the reverse pass (R)
    uint32_t error;                      // first give-up of either pass
    uint32_t ticket_f, done_f, epoch_f;  // the forward pass (A)
    uint32_t pad[9];
};
constexpr size_t kBwdHeaderBytes = sizeof(BwdHeader);
static_assert(kBwdHeaderBytes == 64, "header size");

// Per-block event trace (profiling builds only): compiled with -DWKV_TRACE, each block stamps
// %globaltimer at its phase boundaries into the buffer registered with wkv_bwd_trace_set_buffer
// ([2][units][8] u64: the forward pass's blocks, then the reverse pass's, indexed by ticket;
// slot 7 the SM id); normal builds define the hook away.
#ifdef WKV_TRACE
static __device__ unsigned long long* g_bwd_trace = nullptr;
__device__ __forceinline__ void bwd_trace(int pass, int64_t units, int64_t unit, int ev) {
    if (!g_bwd_trace || threadIdx.x != 0) return;
    unsigned long long t;
    asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
    unsigned long long* p = g_bwd_trace + ((int64_t)pass * units + unit) * 8;
    p[ev] = t;
    if (ev == 0) {
        unsigned sm;
        asm volatile("mov.u32 %0, %smid;" : "=r"(sm));
        p[7] = sm;
    }
}
#define BWD_TRACE(pass, unit, ev) bwd_trace(pass, (int64_t)gridDim.x, unit, ev)
#else
#define BWD_TRACE(pass, unit, ev) ((void)0)
#endif

struct BwdArgs {
    int64_t B, T, C, P;  // P segments of kSeg steps (the last may be shorter)
    const float *w, *u, *k, *v, *gy;
    float *gk, *gv, *gw, *gu;
    float* fs;           // [4][B][P][C] the segments' starting states
    uint64_t* fslots;    // [B][P][4][C] tagged words: a segment's forward record, later the
                         // state at its end (the inclusive record)
    uint64_t* slots;     // [B][P][5][C] tagged words: a segment's local adjoint sums, later what
                         // leaves it to the left (the inclusive sums)
    BwdHeader* hdr;
    uint32_t* dev_err;   // the library's device-wide error word
    uint32_t spin_limit;
};

__device__ __forceinline__ int64_t seg_index(const BwdArgs& a, int64_t b, int64_t j, int64_t c) {
    return (b * a.P + j) * a.C + c;
}

__device__ __forceinline__ FwdState load_state(const BwdArgs& a, int64_t si) {
    const int64_t SP = a.B * a.P * a.C;
    return FwdState{a.fs[si], a.fs[SP + si], a.fs[2 * SP + si], a.fs[3 * SP + si]};
}

// Runs the forward over positions [t0, t1) of one channel (element offset `base` + t C),
// loads issued kBlk steps at a time; `visit(i, out, g)` sees each output (i = t - t0) with its
// gy when WITH_G.
template <bool OUT, bool WITH_G, class Visit>
__device__ __forceinline__ void forward_span(const BwdArgs& a, int64_t base, int64_t t0, int64_t t1, FwdState& s,
                                             float u2, float w2, Visit&& visit) {
    FwdOut o{0.f, 0.f, 0.f};
    int64_t t = t0;
    for (; t + kBlk <= t1; t += kBlk) {
        float kb[kBlk], vb[kBlk], gb[kBlk];
#pragma unroll
        for (int i = 0; i < kBlk; ++i) {
            kb[i] = ld_in(a.k + base + (t + i) * a.C);
            vb[i] = ld_in(a.v + base + (t + i) * a.C);
            if (WITH_G) gb[i] = ld_in(a.gy + base + (t + i) * a.C);
        }
#pragma unroll
        for (int i = 0; i < kBlk; ++i) {
            hold(kb[i]);
            hold(vb[i]);
            if (WITH_G) hold(gb[i]);
        }
#pragma unroll
        for (int i = 0; i < kBlk; ++i) {
            fwd_step<OUT>(s, kb[i] * kLog2e, vb[i], u2, w2, o);
            if (OUT) visit((int)(t - t0) + i, o, WITH_G ? gb[i] : 0.f);
        }
    }
    for (; t < t1; ++t) {
        const int64_t at = base + t * a.C;
        fwd_step<OUT>(s, a.k[at] * kLog2e, a.v[at], u2, w2, o);
        if (OUT) visit((int)(t - t0), o, WITH_G ? a.gy[at] : 0.f);
    }
}

// Published records, one per (sequence, group of kGroupSegs segments, channel): the forward
// pass's record has four 64-bit words, (a | tag), (b | tag), (anc | tag), (n | tag), the
// reverse pass's adjoint sums five, (x, y, x', y', r); each word holds the value's bits in its
// low half and the launch epoch with the record's kind (1 the group's own record, 2 inclusive:
// everything before it, or after it, folded in) in its high half.  Aligned 64-bit accesses are
// single-copy atomic, so a reader that finds one tag in all the words holds one consistent
// record: no fence and no flag.  The group's own record is overwritten by the inclusive one
// (same thread, word by word), so a reader may catch mixed tags and then reads again.  Words
// are stored word-major per (sequence, group), so a warp's access to one word of 32 channels
// is contiguous.
template <int NW>
__device__ __forceinline__ void slot_publish(uint64_t* p, int64_t C, const float (&f)[NW], uint32_t tag) {
#pragma unroll
    for (int i = 0; i < NW; ++i) st_relaxed_u64(p + i * C, ((uint64_t)tag << 32) | __float_as_uint(f[i]));
}

// 2 inclusive, 1 the group's own record, 0 nothing usable yet
template <int NW>
__device__ __forceinline__ int slot_read(const uint64_t* p, int64_t C, uint32_t tag_loc, uint32_t tag_incl,
                                         float (&f)[NW]) {
    uint64_t wd[NW];
#pragma unroll
    for (int i = 0; i < NW; ++i) wd[i] = ld_relaxed_u64(p + i * C);
    const uint32_t t0 = (uint32_t)(wd[0] >> 32);
    bool same = t0 == tag_loc || t0 == tag_incl;
#pragma unroll
    for (int i = 1; i < NW; ++i) same = same && (uint32_t)(wd[i] >> 32) == t0;
    if (!same) return 0;
#pragma unroll
    for (int i = 0; i < NW; ++i) f[i] = __uint_as_float((uint32_t)wd[i]);
    return t0 == tag_incl ? 2 : 1;
}

__device__ __forceinline__ int64_t num_groups(const BwdArgs& a) { return (a.P + kGroupSegs - 1) / kGroupSegs; }

__device__ __forceinline__ float span_len(const BwdArgs& a, int64_t j0, int64_t j1) {  // steps of segments [j0, j1)
    return j1 > j0 ? (float)(min64(a.T, j1 * kSeg) - j0 * kSeg) : 0.f;
}

__device__ __forceinline__ void give_up(const BwdArgs& a) {
    atomicCAS(&a.hdr->error, kDevOk, (uint32_t)kDevTimeoutCarry);
    atomicCAS(a.dev_err, kDevOk, (uint32_t)kDevTimeoutCarry);
}

// A: groups of kGroupSegs segments in time order (an atomic ticket hands the first groups out
// first), one block of kGroupSegs x 128 threads per (group, sequence, channel block): each
// segment's forward from the empty state gives its record; the block folds its segments'
// records in shared memory; a decoupled look-back over the earlier groups of the channel (each
// a smaller ticket) gives the group's starting state, from which every segment's starting
// state follows and is written; the state at the group's end is published for later groups.
// gw, gu are zeroed here for R's atomics.
__global__ void __launch_bounds__(kGroupThreads) bwd_seg_starts(BwdArgs a, int64_t cx) {
    __shared__ Rec s_rec[kGroupSegs][kThreads];  // each segment's record, then its in-group prefix
    __shared__ Rec s_carry[kThreads];            // the state entering the group
    __shared__ uint32_t s_ticket, s_epoch;
    const int tid = threadIdx.x, tc = tid % kThreads, gs = tid / kThreads;
    if (tid == 0) {
        s_ticket = atomicAdd(&a.hdr->ticket_f, 1u);
        s_epoch = (*reinterpret_cast<volatile uint32_t*>(&a.hdr->epoch_f) + 1u) & 0x3FFFFFFFu;
    }
    __syncthreads();
    BWD_TRACE(0, s_ticket, 0);
    const int64_t unit = s_ticket;
    const uint32_t epoch30 = s_epoch;
    const uint32_t tag_loc = (epoch30 << 2) | 1u, tag_incl = (epoch30 << 2) | 2u;
    const int64_t per_grp = a.B * cx, NG = num_groups(a);
    const int64_t J = unit / per_grp;
    const int64_t b = (unit % per_grp) / cx, cb = unit % cx;
    const int64_t c = cb * kThreads + tc;
    const int64_t j = J * kGroupSegs + gs;
    const bool chan = unit < NG * per_grp && c < a.C;
    const bool live = chan && j < a.P;
    const float w2 = chan ? a.w[c] * kLog2e : 0.f;
    if (live) {
        if (b == 0 && j == 0) {  // R accumulates into these
            a.gw[c] = 0.f;
            a.gu[c] = 0.f;
        }
        const float u2 = a.u[c] * kLog2e;
        FwdState st{0.f, 0.f, kPEmpty, 0.f};
        forward_span<false, false>(a, b * a.T * a.C + c, j * kSeg, min64(a.T, (j + 1) * kSeg), st, u2, w2,
                                   [](int, const FwdOut&, float) {});
        s_rec[gs][tc] = Rec{st.a, st.bb, st.anc, st.n};
        BWD_TRACE(0, s_ticket, 1);
    } else {
        s_rec[gs][tc] = rec_identity();
    }
    __syncthreads();
    BWD_TRACE(0, s_ticket, 2);
    if (gs == 0 && chan) {
        // the group's segments folded in time order; each slot keeps its in-group prefix
        Rec agg = rec_identity();
#pragma unroll
        for (int g = 0; g < kGroupSegs; ++g) {
            const Rec r = s_rec[g][tc];
            s_rec[g][tc] = agg;
            const int64_t jg = J * kGroupSegs + g;
            if (jg < a.P) agg = rec_combine(agg, r, span_len(a, jg, jg + 1), w2);
        }
        uint64_t* my = a.fslots + (b * NG + J) * 4 * a.C + c;
        Rec run = rec_identity();  // the earlier groups, folded newest first
        if (J == 0) {
            if (NG > 1) slot_publish<4>(my, a.C, {agg.a, agg.b, agg.anc, agg.n}, tag_incl);
        } else {
            slot_publish<4>(my, a.C, {agg.a, agg.b, agg.anc, agg.n}, tag_loc);
            float span = 0.f;
            int64_t m = J - 1;
            bool done = false;
            uint32_t nap = 32;
            for (uint32_t it = 0; it <= a.spin_limit && !done; ++it) {
                float f[4];
                const int kind = slot_read<4>(a.fslots + (b * NG + m) * 4 * a.C + c, a.C, tag_loc, tag_incl, f);
                if (kind == 0) {
                    __nanosleep(nap);
                    nap = nap < 512 ? nap * 2 : 512;
                    continue;
                }
                nap = 32;
                run = rec_combine(Rec{f[0], f[1], f[2], f[3]}, run, span, w2);
                if (kind == 2) {
                    done = true;
                } else {
                    span += (float)(kGroupSegs * kSeg);  // every group before the last is whole
                    if (--m < 0) done = true;
                }
            }
            if (!done) give_up(a);  // go on with what is there (the gradients are then invalid)
            BWD_TRACE(0, s_ticket, 3);
            if (J + 1 < NG) {
                const Rec inc = rec_combine(run, agg, span_len(a, J * kGroupSegs, (J + 1) * kGroupSegs), w2);
                slot_publish<4>(my, a.C, {inc.a, inc.b, inc.anc, inc.n}, tag_incl);
            }
        }
        s_carry[tc] = run;
    }
    __syncthreads();
    BWD_TRACE(0, s_ticket, 4);
    if (live) {
        // this segment's starting state: the group's, then the group's segments before it
        const Rec st = rec_combine(s_carry[tc], s_rec[gs][tc], span_len(a, J * kGroupSegs, j), w2);
        const int64_t si = seg_index(a, b, j, c), SP = a.B * a.P * a.C;
        a.fs[si] = st.a;
        a.fs[SP + si] = st.b;
        a.fs[2 * SP + si] = st.anc;
        a.fs[3 * SP + si] = st.n;
    }
    BWD_TRACE(0, s_ticket, 5);
    __syncthreads();
    if (tid == 0) {
        __threadfence();
        const uint32_t finished = atomicAdd(&a.hdr->done_f, 1u) + 1u;
        if (finished == gridDim.x) {
            atomicExch(&a.hdr->ticket_f, 0u);
            atomicExch(&a.hdr->done_f, 0u);
            atomicExch(&a.hdr->epoch_f, epoch30);
        }
    }
}

// What leaves a span of len steps to its left: its local sums plus the sums entering it from
// the right carried across it (X decays by e^{-w len}; X' also gains len X).  Spans compose
// associatively: (A then B) leaves adj_compose(loc_A, loc_B, len_A) given nothing from the right.
__device__ __forceinline__ Adj adj_compose(const Adj& loc, const Adj& in, float len, float w2) {
    const float rin = in.r + len * w2;
    const float rn = fminf(loc.r, rin);
    const float fl = ex2(rn - loc.r), fi = ex2(rn - rin);
    Adj out;
    out.x = fmaf(in.x, fi, loc.x * fl);
    out.y = fmaf(in.y, fi, loc.y * fl);
    out.xp = fmaf(fmaf(len, in.x, in.xp), fi, loc.xp * fl);
    out.yp = fmaf(fmaf(len, in.y, in.yp), fi, loc.yp * fl);
    out.r = rn;
    return out;
}

// R: groups in reverse time order, one block of kGroupSegs x 128 threads per (group, sequence,
// channel block): each segment's forward from its starting state keeps its per-position
// values in shared memory while it accumulates its local adjoint sums; the block composes its
// segments' sums right to left; a decoupled look-back over the later groups of the channel
// (each a smaller ticket) gives the sums entering the group; what leaves it is published for
// earlier groups; each segment's incoming sums follow, and its adjoint pass writes gk, gv and
// adds its gw, gu partials.
__global__ void __launch_bounds__(kGroupThreads) bwd_seg_reverse(BwdArgs a, int64_t cx) {
    extern __shared__ float sm[];               // [kGroupSegs][kSeg][3][kThreads]: q, 1 / Dn, y
    __shared__ Adj s_in[kGroupSegs][kThreads];  // each segment's local sums, then its in-group incoming
    __shared__ Adj s_gin[kThreads];             // the sums entering the group from its right
    __shared__ uint32_t s_ticket, s_epoch;
    const int tid = threadIdx.x, tc = tid % kThreads, gs = tid / kThreads;
    if (tid == 0) {
        s_ticket = atomicAdd(&a.hdr->ticket, 1u);
        s_epoch = (*reinterpret_cast<volatile uint32_t*>(&a.hdr->epoch) + 1u) & 0x3FFFFFFFu;
    }
    __syncthreads();
    BWD_TRACE(1, s_ticket, 0);
    const int64_t unit = s_ticket;
    const uint32_t epoch30 = s_epoch;
    const uint32_t tag_loc = (epoch30 << 2) | 1u, tag_incl = (epoch30 << 2) | 2u;
    // tickets hand out the last groups first, then (sequence, channel block) within a group
    const int64_t per_grp = a.B * cx, NG = num_groups(a);
    const int64_t J = NG - 1 - unit / per_grp;
    const int64_t b = (unit % per_grp) / cx, cb = unit % cx;
    const int64_t c = cb * kThreads + tc;
    const int64_t j = J * kGroupSegs + gs;
    const bool chan = unit < NG * per_grp && c < a.C;
    const bool live = chan && j < a.P;
    const float w2 = chan ? a.w[c] * kLog2e : 0.f, u2 = chan ? a.u[c] * kLog2e : 0.f;
    const int64_t t0 = j * kSeg, t1 = min64(a.T, t0 + kSeg);
    const int64_t base = b * a.T * a.C + c;
    float* my_sm = sm + (size_t)gs * kSeg * 3 * kThreads;
    if (live) {
        // forward from the starting state: per-position values kept, local sums accumulated
        FwdState fsd = load_state(a, seg_index(a, b, j, c));
        LocalSums ls{0.f, 0.f, 0.f, 0.f, kRNone, 0.f};
        forward_span<true, true>(a, base, t0, t1, fsd, u2, w2, [&](int i, const FwdOut& o, float g) {
            my_sm[(i * 3 + 0) * kThreads + tc] = o.q;
            my_sm[(i * 3 + 1) * kThreads + tc] = o.rd;
            my_sm[(i * 3 + 2) * kThreads + tc] = o.y;
            ls.add((float)i, g, o, w2);
        });
        s_in[gs][tc] = Adj{ls.x, ls.y, ls.xp, ls.yp, fmaf(ls.Rj, w2, ls.Rq)};
        BWD_TRACE(1, s_ticket, 1);
    } else {
        s_in[gs][tc] = adj_empty();
    }
    __syncthreads();
    BWD_TRACE(1, s_ticket, 2);
    if (gs == 0 && chan) {
        // the group's segments composed right to left; each slot keeps what enters its segment
        // from the group's later segments
        Adj run = adj_empty();
#pragma unroll
        for (int g = kGroupSegs - 1; g >= 0; --g) {
            const Adj loc = s_in[g][tc];
            s_in[g][tc] = run;
            const int64_t jg = J * kGroupSegs + g;
            if (jg < a.P) run = adj_compose(loc, run, span_len(a, jg, jg + 1), w2);
        }
        uint64_t* my = a.slots + (b * NG + J) * 5 * a.C + c;
        // the sums entering the group: the later groups' composed, nearest first, until one that
        // already holds everything to its right (or the sequence's end)
        Adj gin = adj_empty();
        if (J + 1 < NG) {
            slot_publish<5>(my, a.C, {run.x, run.y, run.xp, run.yp, run.r}, tag_loc);
            Adj acc = adj_empty();
            float span = 0.f;
            int64_t m = J + 1;
            bool done = false;
            uint32_t nap = 32;
            for (uint32_t it = 0; it <= a.spin_limit && !done; ++it) {
                float f[5];
                const int kind = slot_read<5>(a.slots + (b * NG + m) * 5 * a.C + c, a.C, tag_loc, tag_incl, f);
                if (kind == 0) {
                    __nanosleep(nap);
                    nap = nap < 512 ? nap * 2 : 512;
                    continue;
                }
                nap = 32;
                const Adj rec{f[0], f[1], f[2], f[3], f[4]};
                if (kind == 2) {
                    gin = adj_compose(acc, rec, span, w2);
                    done = true;
                } else {
                    acc = adj_compose(acc, rec, span, w2);
                    span += span_len(a, m * kGroupSegs, (m + 1) * kGroupSegs);
                    if (++m >= NG) {
                        gin = acc;
                        done = true;
                    }
                }
            }
            if (!done) {  // gave up: go on with what is there (the gradients are then invalid)
                give_up(a);
                gin = acc;
            }
            BWD_TRACE(1, s_ticket, 3);
        }
        if (J > 0) {
            const Adj out = adj_compose(run, gin, span_len(a, J * kGroupSegs, (J + 1) * kGroupSegs), w2);
            slot_publish<5>(my, a.C, {out.x, out.y, out.xp, out.yp, out.r}, tag_incl);
        }
        s_gin[tc] = gin;
    }
    __syncthreads();
    BWD_TRACE(1, s_ticket, 4);
    if (live) {
        // the sums entering this segment: its group's later segments', with the group's own
        // incoming sums carried across them
        Adj st = adj_compose(s_in[gs][tc], s_gin[tc], span_len(a, j + 1, (J + 1) * kGroupSegs), w2);
        float sgw = 0.f, sgu = 0.f;
        auto step = [&](int64_t t, float kt, float vt, float g) {
            const int i = (int)(t - t0);
            const FwdOut o{my_sm[(i * 3 + 0) * kThreads + tc], my_sm[(i * 3 + 1) * kThreads + tc],
                           my_sm[(i * 3 + 2) * kThreads + tc]};
            float gk, gv;
            adj_step(st, kt * kLog2e, vt, g, o, u2, w2, gk, gv, sgw, sgu);
            a.gk[base + t * a.C] = gk;
            a.gv[base + t * a.C] = gv;
        };
        int64_t t = t1;
        for (; t - kBlk >= t0; t -= kBlk) {
            float kb[kBlk], vb[kBlk], gb[kBlk];
#pragma unroll
            for (int i = 0; i < kBlk; ++i) {
                const int64_t at = base + (t - 1 - i) * a.C;
                kb[i] = a.k[at];
                vb[i] = a.v[at];
                gb[i] = a.gy[at];
            }
#pragma unroll
            for (int i = 0; i < kBlk; ++i) step(t - 1 - i, kb[i], vb[i], gb[i]);
        }
        for (; t > t0; --t) {
            const int64_t at = base + (t - 1) * a.C;
            step(t - 1, a.k[at], a.v[at], a.gy[at]);
        }
        BWD_TRACE(1, s_ticket, 5);
        atomicAdd(&a.gw[c], sgw);
        atomicAdd(&a.gu[c], sgu);
    }
    // the launch's last block resets the counters and advances the epoch
    BWD_TRACE(1, s_ticket, 6);
    __syncthreads();
    if (tid == 0) {
        __threadfence();
        const uint32_t finished = atomicAdd(&a.hdr->done, 1u) + 1u;
        if (finished == gridDim.x) {
            atomicExch(&a.hdr->ticket, 0u);
            atomicExch(&a.hdr->done, 0u);
            atomicExch(&a.hdr->epoch, epoch30);
        }
    }
}

}  // namespace

#ifdef WKV_TRACE
extern "C" void wkv_bwd_trace_set_buffer(void* buf) {
    unsigned long long* p = static_cast<unsigned long long*>(buf);
    cudaMemcpyToSymbol(g_bwd_trace, &p, sizeof(p));
}
#endif

int64_t backward_segments(int64_t T) { return (T + kSeg - 1) / kSeg; }

size_t backward_workspace_bytes(int64_t B, int64_t T, int64_t C) {
    const int64_t P = backward_segments(T);
    const size_t bpc = (size_t)B * (size_t)P * (size_t)C;
    const size_t bgc = (size_t)B * (size_t)((P + kGroupSegs - 1) / kGroupSegs) * (size_t)C;
    return kBwdHeaderBytes + bpc * 4 * sizeof(float) + bgc * 9 * sizeof(uint64_t);
}

cudaError_t launch_backward(int64_t B, int64_t T, int64_t C, const float* w, const float* u, const float* k,
                            const float* v, const float* gy, float* gk, float* gv, float* gw, float* gu, void* ws,
                            cudaStream_t s) {
    if (B == 0 || T == 0) {  // no position: the per-channel gradients are zero
        cudaError_t e = cudaMemsetAsync(gw, 0, (size_t)C * sizeof(float), s);
        if (e != cudaSuccess) return e;
        return cudaMemsetAsync(gu, 0, (size_t)C * sizeof(float), s);
    }
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
    const int64_t SP = B * a.P * C;
    unsigned char* base = static_cast<unsigned char*>(ws);
    a.hdr = reinterpret_cast<BwdHeader*>(base);
    a.fs = reinterpret_cast<float*>(base + kBwdHeaderBytes);
    const int64_t NG = (a.P + kGroupSegs - 1) / kGroupSegs;
    a.fslots = reinterpret_cast<uint64_t*>(base + kBwdHeaderBytes + (size_t)SP * 4 * sizeof(float));
    a.slots = a.fslots + (size_t)(B * NG * C) * 4;
    a.dev_err = device_status_word();
    if (!a.dev_err) return cudaErrorInvalidValue;
    a.spin_limit = kSpinLimitDefault;
    const int64_t cx = (C + kThreads - 1) / kThreads;
    const int64_t units = NG * B * cx;
    if (units > INT32_MAX) return cudaErrorInvalidValue;
    static uint64_t attr_done = 0;  // per device; set once so captured launches issue no attribute call
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev >= 64 || !(attr_done & (1ull << dev))) {
        e = cudaFuncSetAttribute(bwd_seg_reverse, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kGradSmem);
        if (e != cudaSuccess) return e;
        if (dev < 64) attr_done |= 1ull << dev;
    }
    bwd_seg_starts<<<(unsigned)units, kGroupThreads, 0, s>>>(a, cx);
    bwd_seg_reverse<<<(unsigned)units, kGroupThreads, kGradSmem, s>>>(a, cx);
    return cudaGetLastError();
}

}  // namespace wkvb
