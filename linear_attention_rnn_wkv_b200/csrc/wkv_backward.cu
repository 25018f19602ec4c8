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
// same sums weighted by (t-1-i).  Over a span of len positions entered with (X, X') from its
// right they compose as X_start = X_local + e^{-w len} X, X'_start = X'_local + e^{-w len}
// (X' + len X), where a span's local sums at its left edge are
// X_local = sum_{t in span} e^{-(t-t0) w} gy_t / D_t and X'_local the same weighted by (t - t0).
//
// The fixed frame.  Inside a span of L steps (local index i), with E_i = e^{k_i + i w} and a
// frame F = 2^G, every quantity of the span is a prefix or a suffix sum of per-position terms:
// the decay factors cancel out of y_t, and out of e^{k_i} X_i, exactly as in the forward's
// re-scan ("Why it collapses into a recurrence": the telescoping of the decay).  With
// E~ = E / F, c = e^{w-u}, the history's B~_h, A~_h and D^_t = B~_t + E~_t / c (B~_t the
// history plus sum_{j<t} E~_j, likewise A~_t with v_j):
//   y_t  = (A~_t + E~_t v_t / c) / D^_t,   g~_t = gy_t / D^_t
//   gv_i = E~_i (g~_i / c + S_i),  gk_i = E~_i (g~_i (v_i - y_i) / c + v_i S_i - S^y_i)
//   gu  += E~_i g~_i (v_i - y_i) / c,  gw -= E~_i (v_i S'_i - S'^y_i)
// with S_i = sum_{t>i} g~_t (plus the sums entering the span, moved into the frame), S^y_i the
// same with g~_t y_t, and S'_{i-1} = S'_i + S_i.  So one exponential and one reciprocal per
// position and no state chain but plain adds.  The frame holds when the span's exponents (its
// keys', its history's and the bonus's) lie within kFrameSpan of one another (G their
// midpoint: every value within 2^{+-80}); a lane whose span does not fit takes the per-step
// stabilised recurrence instead (the same sums, each step re-anchored on its own maximum).
//
// Time-parallel in segments of kSeg steps, one thread per (b, c, segment), groups of kGroupSegs
// segments per block, one launch whose blocks take work items by an atomic ticket so that every
// wait is on a smaller ticket:
//   A  (the first tickets) groups 0 .. NG-2 in time order: each segment's forward record from
//      the empty state, the group's folded in shared memory and published; a decoupled
//      look-back over the earlier groups gives the group's inclusive record, published for the
//      later groups;
//   R  (the rest) all groups in reverse time order: the block recomputes its segments' records,
//      takes the state entering the group by the same look-back over A's records, and each
//      segment's starting state from the in-group prefix; each segment runs its forward in its
//      frame (outputs kept in registers) and publishes its local adjoint sums; the block composes
//      them, publishes the group's, and a decoupled look-back towards the end of the sequence
//      gives the sums entering the group; each segment then runs its adjoint pass -> gk, gv.
//      Each block adds its gw, gu partials with atomics, once the zeros written by A's first
//      block of its channels are visible (that block publishes its record after them).
// k, v are read by A and again by R (A's last groups are R's first, so much of that second read
// is served by the L2), gy once, gk, gv written once.  Nothing per position is stored in global
// memory; a block's inputs are staged in shared memory (cp.async), so a thread holds only its
// segment's outputs in registers and four blocks fit on an SM.
#include "wkv_device.cuh"
#include "wkv_internal.h"
#include "wkv_pipe_common.cuh"

namespace wkvb {
namespace {

constexpr int kSeg = 16;                            // time steps per segment (one thread)
constexpr int kGroupSegs = 8;                       // segments per group: a block's time span
constexpr int kCh = 32;                             // channels per block (a warp's lanes)
constexpr int kThreads = kGroupSegs * kCh;          // warp s works on segment s of the group
constexpr int kGroupSteps = kSeg * kGroupSegs;      // 128
constexpr float kRNone = 3.0e38f;                   // reference of an empty adjoint sum
constexpr float kFrameSpan = 160.f;                 // base-2 range one frame may hold

struct Adj {
    float x, y, xp, yp, r;  // X, Y, X', Y' relative to 2^{-r}
};

__device__ __forceinline__ Adj adj_empty() { return Adj{0.f, 0.f, 0.f, 0.f, kRNone}; }

// Scales the sums by a power of two so that the largest magnitude lies in [1, 2), moving the
// reference with it (exact), so composing two spans keeps the larger one's scale.
__device__ __forceinline__ Adj adj_normalize(Adj s) {
    const float mx = fmaxf(fmaxf(fabsf(s.x), fabsf(s.y)), fmaxf(fabsf(s.xp), fabsf(s.yp)));
    const int ex = (int)((__float_as_uint(mx) >> 23) & 0xffu) - 127;
    if (ex < -126 || ex > 126) return s;  // zero, or not finite: left as it is
    const float sc = __uint_as_float((uint32_t)(127 - ex) << 23);
    s.x *= sc;
    s.y *= sc;
    s.xp *= sc;
    s.yp *= sc;
    s.r -= (float)ex;
    return s;
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

// The per-step stabilised form (lanes whose span does not fit one frame).
// Forward recurrence state: (a, b) relative to 2^{anc - n w} (base 2), the record convention.
struct FwdState {
    float a, bb, anc, n;
};

// What the adjoint needs of one output: its reference exponent q (base 2), 1 / Dn with
// D = Dn 2^q, and y.
struct FwdOut {
    float q, rd, y;
};

// One forward step: the output from the state before the token, then the token folded in
// (decay by counting, re-anchor on a new maximum).
__device__ __forceinline__ void fwd_step(FwdState& s, float k2, float vt, float u2, float w2, FwdOut& o) {
    const float p = fmaf(-s.n, w2, s.anc);
    const float uk = u2 + k2;
    const float e = ex2(-fabsf(p - uk));  // the other weight is exactly 1
    const bool cur = uk > p;
    const float e1 = cur ? e : 1.f, e2 = cur ? 1.f : e;
    o.q = fmaxf(p, uk);
    o.rd = rcp(fmaf(e1, s.bb, e2));
    o.y = fmaf(e1, s.a, e2 * vt) * o.rd;
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

// A segment's local adjoint sums at its left edge in the per-step form, accumulated left to
// right.  Term j is gy/D e^{-j w} = (g rd) 2^{-(q + j w2)}; the sums are held relative to
// 2^{-R} with R = Rq + Rj w2 the smallest term exponent so far, so each rescaling factor is
// <= 1 and the exponent difference is formed without the large j w2 rounded on its own.
struct LocalSums {
    float x, y, xp, yp, Rq, Rj;
    __device__ __forceinline__ void add(float jf, float g, const FwdOut& o, float w2) {
        const float d = fmaf(jf - Rj, w2, o.q - Rq);
        const float e = ex2(-fabsf(d));
        const bool lower = d < 0.f;
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

// A block's inputs are staged in shared memory as tiles of [kGroupSteps][kCh] floats (the
// group's steps by the block's channels), thread (s, lane) owning rows s kSeg .. s kSeg + 15 of
// column lane: by three TMA tensor copies where rows are whole 16-byte units (zero-filled past
// T and C), else by 4-byte cp.async copies that each thread issues for its own elements (no
// registers held while they fly).
__device__ __forceinline__ void cp_async4(float* dst, const float* src) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ uint64_t ld_acquire_u64(const uint64_t* p) {
    uint64_t v;
    asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ void cp_async_wait_all() {
    asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
}

// Workspace header: one 64-bit word whose low half hands out the tickets and whose high half
// is the launch epoch that tags the published records; the block that takes the launch's last
// ticket resets the count and advances the epoch (every block has its ticket by then, and the
// next launch starts after this one ends).
struct BwdHeader {
    unsigned long long tk;
    uint32_t error;  // first give-up of a look-back
    uint32_t pad[13];
};
constexpr size_t kBwdHeaderBytes = sizeof(BwdHeader);
static_assert(kBwdHeaderBytes == 64, "header size");

// Per-block event trace (profiling builds only): compiled with -DWKV_TRACE, each block stamps
// %globaltimer at its phase boundaries into the buffer registered with wkv_bwd_trace_set_buffer
// ([tickets][16] u64: phase times, slot 8 the reverse look-back's polls, slot 15 the SM id);
// normal builds define the hook away.
#ifdef WKV_TRACE
static __device__ unsigned long long* g_bwd_trace = nullptr;
__device__ __forceinline__ void bwd_trace(int64_t unit, int ev) {
    if (!g_bwd_trace || threadIdx.x != 0) return;
    unsigned long long t;
    asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
    unsigned long long* p = g_bwd_trace + unit * 16;
    p[ev] = t;
    if (ev == 0) {
        unsigned sm;
        asm volatile("mov.u32 %0, %smid;" : "=r"(sm));
        p[15] = sm;
    }
}
__device__ __forceinline__ void bwd_trace_value(int64_t unit, int slot, unsigned long long v) {
    if (g_bwd_trace) g_bwd_trace[unit * 16 + slot] = v;
}
#define BWD_TRACE(unit, ev) bwd_trace(unit, ev)
#define BWD_TRACE_VALUE(unit, slot, v) bwd_trace_value(unit, slot, v)
#else
#define BWD_TRACE(unit, ev) ((void)0)
#define BWD_TRACE_VALUE(unit, slot, v) ((void)(v))
#endif

struct BwdArgs {
    int64_t B, T, C;
    int64_t NG, cx;      // groups of kGroupSteps steps; channel blocks of kCh
    int64_t UA;          // A's work items (groups 0 .. NG-2)
    uint32_t units;      // all work items (the grid)
    const float *w, *u, *k, *v, *gy;
    float *gk, *gv, *gw, *gu;
    uint64_t* fslots;    // [B][NG][4][C] tagged words: a group's forward record, later the state
                         // at its end (the inclusive record)
    uint64_t* slots;     // [B][NG][5][C] tagged words: a group's local adjoint sums, later what
                         // leaves it to the left (the inclusive sums)
    BwdHeader* hdr;
    uint32_t* dev_err;   // the library's device-wide error word
    uint32_t spin_limit;
};

// Published records, one per (sequence, group, channel): the forward record has four 64-bit
// words, (a | tag), (b | tag), (anc | tag), (n | tag), the adjoint sums five, (x, y, x', y', r);
// each word holds the value's bits in its low half and the launch epoch with the record's kind
// (1 the group's own record, 2 inclusive: everything before it, or after it, folded in) in its
// high half.  Aligned 64-bit accesses are single-copy atomic, so a reader that finds one tag in
// all the words holds one consistent record: no fence and no flag.  The group's own record is
// overwritten by the inclusive one (same thread, word by word), so a reader may catch mixed
// tags and then reads again.  Words are stored word-major per (sequence, group), so a warp's
// access to one word of 32 channels is contiguous.
template <int NW>
__device__ __forceinline__ void slot_publish(uint64_t* p, int64_t C, const float (&f)[NW], uint32_t tag) {
#pragma unroll
    for (int i = 0; i < NW; ++i) st_relaxed_u64(p + i * C, ((uint64_t)tag << 32) | __float_as_uint(f[i]));
}

template <int NW>
__device__ __forceinline__ void slot_load(const uint64_t* p, int64_t C, uint64_t (&wd)[NW]) {
#pragma unroll
    for (int i = 0; i < NW; ++i) wd[i] = ld_relaxed_u64(p + i * C);
}

// 2 inclusive, 1 the group's own record, 0 nothing usable yet
template <int NW>
__device__ __forceinline__ int slot_decode(const uint64_t (&wd)[NW], uint32_t tag_loc, uint32_t tag_incl,
                                           float (&f)[NW]) {
    const uint32_t t0 = (uint32_t)(wd[0] >> 32);
    bool same = t0 == tag_loc || t0 == tag_incl;
#pragma unroll
    for (int i = 1; i < NW; ++i) same = same && (uint32_t)(wd[i] >> 32) == t0;
    if (!same) return 0;
#pragma unroll
    for (int i = 0; i < NW; ++i) f[i] = __uint_as_float((uint32_t)wd[i]);
    return t0 == tag_incl ? 2 : 1;
}

template <int NW>
__device__ __forceinline__ int slot_read(const uint64_t* p, int64_t C, uint32_t tag_loc, uint32_t tag_incl,
                                         float (&f)[NW]) {
    uint64_t wd[NW];
    slot_load<NW>(p, C, wd);
    return slot_decode<NW>(wd, tag_loc, tag_incl, f);
}

__device__ __forceinline__ void give_up(const BwdArgs& a) {
    atomicCAS(&a.hdr->error, kDevOk, (uint32_t)kDevTimeoutCarry);
    atomicCAS(a.dev_err, kDevOk, (uint32_t)kDevTimeoutCarry);
}

__device__ __forceinline__ int seg_len(const BwdArgs& a, int64_t t0) {
    const int64_t r = a.T - t0;
    return r <= 0 ? 0 : (r >= kSeg ? kSeg : (int)r);
}

// The state entering group J of channel c: the records of the groups before it, folded newest
// first, until one that already holds everything before it (a decoupled look-back; each of
// those groups is a smaller ticket).  Empty for the first group.
__device__ __forceinline__ Rec fwd_lookback(const BwdArgs& a, int64_t b, int64_t J, int64_t c, float w2,
                                            uint32_t tag_loc, uint32_t tag_incl) {
    Rec run = rec_identity();
    float span = 0.f;
    int64_t m = J - 1;
    bool done = m < 0;
    uint32_t nap = 32;
    for (uint32_t it = 0; it <= a.spin_limit && !done; ++it) {
        float f[4];
        const int kind = slot_read<4>(a.fslots + (b * a.NG + m) * 4 * a.C + c, a.C, tag_loc, tag_incl, f);
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
            span += (float)kGroupSteps;  // every group before the last is whole
            if (--m < 0) done = true;
        }
    }
    if (!done) give_up(a);  // go on with what is there (the gradients are then invalid)
    return run;
}

// A segment's own forward record from the empty state, in the frame of its largest exponent:
// x_i = k_i log2 e + i w2 (base 2), value = (sum 2^{x_i - M} v_i, sum 2^{x_i - M}) relative
// to 2^{M - (len-1) w2}, i.e. anc = M and n = len - 1.  Terms far below M flush to zero, which
// the sums could not resolve anyway.  Also returns the smallest exponent m.
template <bool FULL>
__device__ __forceinline__ Rec seg_record(const float* sk, const float* sv, int len, float w2, float& M, float& m) {
    float xs[kSeg];
    M = -3.0e38f;
    m = 3.0e38f;
#pragma unroll
    for (int i = 0; i < kSeg; ++i) {
        if (FULL || i < len) {
            xs[i] = fmaf(sk[i * kCh], kLog2e, (float)i * w2);
            M = fmaxf(M, xs[i]);
            m = fminf(m, xs[i]);
        }
    }
    float sa = 0.f, sb = 0.f;
#pragma unroll
    for (int i = 0; i < kSeg; ++i) {
        if (FULL || i < len) {
            const float e = ex2(xs[i] - M);
            sa = fmaf(e, sv[i * kCh], sa);
            sb += e;
        }
    }
    return Rec{sa, sb, M, (float)(len - 1)};
}

// The forward over a segment in its frame G, from the history (ah, bh) already in the frame:
// outputs into ys, 2^{x_i - G} over the keys in sk, gy / D^ over gy in sg; returns the local
// adjoint sums (relative to 2^{-(G + w2)}: the term of position i is g~_i e^{(i-1) w} e^{-i w} / F).
template <bool FULL>
__device__ __forceinline__ Adj fwd_frame(float* sk, const float* sv, float* sg, float (&ys)[kSeg], int len, float G,
                                         float ic, float ah, float bh, float w2) {
    float A = ah, Bs = bh;
    float sx = 0.f, sy = 0.f, sxp = 0.f, syp = 0.f;
#pragma unroll
    for (int i = 0; i < kSeg; ++i) {
        if (FULL || i < len) {
            const float vt = sv[i * kCh];
            const float e = ex2(fmaf(sk[i * kCh], kLog2e, fmaf((float)i, w2, -G)));
            const float ec = e * ic;
            const float num = fmaf(ec, vt, A);
            const float rd = rcp(Bs + ec);
            const float y = num * rd;
            const float g = sg[i * kCh] * rd;
            A = fmaf(e, vt, A);
            Bs += e;
            sk[i * kCh] = e;
            sg[i * kCh] = g;
            ys[i] = y;
            const float gy = g * y;
            sx += g;
            sy += gy;
            sxp = fmaf((float)i, g, sxp);
            syp = fmaf((float)i, gy, syp);
        }
    }
    return Adj{sx, sy, sxp, syp, G + w2};
}

// The adjoint pass over a segment in its frame, right to left, from the sums entering it
// (already in the frame): gk, gv stored, gw, gu partials added.
template <bool FULL>
__device__ __forceinline__ void adj_frame(const BwdArgs& a, int64_t base, const float* se, const float* sv,
                                          const float* sg, const float (&ys)[kSeg], int len, float ic, float Xs,
                                          float Ys, float Xp, float Yp, float& sgw, float& sgu) {
#pragma unroll
    for (int i = kSeg - 1; i >= 0; --i) {
        if (FULL || i < len) {
            const float e = se[i * kCh], vt = sv[i * kCh], g = sg[i * kCh], y = ys[i];
            const float t1 = g * ic;
            const float gv = e * (t1 + Xs);
            const float td = t1 * (vt - y);
            const float gk = e * (fmaf(vt, Xs, td) - Ys);
            sgu = fmaf(td, e, sgu);
            sgw = fmaf(-e, fmaf(vt, Xp, -Yp), sgw);
            Xp += Xs;
            Yp += Ys;
            Xs += g;
            Ys = fmaf(g, y, Ys);
            a.gk[base + (int64_t)i * a.C] = gk;
            a.gv[base + (int64_t)i * a.C] = gv;
        }
    }
}

// The per-step forward over a segment from its starting state (lanes outside the frame):
// outputs into ys, and each output's q and 1 / Dn parked in this position's gk and gv (the
// same thread reads them back in its adjoint pass before it writes the gradients there);
// returns the local adjoint sums.
template <bool FULL>
__device__ __forceinline__ Adj fwd_steps(const BwdArgs& a, int64_t base, const float* sk, const float* sv,
                                         const float* sg, float (&ys)[kSeg], int len, const Rec& st, float u2,
                                         float w2) {
    FwdState s{st.a, st.b, st.anc, st.n};
    LocalSums ls{0.f, 0.f, 0.f, 0.f, kRNone, 0.f};
#pragma unroll
    for (int i = 0; i < kSeg; ++i) {
        if (FULL || i < len) {
            FwdOut o;
            fwd_step(s, sk[i * kCh] * kLog2e, sv[i * kCh], u2, w2, o);
            a.gk[base + (int64_t)i * a.C] = o.q;
            a.gv[base + (int64_t)i * a.C] = o.rd;
            ys[i] = o.y;
            ls.add((float)i, sg[i * kCh], o, w2);
        }
    }
    return Adj{ls.x, ls.y, ls.xp, ls.yp, fmaf(ls.Rj, w2, ls.Rq)};
}

template <bool FULL>
__device__ __forceinline__ void adj_steps(const BwdArgs& a, int64_t base, const float* sk, const float* sv,
                                          const float* sg, const float (&ys)[kSeg], int len, Adj st, float u2,
                                          float w2, float& sgw, float& sgu) {
#pragma unroll
    for (int i = kSeg - 1; i >= 0; --i) {
        if (FULL || i < len) {
            float* pk = a.gk + base + (int64_t)i * a.C;
            float* pv = a.gv + base + (int64_t)i * a.C;
            const FwdOut o{*pk, *pv, ys[i]};
            float gk, gv;
            adj_step(st, sk[i * kCh] * kLog2e, sv[i * kCh], sg[i * kCh], o, u2, w2, gk, gv, sgw, sgu);
            *pk = gk;
            *pv = gv;
        }
    }
}

// The sums entering group J from its right: the later groups' published sums composed,
// nearest first, until one that already holds everything to its right (or the sequence's end).
// wd holds the nearest later group's words, read before the group's own were composed.
__device__ __forceinline__ Adj adj_lookback(const BwdArgs& a, int b, int J, int c, float w2, uint32_t tag_loc,
                                            uint32_t tag_incl, uint64_t (&wd)[5], uint32_t& polls) {
    Adj acc = adj_empty(), gin = adj_empty();
    float span = 0.f;
    int64_t mg = J + 1;
    bool done = false;
    uint32_t nap = 32;
    for (uint32_t it = 0; it <= a.spin_limit && !done; ++it) {
        float f[5];
        if (it > 0) slot_load<5>(a.slots + ((int64_t)b * a.NG + mg) * 5 * a.C + c, a.C, wd);
        const int kind = slot_decode<5>(wd, tag_loc, tag_incl, f);
        ++polls;
        if (kind == 0) {
            __nanosleep(nap);
            nap = nap < 512 ? nap * 2 : 512;
            continue;
        }
        nap = 32;
        const Adj rg{f[0], f[1], f[2], f[3], f[4]};
        if (kind == 2) {
            gin = adj_compose(acc, rg, span, w2);
            done = true;
        } else {
            acc = adj_normalize(adj_compose(acc, rg, span, w2));
            span += (float)min64(a.T - mg * kGroupSteps, kGroupSteps);
            if (++mg >= a.NG) {
                gin = acc;
                done = true;
            }
        }
    }
    if (!done) {  // gave up: go on with what is there (the gradients are then invalid)
        give_up(a);
        gin = acc;
    }
    return adj_normalize(gin);
}

// Shared memory of a block: the three staged tiles, then the records (each segment's, then its
// starting state) overlaid by the adjoint sums (each segment's local sums, then its incoming
// sums: written only after every thread has read its starting state).
constexpr size_t kTileFloats = (size_t)kGroupSteps * kCh;
static_assert(kTileFloats == (size_t)kSeg * kThreads, "a tile holds one element per thread and step");
constexpr size_t kRecBytes = sizeof(Rec) * kGroupSegs * kCh, kAdjBytes = sizeof(Adj) * kGroupSegs * kCh;
constexpr size_t kSmemBytes = 3 * kTileFloats * sizeof(float) + (kRecBytes > kAdjBytes ? kRecBytes : kAdjBytes);

template <bool TMA>
__global__ void __launch_bounds__(kThreads, 4)
    bwd_kernel(BwdArgs a, const __grid_constant__ CUtensorMap tmk, const __grid_constant__ CUtensorMap tmv,
               const __grid_constant__ CUtensorMap tmg) {
    extern __shared__ __align__(128) float4 sm4[];
    float* sm = reinterpret_cast<float*>(sm4);
    Rec(*s_rec)[kCh] = reinterpret_cast<Rec(*)[kCh]>(sm + 3 * kTileFloats);
    Adj(*s_adj)[kCh] = reinterpret_cast<Adj(*)[kCh]>(sm + 3 * kTileFloats);
    __shared__ Adj s_gin[kCh];          // the sums entering the group from its right
    __shared__ float s_ys[kSeg * kCh];  // warp 0's outputs during the reverse look-back
    __shared__ uint32_t s_ticket, s_epoch;
    __shared__ __align__(8) uint64_t s_bar;  // the TMA copies' completion
    const int tid = threadIdx.x, lane = tid % kCh, seg = tid / kCh;
    float* sk = sm + seg * kSeg * kCh + lane;  // this thread's elements of k (then 2^{x - G}),
    float* sv = sk + kTileFloats;              // of v
    float* sg = sk + 2 * kTileFloats;          // of gy (then gy / D^)
    grid_dep_launch_dependents();
    if (TMA && tid == 0) {
        mbar_init(&s_bar, 1);
        fence_mbar_init();
    }
    grid_dep_wait();  // global memory only from here
    if (tid == 0) {
        const unsigned long long t = atomicAdd(&a.hdr->tk, 1ull);
        const uint32_t tk = (uint32_t)t, ep = (uint32_t)(t >> 32);
        if (tk == a.units - 1u) atomicExch(&a.hdr->tk, (unsigned long long)((ep + 1u) & 0x3FFFFFFFu) << 32);
        s_ticket = tk;
        s_epoch = ep & 0x3FFFFFFFu;
    }
    __syncthreads();
    const uint32_t ticket = s_ticket;
    BWD_TRACE(ticket, 0);
    const uint32_t tag_loc = (s_epoch << 2) | 1u, tag_incl = (s_epoch << 2) | 2u;
    // the work item (all indices below 2^31: the grid's blocks are)
    const bool isA = ticket < (uint32_t)a.UA;
    const uint32_t per = (uint32_t)(a.B * a.cx), cx = (uint32_t)a.cx, r = isA ? ticket : ticket - (uint32_t)a.UA;
    const int J = (int)(isA ? r / per : (uint32_t)a.NG - 1u - r / per);
    const int b = (int)((r % per) / cx), cb = (int)(r % cx);
    const int c = cb * kCh + lane;
    const bool chan = c < a.C;
    const int64_t t0 = J * kGroupSteps + (int64_t)seg * kSeg;
    const int len = chan ? seg_len(a, t0) : 0;
    const float w2 = chan ? a.w[c] * kLog2e : 0.f, u2 = chan ? a.u[c] * kLog2e : 0.f;
    const int64_t base = (b * a.T + t0) * a.C + c;

    // stage the block's tiles (k, v; gy for R)
    if (TMA) {
        if (tid == 0) {
            mbar_arrive_expect_tx(&s_bar, (uint32_t)((isA ? 2 : 3) * kTileFloats * sizeof(float)));
            const int x = (int)(cb * kCh), y = (int)(J * kGroupSteps), z = (int)b;
            tma_load_3d(sm, &tmk, x, y, z, &s_bar);
            tma_load_3d(sm + kTileFloats, &tmv, x, y, z, &s_bar);
            if (!isA) tma_load_3d(sm + 2 * kTileFloats, &tmg, x, y, z, &s_bar);
        }
    } else {
        for (int i = 0; i < len; ++i) {
            cp_async4(sk + i * kCh, a.k + base + (int64_t)i * a.C);
            cp_async4(sv + i * kCh, a.v + base + (int64_t)i * a.C);
            if (!isA) cp_async4(sg + i * kCh, a.gy + base + (int64_t)i * a.C);
        }
    }
    // while the copies fly: R's warp 0 takes the state entering the group (the look-back over
    // A's records); R's warp 1 waits until gw, gu have been zeroed: A's first block of the
    // channel block zeroes them, then (after a fence) publishes its record, which warp 1 reads
    // with acquire semantics; the block barriers then order warp 0's atomics after that read
    Rec gstart = rec_identity();
    if (isA) {
        if (seg == 0 && chan && J == 0 && b == 0) {  // published (after a fence) by this lane
            a.gw[c] = 0.f;
            a.gu[c] = 0.f;
        }
    } else {
        if (seg == 0) {
            if (chan) gstart = fwd_lookback(a, b, J, c, w2, tag_loc, tag_incl);
            if (lane == 0) BWD_TRACE(ticket, 9);
        } else if (seg == 1 && chan && a.NG > 1) {
            bool zeroed = false;
            for (uint32_t it = 0; it <= a.spin_limit && !zeroed; ++it) {
                zeroed = (uint32_t)(ld_acquire_u64(a.fslots + c) >> 32) == tag_incl;  // (b = 0, group 0) word 0
                if (!zeroed) __nanosleep(64);
            }
            if (!zeroed) give_up(a);
        }
    }
    if (TMA) {
        if (!mbar_wait(&s_bar, 0, a.spin_limit) && tid == 0) atomicCAS(a.dev_err, kDevOk, (uint32_t)kDevTimeoutCopy);
    } else {
        cp_async_wait_all();
    }
    BWD_TRACE(ticket, 10);
    float M = 0.f, m = 0.f;
    Rec rec = rec_identity();
    if (len == kSeg)
        rec = seg_record<true>(sk, sv, len, w2, M, m);
    else if (len > 0)
        rec = seg_record<false>(sk, sv, len, w2, M, m);
    s_rec[seg][lane] = rec;
    BWD_TRACE(ticket, 11);
    __syncthreads();
    BWD_TRACE(ticket, 1);

    if (isA) {
        // fold the group's segments, publish, look back, publish the inclusive record
        if (seg == 0 && chan) {
            Rec agg = rec_identity();
#pragma unroll
            for (int s = 0; s < kGroupSegs; ++s) {
                const int ls = seg_len(a, J * kGroupSteps + (int64_t)s * kSeg);
                if (ls > 0) agg = rec_combine(agg, s_rec[s][lane], (float)ls, w2);
            }
            uint64_t* my = a.fslots + ((int64_t)b * a.NG + J) * 4 * a.C + c;
            if (J == 0) {
                if (b == 0) __threadfence();  // the zeros of gw, gu before the record
                slot_publish<4>(my, a.C, {agg.a, agg.b, agg.anc, agg.n}, tag_incl);
            } else {
                slot_publish<4>(my, a.C, {agg.a, agg.b, agg.anc, agg.n}, tag_loc);
                const Rec run = fwd_lookback(a, b, J, c, w2, tag_loc, tag_incl);
                const Rec inc = rec_combine(run, agg, (float)kGroupSteps, w2);
                slot_publish<4>(my, a.C, {inc.a, inc.b, inc.anc, inc.n}, tag_incl);
            }
        }
        BWD_TRACE(ticket, 2);
        return;
    }
    // R: each segment's starting state from the group's
    if (seg == 0 && chan) {
        Rec run = gstart;
#pragma unroll
        for (int s = 0; s < kGroupSegs; ++s) {
            const Rec rs = s_rec[s][lane];
            s_rec[s][lane] = run;
            const int ls = seg_len(a, J * kGroupSteps + (int64_t)s * kSeg);
            if (ls > 0) run = rec_combine(run, rs, (float)ls, w2);
        }
    }
    __syncthreads();
    BWD_TRACE(ticket, 2);
    // the frame: the segment's exponents, its history's and the bonus's
    const Rec st = s_rec[seg][lane];
    __syncthreads();  // the records' space is the adjoint sums' next
    const bool hist = st.b > 0.f;
    const float h = fmaf(-(st.n + 1.f), w2, st.anc);  // the history's exponent one step on
    const float hb = hist ? h + (float)((int)((__float_as_uint(st.b) >> 23) & 0xffu) - 127) : -3.0e38f;
    const float d = u2 - w2;  // log2 of 1 / c
    const float lo = m + fminf(d, 0.f), hi = fmaxf(M + fmaxf(d, 0.f), hb);
    const bool frame = len > 0 && hi - lo <= kFrameSpan;
    const float G = 0.5f * (hi + lo);
    const float ic = ex2(d);
    float ys[kSeg];
    Adj loc = adj_empty();
    if (len > 0) {
        if (frame) {
            const float hs = hist ? ex2(h - G) : 0.f;
            loc = len == kSeg ? fwd_frame<true>(sk, sv, sg, ys, len, G, ic, st.a * hs, st.b * hs, w2)
                              : fwd_frame<false>(sk, sv, sg, ys, len, G, ic, st.a * hs, st.b * hs, w2);
        } else {
            loc = len == kSeg ? fwd_steps<true>(a, base, sk, sv, sg, ys, len, st, u2, w2)
                              : fwd_steps<false>(a, base, sk, sv, sg, ys, len, st, u2, w2);
        }
        loc = adj_normalize(loc);
    }
    s_adj[seg][lane] = loc;
    __syncthreads();
    BWD_TRACE(ticket, 3);
    if (seg == 0 && chan) {
        // (this warp's outputs wait in shared memory meanwhile: fewer registers at the peak)
#pragma unroll
        for (int i = 0; i < kSeg; ++i) s_ys[i * kCh + lane] = ys[i];
        // the nearest later group's record is read first; it travels while the group composes
        const bool later = J + 1 < a.NG;
        uint64_t wd[5];
        if (later) slot_load<5>(a.slots + ((int64_t)b * a.NG + J + 1) * 5 * a.C + c, a.C, wd);
        // the group's segments composed right to left; each slot keeps what enters its segment
        // from the group's later segments
        Adj run = adj_empty();
#pragma unroll
        for (int s = kGroupSegs - 1; s >= 0; --s) {
            const Adj ls = s_adj[s][lane];
            s_adj[s][lane] = run;
            const int l = seg_len(a, J * kGroupSteps + (int64_t)s * kSeg);
            if (l > 0) run = adj_compose(ls, run, (float)l, w2);
        }
        // (normalised once: within a group every factor is at most 1 and the sums of the
        // normalised segment sums stay below 2^11, so the chain needs no rescaling per step)
        run = adj_normalize(run);
        uint64_t* my = a.slots + ((int64_t)b * a.NG + J) * 5 * a.C + c;
        Adj gin = adj_empty();
        if (later) {
            if (J > 0) slot_publish<5>(my, a.C, {run.x, run.y, run.xp, run.yp, run.r}, tag_loc);
            uint32_t polls = 0;
            gin = adj_lookback(a, b, J, c, w2, tag_loc, tag_incl, wd, polls);
            if (lane == 0) {
                BWD_TRACE(ticket, 7);
                BWD_TRACE_VALUE(ticket, 8, polls);
            }
        }
        if (J > 0) {
            const Adj out =
                adj_normalize(adj_compose(run, gin, (float)min64(a.T - (int64_t)J * kGroupSteps, kGroupSteps), w2));
            slot_publish<5>(my, a.C, {out.x, out.y, out.xp, out.yp, out.r}, tag_incl);
        }
        s_gin[lane] = gin;
#pragma unroll
        for (int i = 0; i < kSeg; ++i) ys[i] = s_ys[i * kCh + lane];
    }
    __syncthreads();
    BWD_TRACE(ticket, 4);
    float sgw = 0.f, sgu = 0.f;
    if (len > 0) {
        // the sums entering this segment: its group's later segments', with the group's own
        // incoming sums carried across them
        const float after = (float)(min64(a.T, (int64_t)(J + 1) * kGroupSteps) - (t0 + len));
        const Adj in = adj_compose(s_adj[seg][lane], s_gin[lane], after, w2);
        if (frame) {
            // into the frame: F e^{-(len-1) w} times the sums at the segment's last position
            const float sc = ex2(fminf(G - (float)(len - 1) * w2 - in.r, 126.f));
            if (len == kSeg)
                adj_frame<true>(a, base, sk, sv, sg, ys, len, ic, in.x * sc, in.y * sc, in.xp * sc, in.yp * sc, sgw,
                                sgu);
            else
                adj_frame<false>(a, base, sk, sv, sg, ys, len, ic, in.x * sc, in.y * sc, in.xp * sc, in.yp * sc,
                                 sgw, sgu);
        } else {
            if (len == kSeg)
                adj_steps<true>(a, base, sk, sv, sg, ys, len, in, u2, w2, sgw, sgu);
            else
                adj_steps<false>(a, base, sk, sv, sg, ys, len, in, u2, w2, sgw, sgu);
        }
    }
    // the block's gw, gu partials (each thread's into its own first two k elements, free now)
    sk[0] = sgw;
    sk[kCh] = sgu;
    __syncthreads();
    BWD_TRACE(ticket, 5);
    if (seg == 0 && chan) {
        float pw = 0.f, pu = 0.f;
#pragma unroll
        for (int s = 0; s < kGroupSegs; ++s) {
            pw += sm[s * kSeg * kCh + lane];
            pu += sm[s * kSeg * kCh + kCh + lane];
        }
        atomicAdd(a.gw + c, pw);
        atomicAdd(a.gu + c, pu);
    }
    BWD_TRACE(ticket, 6);
}

}  // namespace

#ifdef WKV_TRACE
extern "C" void wkv_bwd_trace_set_buffer(void* buf) {
    unsigned long long* p = static_cast<unsigned long long*>(buf);
    cudaMemcpyToSymbol(g_bwd_trace, &p, sizeof(p));
}
#endif

int64_t backward_segments(int64_t T) { return (T + kSeg - 1) / kSeg; }

bool backward_fits(int64_t B, int64_t T, int64_t C) {
    const int64_t NG = (T + kGroupSteps - 1) / kGroupSteps, cx = (C + kCh - 1) / kCh;
    if (B <= 0 || NG <= 0 || cx <= 0) return true;  // nothing is launched
    return (2 * NG - 1) <= INT32_MAX / B / cx;       // one launch's blocks
}

size_t backward_workspace_bytes(int64_t B, int64_t T, int64_t C) {
    const size_t NG = (size_t)((T + kGroupSteps - 1) / kGroupSteps);
    return kBwdHeaderBytes + (size_t)B * NG * (size_t)C * 9 * sizeof(uint64_t);
}

cudaError_t launch_backward(int64_t B, int64_t T, int64_t C, const float* w, const float* u, const float* k,
                            const float* v, const float* gy, float* gk, float* gv, float* gw, float* gu, void* ws,
                            cudaStream_t s) {
    const int64_t NG = (T + kGroupSteps - 1) / kGroupSteps;
    if (B == 0 || T == 0 || NG == 1) {  // no position, or no group zeroes them: gw, gu start at 0
        cudaError_t e = cudaMemsetAsync(gw, 0, (size_t)C * sizeof(float), s);
        if (e != cudaSuccess) return e;
        e = cudaMemsetAsync(gu, 0, (size_t)C * sizeof(float), s);
        if (e != cudaSuccess || B == 0 || T == 0) return e;
    }
    BwdArgs a;
    a.B = B;
    a.T = T;
    a.C = C;
    a.NG = NG;
    a.cx = (C + kCh - 1) / kCh;
    a.UA = (NG - 1) * B * a.cx;
    a.w = w;
    a.u = u;
    a.k = k;
    a.v = v;
    a.gy = gy;
    a.gk = gk;
    a.gv = gv;
    a.gw = gw;
    a.gu = gu;
    unsigned char* base = static_cast<unsigned char*>(ws);
    a.hdr = reinterpret_cast<BwdHeader*>(base);
    a.fslots = reinterpret_cast<uint64_t*>(base + kBwdHeaderBytes);
    a.slots = a.fslots + (size_t)(B * NG * C) * 4;
    a.dev_err = device_status_word();
    if (!a.dev_err) return cudaErrorInvalidValue;
    a.spin_limit = kSpinLimitDefault;
    const int64_t units = a.UA + NG * B * a.cx;
    if (units > INT32_MAX) return cudaErrorInvalidValue;
    a.units = (uint32_t)units;
    static uint64_t attr_done = 0;  // per device; set once so captured launches issue no attribute call
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev >= 64 || !(attr_done & (1ull << dev))) {
        e = cudaFuncSetAttribute(bwd_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(bwd_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes);
        if (e != cudaSuccess) return e;
        if (dev < 64) attr_done |= 1ull << dev;
    }
    // TMA tiles where every row is whole 16-byte units and the arrays start on 16 bytes
    CUtensorMap tmk{}, tmv{}, tmg{};
    const bool tma = C % 4 == 0 && ((reinterpret_cast<uintptr_t>(k) | reinterpret_cast<uintptr_t>(v) |
                                     reinterpret_cast<uintptr_t>(gy)) & 15) == 0 &&
                     make_tile_map(&tmk, k, B, T, C, 0, kCh, kGroupSteps) &&
                     make_tile_map(&tmv, v, B, T, C, 0, kCh, kGroupSteps) &&
                     make_tile_map(&tmg, gy, B, T, C, 0, kCh, kGroupSteps);
    if (tma)
        return launch_pdl(bwd_kernel<true>, dim3((unsigned)units), dim3(kThreads), kSmemBytes, s, a, tmk, tmv, tmg);
    else
        return launch_pdl(bwd_kernel<false>, dim3((unsigned)units), dim3(kThreads), kSmemBytes, s, a, tmk, tmv, tmg);
}

}  // namespace wkvb
