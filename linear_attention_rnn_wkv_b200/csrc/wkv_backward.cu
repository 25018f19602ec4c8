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
// Time-parallel in segments of kSeg steps, one thread per (b, c, segment), five launches:
//   A  each segment's forward recurrence from the empty state -> its state record;
//   B  per channel, the records combined in time order -> each segment's starting state
//      (and gw, gu zeroed for the atomics of E), two-level over groups of segments;
//   C  each segment's forward from its starting state, accumulating its local (X, Y, X', Y')
//      left to right as each D_t and y_t appears;
//   D  per channel, the local sums composed right to left -> each segment's incoming sums,
//      two-level like B;
//   E  each segment's forward again, keeping per position the output's reference exponent q_t,
//      1 / Dn_t (D_t = Dn_t 2^{q_t}) and y_t in shared memory, then its adjoint recurrence from
//      the incoming sums -> gk, gv, and gw, gu partials added with atomics.
// k, v are read three times and gy twice (40 B per element with gk, gv written); nothing per
// position is stored in global memory.
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
constexpr int kScanBlk = 8;        // segment records loaded together by the per-channel scans
constexpr int kThreads = 128;      // threads per block (channels of one (b, segment))
constexpr float kRNone = 3.0e38f;  // reference of an empty adjoint sum
// E's per-position values: [kSeg][3][kThreads] floats, each thread its own column
constexpr size_t kGradSmem = (size_t)kSeg * 3 * kThreads * sizeof(float);
static_assert(kGradSmem <= 48 * 1024, "fits the default dynamic shared memory limit");

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

struct BwdArgs {
    int64_t B, T, C, P;  // P segments of kSeg steps (the last may be shorter)
    const float *w, *u, *k, *v, *gy;
    float *gk, *gv, *gw, *gu;
    float* fs;  // [4][B][P][C] segment records, then starting states
    float* as;  // [5][B][P][C] local adjoint sums, then incoming sums
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

// A: each segment's forward from the empty state -> its record
__global__ void __launch_bounds__(kThreads) bwd_seg_forward(BwdArgs a) {
    const int64_t c = (int64_t)blockIdx.x * kThreads + threadIdx.x;
    const int64_t j = blockIdx.y, b = blockIdx.z;
    if (c >= a.C) return;
    const float w2 = a.w[c] * kLog2e, u2 = a.u[c] * kLog2e;
    const int64_t t0 = j * kSeg, t1 = min64(a.T, t0 + kSeg);
    FwdState s{0.f, 0.f, kPEmpty, 0.f};
    forward_span<false, false>(a, b * a.T * a.C + c, t0, t1, s, u2, w2, [](int, const FwdOut&, float) {});
    const int64_t si = seg_index(a, b, j, c), SP = a.B * a.P * a.C;
    a.fs[si] = s.a;
    a.fs[SP + si] = s.bb;
    a.fs[2 * SP + si] = s.anc;
    a.fs[3 * SP + si] = s.n;
}

// The two per-channel scans (B, D) split a channel's segments into kGroups consecutive groups:
// every group folds its own segments (in parallel with the others), each group then combines
// the aggregates of the groups before it (B) or after it (D), and walks its segments again from
// that carry, writing each segment's carry.  The serial chain per channel is one group long.
constexpr int kGroups = 8;
constexpr int kScanCh = 32;  // channels per scan block: one warp per group
constexpr int kScanThreadsB = kScanCh * kGroups;

struct GroupSpan {
    int64_t j0, j1;  // the group's segments [j0, j1) (possibly empty)
};

__device__ __forceinline__ GroupSpan group_span(const BwdArgs& a, int g) {
    const int64_t per = (a.P + kGroups - 1) / kGroups;
    const int64_t j0 = min64(a.P, g * per);
    return GroupSpan{j0, min64(a.P, j0 + per)};
}

__device__ __forceinline__ float seg_len(const BwdArgs& a, int64_t j) {
    return (float)(min64(a.T, (j + 1) * kSeg) - j * kSeg);
}

__device__ __forceinline__ float group_len(const BwdArgs& a, int g) {
    const GroupSpan s = group_span(a, g);
    return s.j1 > s.j0 ? (float)(min64(a.T, s.j1 * kSeg) - s.j0 * kSeg) : 0.f;
}

__device__ __forceinline__ Rec load_rec(const BwdArgs& a, int64_t si) {
    const int64_t SP = a.B * a.P * a.C;
    return Rec{a.fs[si], a.fs[SP + si], a.fs[2 * SP + si], a.fs[3 * SP + si]};
}

// B: per channel, segment records combined left to right -> each segment's starting state
// (and gw, gu zeroed for the atomics of E).
__global__ void __launch_bounds__(kScanThreadsB) bwd_seg_carry(BwdArgs a) {
    __shared__ Rec agg[kGroups][kScanCh];
    const int lane = threadIdx.x % kScanCh, g = threadIdx.x / kScanCh;
    const int64_t c = (int64_t)blockIdx.x * kScanCh + lane, b = blockIdx.y;
    const bool live = c < a.C;
    const float w2 = live ? a.w[c] * kLog2e : 0.f;
    const GroupSpan sp = group_span(a, g);
    const int64_t SP = a.B * a.P * a.C;
    Rec run = rec_identity();
    if (live) {
        if (b == 0 && g == 0) {  // E accumulates into these
            a.gw[c] = 0.f;
            a.gu[c] = 0.f;
        }
        for (int64_t j0 = sp.j0; j0 < sp.j1; j0 += kScanBlk) {
            const int nb = (int)min64(kScanBlk, sp.j1 - j0);
            Rec seg[kScanBlk];
#pragma unroll
            for (int i = 0; i < kScanBlk; ++i)
                if (i < nb) seg[i] = load_rec(a, seg_index(a, b, j0 + i, c));
#pragma unroll
            for (int i = 0; i < kScanBlk; ++i)
                if (i < nb) run = rec_combine(run, seg[i], seg_len(a, j0 + i), w2);
        }
    }
    agg[g][lane] = run;
    __syncthreads();
    if (!live) return;
    Rec carry = rec_identity();  // the groups before this one, in time order
    for (int q = 0; q < g; ++q) carry = rec_combine(carry, agg[q][lane], group_len(a, q), w2);
    for (int64_t j0 = sp.j0; j0 < sp.j1; j0 += kScanBlk) {
        const int nb = (int)min64(kScanBlk, sp.j1 - j0);
        Rec seg[kScanBlk];
#pragma unroll
        for (int i = 0; i < kScanBlk; ++i)
            if (i < nb) seg[i] = load_rec(a, seg_index(a, b, j0 + i, c));
#pragma unroll
        for (int i = 0; i < kScanBlk; ++i) {
            if (i < nb) {
                const int64_t si = seg_index(a, b, j0 + i, c);
                a.fs[si] = carry.a;
                a.fs[SP + si] = carry.b;
                a.fs[2 * SP + si] = carry.anc;
                a.fs[3 * SP + si] = carry.n;
                carry = rec_combine(carry, seg[i], seg_len(a, j0 + i), w2);
            }
        }
    }
}

// C: each segment's forward from its starting state -> its local adjoint sums
__global__ void __launch_bounds__(kThreads) bwd_seg_local(BwdArgs a) {
    const int64_t c = (int64_t)blockIdx.x * kThreads + threadIdx.x;
    const int64_t j = blockIdx.y, b = blockIdx.z;
    if (c >= a.C) return;
    const float w2 = a.w[c] * kLog2e, u2 = a.u[c] * kLog2e;
    const int64_t t0 = j * kSeg, t1 = min64(a.T, t0 + kSeg);
    const int64_t base = b * a.T * a.C + c;
    const int64_t si = seg_index(a, b, j, c), SP = a.B * a.P * a.C;
    FwdState s = load_state(a, si);
    LocalSums ls{0.f, 0.f, 0.f, 0.f, kRNone, 0.f};
    forward_span<true, true>(a, base, t0, t1, s, u2, w2,
                             [&](int i, const FwdOut& o, float g) { ls.add((float)i, g, o, w2); });
    a.as[si] = ls.x;
    a.as[SP + si] = ls.y;
    a.as[2 * SP + si] = ls.xp;
    a.as[3 * SP + si] = ls.yp;
    a.as[4 * SP + si] = fmaf(ls.Rj, w2, ls.Rq);
}

// What leaves a span of len steps to its left: its local sums plus the sums entering it from
// the right carried across it (X decays by e^{-w len}; X' also gains len X).
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

__device__ __forceinline__ Adj load_adj(const BwdArgs& a, int64_t si) {
    const int64_t SP = a.B * a.P * a.C;
    return Adj{a.as[si], a.as[SP + si], a.as[2 * SP + si], a.as[3 * SP + si], a.as[4 * SP + si]};
}

// D: per channel, local sums composed right to left -> each segment's incoming sums
__global__ void __launch_bounds__(kScanThreadsB) bwd_seg_adjoint_carry(BwdArgs a) {
    __shared__ Adj agg[kGroups][kScanCh];
    const int lane = threadIdx.x % kScanCh, g = threadIdx.x / kScanCh;
    const int64_t c = (int64_t)blockIdx.x * kScanCh + lane, b = blockIdx.y;
    const bool live = c < a.C;
    const float w2 = live ? a.w[c] * kLog2e : 0.f;
    const GroupSpan sp = group_span(a, g);
    const int64_t SP = a.B * a.P * a.C;
    Adj run = adj_empty();
    if (live) {
        for (int64_t j1 = sp.j1; j1 > sp.j0; j1 -= kScanBlk) {
            const int nb = (int)min64(kScanBlk, j1 - sp.j0);
            Adj loc[kScanBlk];
#pragma unroll
            for (int i = 0; i < kScanBlk; ++i)
                if (i < nb) loc[i] = load_adj(a, seg_index(a, b, j1 - 1 - i, c));
#pragma unroll
            for (int i = 0; i < kScanBlk; ++i)
                if (i < nb) run = adj_compose(loc[i], run, seg_len(a, j1 - 1 - i), w2);
        }
    }
    agg[g][lane] = run;
    __syncthreads();
    if (!live) return;
    Adj in = adj_empty();  // the groups after this one, composed right to left
    for (int q = kGroups - 1; q > g; --q) in = adj_compose(agg[q][lane], in, group_len(a, q), w2);
    for (int64_t j1 = sp.j1; j1 > sp.j0; j1 -= kScanBlk) {
        const int nb = (int)min64(kScanBlk, j1 - sp.j0);
        Adj loc[kScanBlk];
#pragma unroll
        for (int i = 0; i < kScanBlk; ++i)
            if (i < nb) loc[i] = load_adj(a, seg_index(a, b, j1 - 1 - i, c));
#pragma unroll
        for (int i = 0; i < kScanBlk; ++i) {
            if (i < nb) {
                const int64_t j = j1 - 1 - i, si = seg_index(a, b, j, c);
                a.as[si] = in.x;
                a.as[SP + si] = in.y;
                a.as[2 * SP + si] = in.xp;
                a.as[3 * SP + si] = in.yp;
                a.as[4 * SP + si] = in.r;
                in = adj_compose(loc[i], in, seg_len(a, j), w2);
            }
        }
    }
}

// E: each segment's forward again (per-position values into shared memory), then its adjoint
// recurrence from its incoming sums -> gradients
__global__ void __launch_bounds__(kThreads) bwd_seg_grads(BwdArgs a) {
    extern __shared__ float sm[];  // [kSeg][3][kThreads]
    const int tid = threadIdx.x;
    const int64_t c = (int64_t)blockIdx.x * kThreads + tid;
    const int64_t j = blockIdx.y, b = blockIdx.z;
    if (c >= a.C) return;  // no block-wide synchronisation below: each thread uses its own column
    const float w2 = a.w[c] * kLog2e, u2 = a.u[c] * kLog2e;
    const int64_t t0 = j * kSeg, t1 = min64(a.T, t0 + kSeg);
    const int64_t base = b * a.T * a.C + c;
    const int64_t si = seg_index(a, b, j, c), SP = a.B * a.P * a.C;
    FwdState fsd = load_state(a, si);
    forward_span<true, false>(a, base, t0, t1, fsd, u2, w2, [&](int i, const FwdOut& o, float) {
        sm[(i * 3 + 0) * kThreads + tid] = o.q;
        sm[(i * 3 + 1) * kThreads + tid] = o.rd;
        sm[(i * 3 + 2) * kThreads + tid] = o.y;
    });
    Adj s{a.as[si], a.as[SP + si], a.as[2 * SP + si], a.as[3 * SP + si], a.as[4 * SP + si]};
    float sgw = 0.f, sgu = 0.f;
    auto step = [&](int64_t t, float kt, float vt, float g) {
        const int i = (int)(t - t0);
        const FwdOut o{sm[(i * 3 + 0) * kThreads + tid], sm[(i * 3 + 1) * kThreads + tid],
                       sm[(i * 3 + 2) * kThreads + tid]};
        float gk, gv;
        adj_step(s, kt * kLog2e, vt, g, o, u2, w2, gk, gv, sgw, sgu);
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
    atomicAdd(&a.gw[c], sgw);
    atomicAdd(&a.gu[c], sgu);
}

}  // namespace

int64_t backward_segments(int64_t T) { return (T + kSeg - 1) / kSeg; }

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
    a.fs = static_cast<float*>(ws);
    a.as = a.fs + 4 * SP;
    const unsigned cx = (unsigned)((C + kThreads - 1) / kThreads);
    const dim3 seg_grid(cx, (unsigned)a.P, (unsigned)B);
    const dim3 scan_grid((unsigned)((C + kScanCh - 1) / kScanCh), (unsigned)B);
    bwd_seg_forward<<<seg_grid, kThreads, 0, s>>>(a);
    bwd_seg_carry<<<scan_grid, kScanThreadsB, 0, s>>>(a);
    bwd_seg_local<<<seg_grid, kThreads, 0, s>>>(a);
    bwd_seg_adjoint_carry<<<scan_grid, kScanThreadsB, 0, s>>>(a);
    bwd_seg_grads<<<seg_grid, kThreads, kGradSmem, s>>>(a);
    return cudaGetLastError();
}

}  // namespace wkvb
