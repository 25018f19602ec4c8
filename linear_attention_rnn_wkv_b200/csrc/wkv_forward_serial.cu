// Serial-scan WKV forward: one thread per (b, c) walks all of T.
//
// The recurrence is the running-maximum form of the RWKV transformer-math page
// (aicassindra.com, tm_rwkv_math), section "Numerical stability: carry the
// exponent", evaluated token after token in the anchored form of scan_step: the
// history decays by counting steps, so long scans do not drift.
//
// Data movement (bulk path, C a multiple of 16 bytes): a CTA owns NT consecutive
// channels of one sequence.  Tiles of TS time steps x NT channels of k and v are
// brought into a shared-memory ring of NS stages by the TMA engine
// (cp.async.bulk, one copy per row, completion on an mbarrier); every thread then
// reads its own column.  y is written straight to global memory (a warp writes one
// contiguous row segment per step).  Ragged C falls back to per-element loads.
#include "wkv_device.cuh"
#include "wkv_internal.h"

namespace wkvb {
namespace {

template <typename TIO>
struct SerialChannel {
    float a, b, anc, n;
    float w2, u2;

    __device__ __forceinline__ void init(const float* w, const float* u, const float* state_in, int64_t bc,
                                         int64_t BC, int64_t c) {
        w2 = w[c] * kLog2e;
        u2 = u[c] * kLog2e;
        if (state_in) {
            a = state_in[bc];
            b = state_in[BC + bc];
            anc = state_in[2 * BC + bc] * kLog2e;
        } else {
            a = 0.f;
            b = 0.f;
            anc = kPEmpty;
        }
        n = 0.f;
    }

    __device__ __forceinline__ float step(float kk, float vv) { return scan_step(a, b, anc, n, kk * kLog2e, vv, u2, w2); }

    __device__ __forceinline__ void store_state(float* state_out, int64_t bc, int64_t BC) {
        state_out[bc] = a;
        state_out[BC + bc] = b;
        state_out[2 * BC + bc] = fmaf(-n, w2, anc) * kLn2;
    }
};

// Bulk-copy path.  Shared memory: NS stages of [TS][NT] k then [TS][NT] v, then NS mbarriers.
template <typename TIO, int NT, int TS, int NS>
__global__ void __launch_bounds__(NT) serial_bulk_kernel(ForwardArgs args) {
    grid_dep_launch_dependents();
    grid_dep_wait();  // before any global memory access
    extern __shared__ __align__(128) unsigned char smem[];
    constexpr int kStageElems = TS * NT;
    TIO* stage_base = reinterpret_cast<TIO*>(smem);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + sizeof(TIO) * 2 * kStageElems * NS);

    const int64_t B = args.B, T = args.T, C = args.C;
    const int64_t groups_per_b = (C + NT - 1) / NT;
    const int64_t b = blockIdx.x / groups_per_b;
    const int64_t c0 = (blockIdx.x % groups_per_b) * NT;
    const int nch = (int)min64(NT, C - c0);
    const int tid = threadIdx.x;
    const bool active = tid < nch;
    const int64_t c = c0 + tid;
    const uint32_t row_bytes = (uint32_t)nch * sizeof(TIO);
    const TIO* kg = static_cast<const TIO*>(args.k) + (b * T) * C + c0;
    const TIO* vg = static_cast<const TIO*>(args.v) + (b * T) * C + c0;
    TIO* yg = static_cast<TIO*>(args.y) + (b * T) * C + c0;
    const int64_t ntiles = (T + TS - 1) / TS;

    if (tid == 0) {
        for (int s = 0; s < NS; ++s) mbar_init(&bars[s], 1);
        fence_mbar_init();
    }
    __syncthreads();

    auto issue = [&](int64_t tile, int s) {
        // warp 0 only
        const int lane = tid & 31;
        const int64_t r0 = tile * TS;
        const int nrows = (int)min64(TS, T - r0);
        if (lane == 0) mbar_arrive_expect_tx(&bars[s], 2u * (uint32_t)nrows * row_bytes);
        __syncwarp();
        TIO* ks = stage_base + (size_t)s * 2 * kStageElems;
        TIO* vs = ks + kStageElems;
        for (int r = lane; r < nrows; r += 32) {
            bulk_g2s(ks + r * NT, kg + (r0 + r) * C, row_bytes, &bars[s]);
            bulk_g2s(vs + r * NT, vg + (r0 + r) * C, row_bytes, &bars[s]);
        }
    };

    if (tid < 32) {
        for (int s = 0; s < NS && s < ntiles; ++s) issue(s, s);
    }

    SerialChannel<TIO> ch;
    const int64_t BC = B * C;
    const int64_t bc = b * C + c;
    if (active) ch.init(args.w, args.u, args.state_in, bc, BC, c);

    bool failed = false;
    int64_t failed_tile = ntiles;
    for (int64_t tile = 0; tile < ntiles; ++tile) {
        const int s = (int)(tile % NS);
        const uint32_t parity = (uint32_t)((tile / NS) & 1);
        bool timed_out = false;
        for (uint32_t it = 0; !mbar_try_wait(&bars[s], parity); ++it) {
            if (it >= args.spin_limit) {
                timed_out = true;
                break;
            }
            __nanosleep(64);
        }
        // one CTA-wide decision, so warp 0 keeps its copies and expectations in step
        if (__syncthreads_or(timed_out)) {
            if (tid == 0) {
                atomicCAS(args.err, kDevOk, kDevTimeoutCopy);
                atomicCAS(args.dev_err, kDevOk, kDevTimeoutCopy);
            }
            failed = true;
            failed_tile = tile;
            break;
        }
        const TIO* ks = stage_base + (size_t)s * 2 * kStageElems;
        const TIO* vs = ks + kStageElems;
        const int64_t r0 = tile * TS;
        const int nrows = (int)min64(TS, T - r0);
        if (active) {
#pragma unroll 4
            for (int r = 0; r < nrows; ++r) {
                float kk = io<TIO>::to_f(ks[r * NT + tid]);
                float vv = io<TIO>::to_f(vs[r * NT + tid]);
                float yy = ch.step(kk, vv);
                io<TIO>::store(yg + (r0 + r) * C + tid, yy);
            }
        }
        __syncthreads();  // stage s fully consumed
        if (tid < 32 && tile + NS < ntiles) issue(tile + NS, s);
    }
    if (failed) {
        // Tiles [failed_tile, failed_tile + NS) may still have copies in flight: let them
        // land (bounded) before the CTA's shared memory is released.
        for (int64_t tile = failed_tile; tile < ntiles && tile < failed_tile + NS; ++tile) {
            const int s = (int)(tile % NS);
            const uint32_t parity = (uint32_t)((tile / NS) & 1);
            for (uint32_t it = 0; it < args.spin_limit && !mbar_try_wait(&bars[s], parity); ++it) __nanosleep(64);
        }
        return;
    }
    if (active && args.state_out) ch.store_state(args.state_out, bc, BC);
}

// Per-element path for C not a multiple of 16 bytes: coalesced scalar loads.
template <typename TIO, int NT>
__global__ void __launch_bounds__(NT) serial_plain_kernel(ForwardArgs args) {
    grid_dep_launch_dependents();
    grid_dep_wait();  // before any global memory access
    const int64_t B = args.B, T = args.T, C = args.C;
    const int64_t groups_per_b = (C + NT - 1) / NT;
    const int64_t b = blockIdx.x / groups_per_b;
    const int64_t c = (blockIdx.x % groups_per_b) * NT + threadIdx.x;
    if (c >= C) return;
    const TIO* kg = static_cast<const TIO*>(args.k) + (b * T) * C + c;
    const TIO* vg = static_cast<const TIO*>(args.v) + (b * T) * C + c;
    TIO* yg = static_cast<TIO*>(args.y) + (b * T) * C + c;
    SerialChannel<TIO> ch;
    const int64_t BC = B * C;
    const int64_t bc = b * C + c;
    ch.init(args.w, args.u, args.state_in, bc, BC, c);
#pragma unroll 4
    for (int64_t t = 0; t < T; ++t) {
        float kk = io<TIO>::load(kg + t * C);
        float vv = io<TIO>::load(vg + t * C);
        io<TIO>::store(yg + t * C, ch.step(kk, vv));
    }
    if (args.state_out) ch.store_state(args.state_out, bc, BC);
}

template <typename TIO>
cudaError_t launch_serial_t(const ForwardArgs& a, cudaStream_t s) {
    constexpr int NT = 128;
    const int64_t groups = (a.C + NT - 1) / NT;
    const int64_t grid = a.B * groups;
    const bool bulk = ((a.C * (int64_t)sizeof(TIO)) % 16) == 0;
    if (bulk) {
        constexpr int TS = 32, NS = 4;
        const size_t smem = sizeof(TIO) * 2 * TS * NT * NS + 8 * NS;
        auto kern = serial_bulk_kernel<TIO, NT, TS, NS>;
        static uint64_t attr_done = 0;  // per device, so captured launches issue no attribute call
        int dev = 0;
        cudaError_t e = cudaGetDevice(&dev);
        if (e != cudaSuccess) return e;
        if (dev >= 64 || !(attr_done & (1ull << dev))) {
            e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
            if (e != cudaSuccess) return e;
            if (dev < 64) attr_done |= 1ull << dev;
        }
        return launch_pdl(kern, dim3((unsigned)grid), dim3(NT), smem, s, a);
    } else {
        return launch_pdl(serial_plain_kernel<TIO, NT>, dim3((unsigned)grid), dim3(NT), 0, s, a);
    }
}

}  // namespace

cudaError_t launch_forward_serial(const ForwardArgs& a, cudaStream_t s) {
    return a.io == 1 ? launch_serial_t<__nv_bfloat16>(a, s) : launch_serial_t<float>(a, s);
}

}  // namespace wkvb
