// Eagle (RWKV-5) matrix-state WKV: per sequence and head of 64 channels
//   S_t = diag(d) S_{t-1} + k_t v_t^T,   y_t = r_t^T S_t,   d = e^{-w} per key channel
// ("RWKV (Attention-RNN Hybrid)", vanos001.github.io, section "Versions: RWKV-4 -> Eagle ->
// Finch": the matrix form of the recurrence and its read-out; one 64 x 64 state per head,
// section "O(N) Inference Characteristics").  Row m of S is a key channel, column j a value
// channel; columns never mix, so each (sequence, head, column) is an independent scan whose
// state is a 64-vector.
//
// Prefill, time-parallel in chunks of kEL tokens (three launches):
//   1 eagle_chunk_sum   each chunk's own contribution to the state at its end, from zero:
//                       U_c = sum_l diag(d)^{len-1-l} k_l v_l^T = (K ⊙ D')^T V, one tensor-core
//                       product (tcgen05, tf32 operands split hi + lo for fp32-level error);
//   2 eagle_state_scan  per state entry, the chunks in time order: S_start(c) and, after the
//                       last chunk, the final state (S <- d^len S + U_c);
//   3 eagle_chunk_out   each chunk's tokens again from its S_start: update, then read-out.
// Decode (eagle_decode): one token of the recurrence per (row, head), the state read and
// written once (section "O(N) Inference Characteristics": one matrix-vector product per token).
//
// The scan, the outputs and the decode are fp32 on the CUDA cores (packed f32x2 where a lane
// holds two key rows); the decay powers are single exponentials 2^{-n w log2 e} of exact
// integer n, so no rounding accumulates in them.
#include <cuda_runtime.h>

#include "wkv_device.cuh"
#include "wkv_eagle_internal.h"
#include "wkv_internal.h"
#include "wkv_pipe_common.cuh"

namespace wkvb {
namespace {

constexpr int kHead = 64;  // channels per head
constexpr int kEL = 64;    // tokens per chunk
constexpr int kSS = kHead * kHead;

struct EagleArgs {
    int64_t B, T, C, H, P;  // P chunks of kEL tokens (the last may be shorter)
    const float *w, *r, *k, *v, *state_in;
    float *y, *state_out;
    float* ch;          // [B][H][P][64][64]: chunk sums U_c, then chunk starting states
    uint32_t* dev_err;  // the library's device-wide error word
    uint32_t spin_limit;
};

constexpr uint32_t kTileBytes = kEL * kHead * sizeof(float);  // one [64 tokens][64 channels] box

// The chunk's rows of r, k, v arrive by TMA tensor copies (rows past T read as zeros); every
// thread waits on the barrier, bounded: a copy that never lands is recorded in the error word
// and the block goes on with what it has (its outputs are then invalid).
__device__ __forceinline__ void wait_tiles(const EagleArgs& a, uint64_t* bar) {
    if (!mbar_wait(bar, 0, a.spin_limit) && threadIdx.x == 0) atomicCAS(a.dev_err, kDevOk, (uint32_t)kDevTimeoutCopy);
}

__device__ __forceinline__ float* chunk_state(const EagleArgs& a, int64_t b, int64_t h, int64_t c) {
    return a.ch + ((b * a.H + h) * a.P + c) * kSS;
}

// Both chunk kernels run 128 threads per (chunk, head, sequence): two per value column j, each
// holding 32 key rows of the column's state.  Lanes 0-15 of a warp take rows 0-31 and lanes
// 16-31 rows 32-63 of the same 16 columns; a thread's register block i (four rows) is key rows
// 32 half + 4 ((i + half) mod 8): the two halves of a warp then read different banks of a
// shared row in the same instruction (each half's lanes read one address, a broadcast).
constexpr int kChunkThreads = 128;

__device__ __forceinline__ int row_block(int half, int i) { return 32 * half + 4 * ((i + half) & 7); }

// ---------------------------------------------------------------------------------------------
// Tensor-core pieces (tcgen05, tf32).  An operand is 64 rows x 64 K fp32 stored K-major in
// 8-row x 16-byte core matrices: element (row, k) at byte (row/8)*2048 + (k/4)*128 + (row%8)*16
// + (k%4)*4, so the descriptor's leading offset (next 4 k) is 128 B and its stride offset (next
// 8 rows) 2048 B; an MMA consumes K = 8 (two core-matrix columns), the next one starts 256 B on.
// fp32 accuracy from split operands: x = hi + lo with hi = x cut to tf32 (its low 13 mantissa
// bits cleared, exact) and lo = x - hi (exact, |lo| < 2^-10 |x|); a product is taken as
// hi*hi + hi*lo + lo*hi, the dropped lo*lo below 2^-20 of it.
// ---------------------------------------------------------------------------------------------
constexpr uint32_t kOpBytes = 64 * 64 * sizeof(float);

__device__ __forceinline__ int op_index(int row, int k) { return (row >> 3) * 512 + (k >> 2) * 32 + (row & 7) * 4 + (k & 3); }

__device__ __forceinline__ void split_tf32(float x, float& hi, float& lo) {
    hi = __uint_as_float(__float_as_uint(x) & 0xFFFFE000u);
    lo = x - hi;
}

// shared-memory matrix descriptor: start, leading offset 128 B, stride offset 2048 B, version 1,
// no swizzle
__device__ __forceinline__ uint64_t op_desc(uint32_t saddr) {
    return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)(128u >> 4) << 16) | ((uint64_t)(2048u >> 4) << 32) |
           ((uint64_t)1 << 46);
}

// instruction descriptor: fp32 accumulate, tf32 A and B, both K-major, M x N
__host__ __device__ constexpr uint32_t tf32_idesc(int M, int N) {
    return (1u << 4) | (2u << 7) | (2u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

__device__ __forceinline__ void mma_tf32(uint32_t tmem_d, uint64_t ad, uint64_t bd, uint32_t idesc, uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
        "l"(ad), "l"(bd), "r"(idesc), "r"(acc));
}

__device__ __forceinline__ void mma_commit(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}

__device__ __forceinline__ void tm_alloc(uint32_t* slot, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(slot)), "r"(ncols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tm_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tm_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tm_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// 16 consecutive fp32 columns of this warp's 32 TMEM lanes
__device__ __forceinline__ void tm_ld16(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
          "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;"
                 : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]),
                   "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]),
                   "+r"(r[15])::"memory");
}

// 1: U_c = (K ⊙ D')^T V as one tensor-core product per (chunk, head, sequence):
//    U_c[m][j] = sum_{l < len} (k_l[m] e^{-(len-1-l) w_m}) v_l[j], M = 64 key rows, N = 64 value
//    columns, K = the chunk's 64 tokens (tokens past T enter as zeros).  The threads write both
//    operands transposed (key and value channel as the row, token as K) and split; one thread
//    issues 8 K-steps x 3 MMAs; the accumulator (M = 64: rows 16q..16q+15 in lanes 32q..32q+15)
//    is read back by the warp of each quadrant.
constexpr size_t kSumSmem = 4 * (size_t)kOpBytes + 64;

__global__ void __launch_bounds__(kChunkThreads) eagle_chunk_sum(EagleArgs a) {
    extern __shared__ __align__(1024) unsigned char smem[];
    float* Ahi = reinterpret_cast<float*>(smem);
    float* Alo = Ahi + 4096;
    float* Bhi = Alo + 4096;
    float* Blo = Bhi + 4096;
    uint64_t* bar = reinterpret_cast<uint64_t*>(smem + 4 * kOpBytes);
    uint32_t* tslot = reinterpret_cast<uint32_t*>(smem + 4 * kOpBytes + 8);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t c = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int64_t t0 = c * kEL;
    const int len = (int)min64(kEL, a.T - t0);
    const int64_t row0 = (b * a.T + t0) * a.C + h * kHead;
    if (warp == 0) tm_alloc(tslot, 64);
    if (tid == 0) {
        mbar_init(bar, 1);
        fence_mbar_init();
    }
    const int ch = tid & 63, t_first = tid >> 6;  // channel (A's / B's row); tokens t_first + 2i
    const float w2 = a.w[h * kHead + ch] * kLog2e;
    constexpr int kPer = kEL / 2;  // tokens per thread
    float kx[kPer], vx[kPer];
#pragma unroll
    for (int i = 0; i < kPer; ++i) {  // every load issued before any is used
        const int t = t_first + 2 * i;
        kx[i] = 0.f;
        vx[i] = 0.f;
        if (t < len) {
            kx[i] = a.k[row0 + (int64_t)t * a.C + ch];
            vx[i] = a.v[row0 + (int64_t)t * a.C + ch];
        }
    }
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
        const int t = t_first + 2 * i;
        const int o = op_index(ch, t);
        // past the sequence the token is zero and so is its weight (2^{+n w} there could be inf)
        const float f = t < len ? ex2(-(float)(len - 1 - t) * w2) : 0.f;
        float hi, lo;
        split_tf32(kx[i] * f, hi, lo);
        Ahi[o] = hi;
        Alo[o] = lo;
        split_tf32(vx[i], hi, lo);
        Bhi[o] = hi;
        Blo[o] = lo;
    }
    fence_proxy_async_smem();  // the operands, written by the threads, are read by the tensor core
    tm_fence_before();
    __syncthreads();
    tm_fence_after();
    const uint32_t tmem = *tslot;
    if (tid == 0) {
        constexpr uint32_t id = tf32_idesc(64, 64);
        const uint32_t ah = smem_u32(Ahi), al = smem_u32(Alo), bh = smem_u32(Bhi), bl = smem_u32(Blo);
#pragma unroll
        for (uint32_t st = 0; st < kEL / 8; ++st) {
            const uint32_t off = 256u * st;
            mma_tf32(tmem, op_desc(ah + off), op_desc(bh + off), id, st);
            mma_tf32(tmem, op_desc(ah + off), op_desc(bl + off), id, 1);
            mma_tf32(tmem, op_desc(al + off), op_desc(bh + off), id, 1);
        }
        mma_commit(bar);
    }
    if (!mbar_wait(bar, 0, a.spin_limit) && lane == 0) atomicCAS(a.dev_err, kDevOk, (uint32_t)kDevTimeoutCopy);
    tm_fence_after();
    float* out = chunk_state(a, b, h, c) + (int64_t)(16 * warp + lane) * kHead;
#pragma unroll
    for (int cb = 0; cb < kHead; cb += 16) {
        uint32_t r[16];
        tm_ld16(tmem + ((uint32_t)(32 * warp) << 16) + (uint32_t)cb, r);
        if (lane < 16) {
#pragma unroll
            for (int q = 0; q < 16; q += 4)
                *reinterpret_cast<float4*>(out + cb + q) = make_float4(__uint_as_float(r[q]), __uint_as_float(r[q + 1]),
                                                                       __uint_as_float(r[q + 2]), __uint_as_float(r[q + 3]));
        }
    }
    tm_fence_before();
    __syncthreads();
    if (warp == 0) tm_dealloc(tmem, 64);
}

constexpr int kScanThreads = 256;
constexpr int kScanBlk = 16;  // chunk sums loaded before any is overwritten

// 2: per state entry (b, h, m, j), in time order: the slot of chunk c receives S_start(c),
// then S <- e^{-len_c w_m} S + U_c; the state after the last chunk is the final state.
__global__ void __launch_bounds__(kScanThreads) eagle_state_scan(EagleArgs a) {
    const int64_t e = (int64_t)blockIdx.x * kScanThreads + threadIdx.x;
    if (e >= a.B * a.H * kSS) return;
    const int64_t bh = e / kSS;
    const int mj = (int)(e % kSS), m = mj / kHead;
    const int64_t h = bh % a.H;
    const float w2 = a.w[h * kHead + m] * kLog2e;
    const float d_full = ex2(-(float)kEL * w2);
    float S = a.state_in ? a.state_in[bh * kSS + mj] : 0.f;
    float* p = a.ch + bh * a.P * kSS + mj;
    for (int64_t c0 = 0; c0 < a.P; c0 += kScanBlk) {
        const int nb = (int)min64(kScanBlk, a.P - c0);
        float u[kScanBlk];
#pragma unroll
        for (int i = 0; i < kScanBlk; ++i)
            if (i < nb) u[i] = p[(c0 + i) * kSS];
#pragma unroll
        for (int i = 0; i < kScanBlk; ++i) {
            if (i < nb) {
                const int64_t c = c0 + i;
                p[c * kSS] = S;
                const int64_t len = min64(kEL, a.T - c * kEL);
                const float d = len == kEL ? d_full : ex2(-(float)len * w2);
                S = fmaf(d, S, u[i]);
            }
        }
    }
    if (a.state_out) a.state_out[bh * kSS + mj] = S;
}

// 3: each chunk's tokens from its starting state: S <- diag(d) S + k_l v_l^T, y_l = r_l^T S
constexpr size_t kOutSmem = 3 * (size_t)kTileBytes + 128;  // r, k, v tiles and the barrier

__global__ void __launch_bounds__(kChunkThreads) eagle_chunk_out(EagleArgs a, const __grid_constant__ CUtensorMap tmr,
                                                                 const __grid_constant__ CUtensorMap tmk,
                                                                 const __grid_constant__ CUtensorMap tmv) {
    extern __shared__ __align__(1024) unsigned char smem[];
    float(*rs)[kHead] = reinterpret_cast<float(*)[kHead]>(smem);
    float(*ks)[kHead] = reinterpret_cast<float(*)[kHead]>(smem + kTileBytes);
    float(*vs)[kHead] = reinterpret_cast<float(*)[kHead]>(smem + 2 * kTileBytes);
    uint64_t* bar = reinterpret_cast<uint64_t*>(smem + 3 * kTileBytes);
    const int tid = threadIdx.x, lane = tid & 31, half = lane >> 4;
    const int j = (tid >> 5) * 16 + (lane & 15);
    const int64_t c = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int64_t t0 = c * kEL;
    const int len = (int)min64(kEL, a.T - t0);
    if (tid == 0) {
        mbar_init(bar, 1);
        fence_mbar_init();
        mbar_arrive_expect_tx(bar, 3 * kTileBytes);
        tma_load_3d(&rs[0][0], &tmr, (int)(h * kHead), (int)t0, (int)b, bar);
        tma_load_3d(&ks[0][0], &tmk, (int)(h * kHead), (int)t0, (int)b, bar);
        tma_load_3d(&vs[0][0], &tmv, (int)(h * kHead), (int)t0, (int)b, bar);
    }
    // this thread's half of the starting state and its decays while the tiles are in flight
    const float* st = chunk_state(a, b, h, c) + j;
    const float* wh = a.w + h * kHead;
    float2 S[16], d[16];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int m = row_block(half, i);
        S[2 * i] = make_float2(st[(m + 0) * kHead], st[(m + 1) * kHead]);
        S[2 * i + 1] = make_float2(st[(m + 2) * kHead], st[(m + 3) * kHead]);
        d[2 * i] = make_float2(ex2(-wh[m] * kLog2e), ex2(-wh[m + 1] * kLog2e));
        d[2 * i + 1] = make_float2(ex2(-wh[m + 2] * kLog2e), ex2(-wh[m + 3] * kLog2e));
    }
    __syncthreads();  // the barrier is initialised
    wait_tiles(a, bar);
    float* yrow = a.y + (b * a.T + t0) * a.C + h * kHead + j;
    for (int l = 0; l < len; ++l) {
        const float vj = vs[l][j];
        const float2 vv = make_float2(vj, vj);
        float2 acc[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                         make_float2(0.f, 0.f)};
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int m = row_block(half, i);
            const float4 kk = *reinterpret_cast<const float4*>(&ks[l][m]);
            const float4 rr = *reinterpret_cast<const float4*>(&rs[l][m]);
            S[2 * i] = __ffma2_rn(d[2 * i], S[2 * i], __fmul2_rn(make_float2(kk.x, kk.y), vv));
            S[2 * i + 1] = __ffma2_rn(d[2 * i + 1], S[2 * i + 1], __fmul2_rn(make_float2(kk.z, kk.w), vv));
            acc[i & 3] = __ffma2_rn(make_float2(rr.x, rr.y), S[2 * i], acc[i & 3]);
            acc[i & 3] = __ffma2_rn(make_float2(rr.z, rr.w), S[2 * i + 1], acc[i & 3]);
        }
        const float2 s01 = __fadd2_rn(acc[0], acc[1]), s23 = __fadd2_rn(acc[2], acc[3]);
        const float2 sp = __fadd2_rn(s01, s23);
        float yv = sp.x + sp.y;
        yv += __shfl_xor_sync(0xffffffffu, yv, 16);  // the other 32 key rows
        if (half == 0) yrow[(int64_t)l * a.C] = yv;
    }
}

// One token per (row, head): rows = N L, w [L][C] by the row's layer, state [rows][H][64][64].
__global__ void __launch_bounds__(kHead) eagle_decode(int64_t L, int64_t C, int64_t H, const float* w,
                                                      const float* r, const float* k, const float* v,
                                                      float* state, float* y) {
    __shared__ float rs[kHead], ks[kHead], ds[kHead];
    const int j = threadIdx.x;
    const int64_t idx = blockIdx.x, row = idx / H, h = idx % H, layer = row % L;
    const int64_t base = row * C + h * kHead;
    rs[j] = r[base + j];
    ks[j] = k[base + j];
    ds[j] = ex2(-w[layer * C + h * kHead + j] * kLog2e);
    const float vj = v[base + j];
    float* S = state + idx * kSS + j;
    float s[kHead];
#pragma unroll
    for (int m = 0; m < kHead; ++m) s[m] = S[m * kHead];
    __syncthreads();
    float acc0 = 0.f, acc1 = 0.f;
#pragma unroll
    for (int m = 0; m < kHead; m += 2) {
        s[m] = fmaf(ds[m], s[m], ks[m] * vj);
        s[m + 1] = fmaf(ds[m + 1], s[m + 1], ks[m + 1] * vj);
        acc0 = fmaf(rs[m], s[m], acc0);
        acc1 = fmaf(rs[m + 1], s[m + 1], acc1);
    }
#pragma unroll
    for (int m = 0; m < kHead; ++m) S[m * kHead] = s[m];
    y[base + j] = acc0 + acc1;
}

}  // namespace

int64_t eagle_chunks(int64_t T) { return (T + kEL - 1) / kEL; }

cudaError_t launch_eagle_forward(int64_t B, int64_t T, int64_t C, const float* w, const float* r, const float* k,
                                 const float* v, const float* state_in, float* y, float* state_out, void* ws,
                                 cudaStream_t s) {
    const int64_t H = C / kHead;
    if (T == 0) {  // no token: the state passes through (zero without one)
        if (!state_out) return cudaSuccess;
        const size_t bytes = (size_t)B * (size_t)H * kSS * sizeof(float);
        if (state_in) return cudaMemcpyAsync(state_out, state_in, bytes, cudaMemcpyDeviceToDevice, s);
        return cudaMemsetAsync(state_out, 0, bytes, s);
    }
    CUtensorMap tmr, tmk, tmv;
    if (!make_tile_map(&tmr, r, B, T, C, 0, kHead, kEL) || !make_tile_map(&tmk, k, B, T, C, 0, kHead, kEL) ||
        !make_tile_map(&tmv, v, B, T, C, 0, kHead, kEL))
        return cudaErrorInvalidValue;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    static uint64_t attr_done = 0;
    if (dev >= 64 || !(attr_done & (1ull << dev))) {
        e = cudaFuncSetAttribute(eagle_chunk_out, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kOutSmem);
        if (e != cudaSuccess) return e;
        e = cudaFuncSetAttribute(eagle_chunk_sum, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSumSmem);
        if (e != cudaSuccess) return e;
        if (dev < 64) attr_done |= 1ull << dev;
    }
    EagleArgs a;
    a.B = B;
    a.T = T;
    a.C = C;
    a.H = H;
    a.P = eagle_chunks(T);
    a.w = w;
    a.r = r;
    a.k = k;
    a.v = v;
    a.state_in = state_in;
    a.y = y;
    a.state_out = state_out;
    a.ch = static_cast<float*>(ws);
    a.dev_err = device_status_word();
    a.spin_limit = kSpinLimitDefault;
    if (!a.dev_err) return cudaErrorInvalidValue;
    const dim3 grid((unsigned)a.P, (unsigned)H, (unsigned)B);
    eagle_chunk_sum<<<grid, kChunkThreads, kSumSmem, s>>>(a);
    const int64_t entries = B * H * kSS;
    eagle_state_scan<<<(unsigned)((entries + kScanThreads - 1) / kScanThreads), kScanThreads, 0, s>>>(a);
    eagle_chunk_out<<<grid, kChunkThreads, kOutSmem, s>>>(a, tmr, tmk, tmv);
    return cudaGetLastError();
}

cudaError_t launch_eagle_decode(int64_t N, int64_t L, int64_t C, const float* w, const float* r, const float* k,
                                const float* v, float* state, float* y, cudaStream_t s) {
    const int64_t H = C / kHead;
    eagle_decode<<<(unsigned)(N * L * H), kHead, 0, s>>>(L, C, H, w, r, k, v, state, y);
    return cudaGetLastError();
}

}  // namespace wkvb
