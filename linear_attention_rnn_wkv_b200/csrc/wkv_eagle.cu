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
#include <cuda_bf16.h>
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

// Threads 0-15 of the warp: 16 (8) consecutive fp32 columns of lanes 0-15 of this warp's TMEM
// quadrant; threads 16-31: the same lanes, the columns 16 (8) further on.
__device__ __forceinline__ void tm_ld16x2(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.16x32bx2.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
        "%14, %15}, [%16], 16;"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
          "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;"
                 : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]),
                   "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]),
                   "+r"(r[15])::"memory");
}
// two such loads (two column ranges), then one wait
__device__ __forceinline__ void tm_ld16x2_pair(uint32_t ta, uint32_t tb, uint32_t (&r)[16], uint32_t (&s)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.16x32bx2.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
        "%14, %15}, [%16], 16;"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
          "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(ta));
    asm volatile(
        "tcgen05.ld.sync.aligned.16x32bx2.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
        "%14, %15}, [%16], 16;"
        : "=r"(s[0]), "=r"(s[1]), "=r"(s[2]), "=r"(s[3]), "=r"(s[4]), "=r"(s[5]), "=r"(s[6]), "=r"(s[7]), "=r"(s[8]),
          "=r"(s[9]), "=r"(s[10]), "=r"(s[11]), "=r"(s[12]), "=r"(s[13]), "=r"(s[14]), "=r"(s[15])
        : "r"(tb));
    asm volatile("tcgen05.wait::ld.sync.aligned;"
                 : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]),
                   "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]),
                   "+r"(r[15]), "+r"(s[0]), "+r"(s[1]), "+r"(s[2]), "+r"(s[3]), "+r"(s[4]), "+r"(s[5]), "+r"(s[6]),
                   "+r"(s[7]), "+r"(s[8]), "+r"(s[9]), "+r"(s[10]), "+r"(s[11]), "+r"(s[12]), "+r"(s[13]),
                   "+r"(s[14]), "+r"(s[15])::"memory");
}
__device__ __forceinline__ void tm_ld8x2(uint32_t taddr, uint32_t (&r)[8]) {
    asm volatile("tcgen05.ld.sync.aligned.16x32bx2.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8], 8;"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
                 : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;"
                 : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7])::"memory");
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

// ---------------------------------------------------------------------------------------------
// 4: the whole prefill in one launch: one block per (sequence, head) walks its chunks in order,
//    every product on the tensor cores and the state carried in registers.  A chunk's tokens
//    fall into four blocks of 16; for a token l of block I (first token s_I, bl tokens) with S
//    the state before the block,
//      y_l = r_l^T diag(d)^{l-s_I+1} S  +  sum_{s_I <= l' <= l} (sum_m r_l[m] d_m^{l-l'} k_l'[m]) v_l',
//      S  <- diag(d)^{bl} S + U_I,   U_I = sum_{l' in I} diag(d)^{s_I+bl-1-l'} k_l' v_l'^T,
//    which is the recurrence unrolled over the block.  With value column j as the MMA's M:
//      Y_I^T = Ŝ^T Rc_I^T + V_I^T A_I^T   (N = the block's 16 tokens; K = 64 key rows, then 16 tokens)
//      U_I^T = V_I^T Kt_I                 (N = 64 key rows, K = the block's 16 tokens)
//      A     = Rc Kc^T                    (64 x 64 over the chunk; its diagonal 16 x 16 blocks, kept
//                                          where l' <= l, are the A_I)
//    with every operand scaled about its block's midpoint c_I = s_I + 8:
//      Rc[l][m] = r_l[m] d_m^{l-c_I},  Kc[l'][m] = k_l'[m] d_m^{c_I-l'},  Ŝ[m][j] = S[m][j] d_m^9,
//      Kt[m][l'] = k_l'[m] d_m^{s_I+bl-1-l'},
//    so Rc Kc^T carries d^{l-l'} inside a block and Ŝ^T Rc^T carries d^{l-s_I+1}.  No factor is
//    outside [d^8, d^-8]; a head whose fastest channel has |w| log2e > 8 (|w| > 5.5, a decay
//    below 0.004 per token) would put factors beyond 2^64 into the operands, so its block takes
//    the token-by-token form instead (decided per block, same launch).
//
//    Operands are bf16 pairs x = hi + lo (hi = x rounded to bf16, lo = the rest rounded to
//    bf16, so |x - hi - lo| <= 2^-18 |x|), each product taken as hi*hi + hi*lo + lo*hi
//    (kind::f16, fp32 accumulate; the dropped lo*lo is below 2^-18 of the term): about 2^-16
//    of each product's magnitude sum, against a fifth of that for tf32 pairs at twice the
//    instructions -- and a tcgen05.mma costs the same ~40 cycles to issue whatever its shape,
//    so the instruction count is what sets the chunk's time.  K-major operands in 8-row x
//    16-byte core matrices (8 bf16 along K): element (row, k) of a K-wide operand at byte
//    (row/8)(2K) + (k/8)128 + (row%8)16 + (k%8)2.
//
//    Roles.  Warps 0-7 build the operands from the chunk's r, k, v rows (brought by TMA with the
//    128-byte swizzle), mask and split the A_I, run the state from block to block (thread t of
//    warp w holds key rows 32 (w / 4) + 16 (t / 16) .. + 15 of value column 16 (w % 4) + t % 16)
//    and read y out into a shared tile.  Lane 0 of warp 8 issues the U_I and A and the next
//    chunk's row loads, lane 0 of warp 9 the Y_I (two issuing warps keep the tensor core fed),
//    lane 0 of warp 10 stores each y tile by TMA.  Rc and the Y accumulator have a buffer per
//    chunk parity, so the math warps build chunk c + 1's operands while chunk c's Y products
//    run, and read chunk c's y out before chunk c + 1's state chain.
//    Hand-overs are mbarriers with bounded waits: raw (a chunk's rows landed), kv (Kt and V^T
//    of a chunk written), ops (all its operands written), diag (A_I written), s123 and s0 (once
//    per chunk each: Ŝ^T of its blocks 1-3, and of the next chunk's block 0, written; block I
//    uses buffer I), yt / yf (a y tile written / stored), and tensor-core commits U, A (warp 8,
//    in that order), Y0 (block 0's Y product), diagdone (the diagonal products) and done[2]
//    (every product of warp 9 in a chunk, per chunk parity).
// ---------------------------------------------------------------------------------------------
// Per-chunk event trace of block 0 (profiling builds only): compiled with -DWKV_TRACE, the
// sequence kernel stamps %globaltimer at its hand-overs into the buffer registered with
// wkv_eagle_trace_set_buffer ([chunks][32] u64); normal builds define the hook away.
#ifdef WKV_TRACE
static __device__ unsigned long long* g_eagle_trace = nullptr;
__device__ __forceinline__ void eagle_trace(int64_t c, int ev) {
    if (!g_eagle_trace || blockIdx.x != 0) return;
    unsigned long long t;
    asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
    g_eagle_trace[c * 32 + ev] = t;
}
#define EAGLE_TRACE(c, ev) eagle_trace(c, ev)
#else
#define EAGLE_TRACE(c, ev) ((void)0)
#endif

constexpr int kSeqMath = 256;                 // warps 0-7
constexpr int kSeqWarpY = 10;                 // the y-store warp
constexpr int kSeqThreads = kSeqMath + 96;    // and the two issuing warps and the y-store warp
constexpr int kPwRows = 25;                   // d^e, e = -8 .. 16
constexpr int kPwStride = 68;                 // floats per row: consecutive rows 16 B apart in the banks
constexpr float kSeqMaxW2 = 8.f;              // |w| log2e admitted by the scaled form
constexpr int64_t kSeqMinHeads = 24;          // sequence-heads from which the one-launch form is used
constexpr int64_t kSeqMaxChunksAnyHeads = 8;  // ... and chunks per sequence up to which it always is

constexpr uint32_t kBOp = 64 * 64 * 2;                 // one bf16 64 x 64 operand part (8 KB)
constexpr uint32_t kSqRc = 0;                          // Rc hi, lo    [l][m], buffers 0 and 1 (chunk parity)
constexpr uint32_t kSqKc = 4 * kBOp;                   // Kc hi, lo    [l'][m]
constexpr uint32_t kSqKt = 6 * kBOp;                   // Kt hi, lo    [m][l']
constexpr uint32_t kSqVt = 8 * kBOp;                   // V^T hi, lo   [j][l']
constexpr uint32_t kSqS = 10 * kBOp;                   // Ŝ^T hi, lo   [j][m], buffers 0 .. 3
constexpr uint32_t kSqAd = 18 * kBOp;                  // A_I hi (4 x 512 B), then lo
constexpr uint32_t kSqPw = kSqAd + 4096;               // d^e table
constexpr uint32_t kSqW2 = kSqPw + kPwRows * kPwStride * 4;  // w log2e of the head's 64 channels
constexpr uint32_t kSqBar = kSqW2 + 64 * 4;            // mbarriers, the TMEM address, the form flag
constexpr uint32_t kSqY = (kSqBar + 256 + 1023) / 1024 * 1024;  // y tile [64 tokens][64 columns], TMA store source
constexpr uint32_t kSqRaw = kSqY + kTileBytes;         // the chunk's r, k, v rows: 6 boxes [64 tokens][32 channels]
constexpr uint32_t kRawBox = kEL * 32 * 4;             // 8 KB, 128-byte rows with the 128-byte swizzle
constexpr size_t kSqSmem = kSqRaw + 6 * kRawBox;
static_assert(kSqY % 1024 == 0 && kSqS % 1024 == 0 && kSqAd % 1024 == 0 && kSqRaw % 1024 == 0,
              "operand and TMA buffers 1 KB aligned");
static_assert(kSqSmem <= 232448, "shared memory of one block");
// the token-by-token form stages r, k, v and its partial sums in the operand area
static_assert(2 * kTileBytes + 4 * kTileBytes <= kSqPw, "token-by-token staging fits below the table");

constexpr uint32_t kColA = 0, kColU = 64, kColY = 320, kSeqCols = 512;  // TMEM columns (Y: two buffers of 64)

enum { kBarOps = 0, kBarKV, kBarDiag, kBarS0, kBarS123, kBarA, kBarU, kBarY0, kBarDiagDone, kBarDone, kBarRaw = kBarDone + 2,
       kBarYT, kBarYF, kNumSeqBars };
static_assert(kNumSeqBars * 8 + 8 <= 256, "barriers, TMEM address and form flag fit their area");

// bf16 K-major operand index (in elements) of (row, k) for a K-wide operand
template <int K>
__device__ __forceinline__ int bop_index(int row, int k) {
    return (row >> 3) * (8 * K) + (k >> 3) * 64 + (row & 7) * 8 + (k & 7);
}

// Byte offset of (token l, channel ch of the head) in the raw stage: box 2 x + ch / 32 of the
// tensor x (r 0, k 1, v 2), 128-byte rows, the 16-byte chunk index XORed with l % 8 (the
// TMA's 128-byte swizzle, so that eight rows' same chunk and one row's eight chunks both fall
// in eight different bank groups).
__device__ __forceinline__ uint32_t raw_off(int x, int l, int ch) {
    return (uint32_t)(2 * x + (ch >> 5)) * kRawBox + (uint32_t)l * 128u + ((((ch & 31) >> 2) ^ (l & 7)) << 4) + ((ch & 3) << 2);
}

__device__ __forceinline__ uint64_t op_desc_sbo(uint32_t saddr, uint32_t sbo) {
    return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)(128u >> 4) << 16) | ((uint64_t)(sbo >> 4) << 32) |
           ((uint64_t)1 << 46);
}

// instruction descriptor: fp32 accumulate, bf16 A and B, both K-major, M x N
__host__ __device__ constexpr uint32_t bf16_idesc(int M, int N) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

__device__ __forceinline__ void mma_bf16(uint32_t tmem_d, uint64_t ad, uint64_t bd, uint32_t idesc, uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
        "l"(ad), "l"(bd), "r"(idesc), "r"(acc));
}

// A split product over NK K-steps of 16 into TMEM column d: per step hi*hi + hi*lo + lo*hi, A
// and B advancing by 256 B (two core-matrix columns); acc0 = 0 starts the accumulator afresh.
// The descriptors arrive whole (start address / 16 in the low bits): a step adds 16 to them.
template <int NK>
__device__ __forceinline__ void mma_product(uint32_t d, uint64_t da, uint64_t da_lo, uint64_t db, uint64_t db_lo,
                                            uint32_t idesc, uint32_t acc0) {
#pragma unroll
    for (uint32_t ks = 0; ks < NK; ++ks) {
        const uint64_t o = 16u * ks;
        mma_bf16(d, da + o, db + o, idesc, (ks > 0 || acc0) ? 1u : 0u);
        mma_bf16(d, da + o, db_lo + o, idesc, 1);
        mma_bf16(d, da_lo + o, db + o, idesc, 1);
    }
}

// x = hi + lo as bf16 pairs, packed two to a word (first element in the low half)
__device__ __forceinline__ void split_bf16x2(float x0, float x1, uint32_t& hi, uint32_t& lo) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(x0, x1);
    const float2 hf = __bfloat1622float2(h);
    const __nv_bfloat162 l = __floats2bfloat162_rn(x0 - hf.x, x1 - hf.y);
    hi = *reinterpret_cast<const uint32_t*>(&h);
    lo = *reinterpret_cast<const uint32_t*>(&l);
}

// eight consecutive elements (one 16-byte core-matrix row) split and stored as hi and lo
__device__ __forceinline__ void store_split8(unsigned char* hi, unsigned char* lo, const float (&x)[8]) {
    uint4 h, l;
    split_bf16x2(x[0], x[1], h.x, l.x);
    split_bf16x2(x[2], x[3], h.y, l.y);
    split_bf16x2(x[4], x[5], h.z, l.z);
    split_bf16x2(x[6], x[7], h.w, l.w);
    *reinterpret_cast<uint4*>(hi) = h;
    *reinterpret_cast<uint4*>(lo) = l;
}

__device__ __forceinline__ void seq_wait(const EagleArgs& a, uint64_t* bar, uint32_t parity) {
    if (!mbar_wait(bar, parity, a.spin_limit)) atomicCAS(a.dev_err, kDevOk, (uint32_t)kDevTimeoutCopy);
}

// The token-by-token form for a head outside the scaled form's range: threads (column j, key
// rows 16 mq .. + 15) carry their state entries; a chunk's r and k rows are staged in shared
// memory (v is read per token) and each token's read-out is summed over the four row groups
// there.
__device__ void eagle_seq_tokens(const EagleArgs& a, unsigned char* smem, const float* pw, int64_t b, int64_t h) {
    float* rs = reinterpret_cast<float*>(smem);  // [64][64] each: r and k rows of the chunk
    float* ks = rs + 4096;
    float* red = ks + 4096;  // [4][64][64] partial read-outs
    const int tid = threadIdx.x, j = tid & 63, mq = (tid >> 6) & 3;
    const bool math = tid < kSeqMath;
    const int64_t sb = (b * a.H + h) * kSS;
    float S[16], dm[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        const int m = 16 * mq + i;
        dm[i] = pw[9 * kPwStride + m];  // d^1
        S[i] = (math && a.state_in) ? a.state_in[sb + m * kHead + j] : 0.f;
    }
    for (int64_t c = 0; c < a.P; ++c) {
        const int64_t t0 = c * kEL;
        const int len = (int)min64(kEL, a.T - t0);
        const int64_t row0 = (b * a.T + t0) * a.C + h * kHead;
        __syncthreads();  // the previous chunk's tiles and sums are consumed
        if (math)
            for (int idx = tid; idx < 2 * kEL * 16; idx += kSeqMath) {
                const int arr = idx / (kEL * 16), l = (idx / 16) % kEL, q4 = idx % 16;
                const float* src = arr == 0 ? a.r : a.k;
                float* dst = arr == 0 ? rs : ks;
                const float4 x = l < len ? *reinterpret_cast<const float4*>(src + row0 + (int64_t)l * a.C + 4 * q4)
                                         : make_float4(0.f, 0.f, 0.f, 0.f);
                *reinterpret_cast<float4*>(dst + l * kHead + 4 * q4) = x;
            }
        __syncthreads();
        if (math)
            for (int l = 0; l < len; ++l) {
                const float vj = a.v[row0 + (int64_t)l * a.C + j];
                float acc = 0.f;
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const int m = 16 * mq + i;
                    S[i] = fmaf(dm[i], S[i], ks[l * kHead + m] * vj);
                    acc = fmaf(rs[l * kHead + m], S[i], acc);
                }
                red[(mq * kEL + l) * kHead + j] = acc;
            }
        __syncthreads();
        if (math)
            for (int idx = tid; idx < len * kHead; idx += kSeqMath) {
                const int l = idx >> 6, jj = idx & 63;
                a.y[row0 + (int64_t)l * a.C + jj] = (red[l * kHead + jj] + red[(kEL + l) * kHead + jj]) +
                                                    (red[(2 * kEL + l) * kHead + jj] + red[(3 * kEL + l) * kHead + jj]);
            }
    }
    if (math && a.state_out)
#pragma unroll
        for (int i = 0; i < 16; ++i) a.state_out[sb + (16 * mq + i) * kHead + j] = S[i];
}

__global__ void __launch_bounds__(kSeqThreads, 1) eagle_seq_tc(EagleArgs a, const __grid_constant__ CUtensorMap tmr,
                                                                 const __grid_constant__ CUtensorMap tmk,
                                                                 const __grid_constant__ CUtensorMap tmv,
                                                                 const __grid_constant__ CUtensorMap tmy) {
    extern __shared__ __align__(1024) unsigned char smem[];
    float* const pw = reinterpret_cast<float*>(smem + kSqPw);
    float* const w2s = reinterpret_cast<float*>(smem + kSqW2);
    uint64_t* const bars = reinterpret_cast<uint64_t*>(smem + kSqBar);
    uint32_t* const tslot = reinterpret_cast<uint32_t*>(bars + kNumSeqBars);
    int& s_tokens = *reinterpret_cast<int*>(tslot + 1);  // 1: this head takes the token-by-token form
    float* const ytile = reinterpret_cast<float*>(smem + kSqY);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t b = blockIdx.x / a.H, h = blockIdx.x % a.H;
    if (tid == 0) s_tokens = 0;
    __syncthreads();
    if (tid < kHead) {
        const float w2 = a.w[h * kHead + tid] * kLog2e;
        w2s[tid] = w2;
        if (!(fabsf(w2) <= kSeqMaxW2)) s_tokens = 1;
    }
    if (tid == 0) {
        for (int i = 0; i < kNumSeqBars; ++i)
            mbar_init(&bars[i], (i == kBarOps || i == kBarKV || i == kBarDiag || i == kBarS0 || i == kBarS123 || i == kBarYT)
                                    ? kSeqMath : 1);
        fence_mbar_init();
    }
    __syncthreads();
    // d^e for e = -8 .. 16 (exact integer multiples of w; within 2^{+-64} for an admitted head)
    for (int idx = tid; idx < kPwRows * kHead; idx += kSeqThreads) {
        const int e = idx / kHead - 8, m = idx % kHead;
        pw[(e + 8) * kPwStride + m] = ex2(-(float)e * w2s[m]);
    }
    const bool tokens = s_tokens != 0;
    if (!tokens && warp == 8) tm_alloc(tslot, kSeqCols);
    tm_fence_before();
    __syncthreads();
    tm_fence_after();
    if (tokens) {
        eagle_seq_tokens(a, smem, pw, b, h);
        return;
    }
    const uint32_t tmem = *tslot;
    const uint32_t sm = smem_u32(smem);
    const int64_t P = a.P;

    if (warp == kSeqWarpY) {
        // ---- lane 0 of warp 10: each chunk's y tile to global memory by one TMA store (rows past
        // T clipped), the tile handed back once the store has read it ----
        if (lane == 0) {
            for (int64_t c = 0; c < P; ++c) {
                seq_wait(a, &bars[kBarYT], (uint32_t)(c & 1));
                tma_store_3d(&tmy, ytile, (int)(h * kHead), (int)(c * kEL), (int)b);
                bulk_commit();
                bulk_wait_read();
                mbar_arrive(&bars[kBarYF]);
            }
            bulk_wait_all();  // the last stores are complete before the block exits
        }
        __syncwarp();
    } else if (warp >= 8) {
        // ---- lane 0 of warp 8: A and the U_I; lane 0 of warp 9: the Y_I ----
        if (lane == 0) {
            constexpr uint32_t id64 = bf16_idesc(64, 64), id16 = bf16_idesc(64, 16);
            // the chunk's r, k, v rows by TMA (rows past T read as zeros), one chunk ahead
            auto load_raw = [&](int64_t c) {
                mbar_arrive_expect_tx(&bars[kBarRaw], 6 * kRawBox);
                const CUtensorMap* maps[3] = {&tmr, &tmk, &tmv};
#pragma unroll
                for (int x = 0; x < 3; ++x)
#pragma unroll
                    for (int hb = 0; hb < 2; ++hb)
                        tma_load_3d(smem + kSqRaw + (2 * x + hb) * kRawBox, maps[x], (int)(h * kHead + 32 * hb),
                                    (int)(c * kEL), (int)b, &bars[kBarRaw]);
            };
            if (warp == 8) load_raw(0);
            for (int64_t c = 0; c < P; ++c) {
                const uint32_t par = (uint32_t)(c & 1);
                // base descriptors, re-derived each chunk through an opaque move so that no
                // table of descriptors stays live across the loop
                uint64_t q1k = op_desc_sbo(sm, 1024), q256 = op_desc_sbo(sm, 256);
                asm volatile("" : "+l"(q1k), "+l"(q256));
                auto D = [&](uint32_t off) { return q1k + (off >> 4); };
                if (warp == 8) {
                    seq_wait(a, &bars[kBarKV], par);
                    tm_fence_after();
                    EAGLE_TRACE(c, 0);
                    // U_I^T = V_I^T Kt_I (M = 64 columns, N = 64 key rows, K = the block's 16 tokens),
                    // as soon as Kt and V^T are written: the state chain waits for it
#pragma unroll
                    for (uint32_t I = 0; I < 4; ++I)
                        mma_product<1>(tmem + kColU + 64 * I, D(kSqVt + 256 * I), D(kSqVt + kBOp + 256 * I),
                                       D(kSqKt + 256 * I), D(kSqKt + kBOp + 256 * I), id64, 0);
                    mma_commit(&bars[kBarU]);
                    EAGLE_TRACE(c, 9);
                    // A = Rc Kc^T (M = N = 64 tokens, K = 64 key rows)
                    seq_wait(a, &bars[kBarOps], par);
                    tm_fence_after();
                    const uint32_t rc = kSqRc + 2 * kBOp * (uint32_t)(c & 1);
                    mma_product<4>(tmem + kColA, D(rc), D(rc + kBOp), D(kSqKc), D(kSqKc + kBOp), id64, 0);
                    mma_commit(&bars[kBarA]);
                    EAGLE_TRACE(c, 1);
                    if (c + 1 < P) load_raw(c + 1);  // the raw stage is consumed
                } else {
                    // Y_0^T: the state part of block 0
                    const uint32_t ty = tmem + kColY + 64 * (uint32_t)(c & 1);  // Y buffer of the chunk
                    const uint32_t rc = kSqRc + 2 * kBOp * (uint32_t)(c & 1);
                    seq_wait(a, &bars[kBarOps], par);
                    seq_wait(a, &bars[kBarS0], par);  // Ŝ^T of block 0 (written at the end of the last chunk's chain)
                    tm_fence_after();
                    mma_product<4>(ty, D(kSqS), D(kSqS + kBOp), D(rc), D(rc + kBOp), id16, 0);
                    mma_commit(&bars[kBarY0]);
                    EAGLE_TRACE(c, 2);
                    // the diagonal blocks: Y_I^T += V_I^T A_I^T (K = the block's 16 tokens)
                    seq_wait(a, &bars[kBarDiag], par);
                    tm_fence_after();
                    EAGLE_TRACE(c, 3);
#pragma unroll
                    for (uint32_t I = 0; I < 4; ++I) {
                        const uint64_t ob = q256 + ((kSqAd + 512 * I) >> 4);
                        mma_product<1>(ty + 16 * I, D(kSqVt + 256 * I), D(kSqVt + kBOp + 256 * I), ob,
                                       ob + (2048 >> 4), id16, I == 0 ? 1u : 0u);
                    }
                    mma_commit(&bars[kBarDiagDone]);
                    // blocks 1-3: the state part, once the chain has written the states before them
                    seq_wait(a, &bars[kBarS123], par);
                    tm_fence_after();
                    EAGLE_TRACE(c, 5);
#pragma unroll 1
                    for (uint32_t I = 1; I < 4; ++I) {
                        const uint32_t sb = kSqS + 2 * kBOp * I;
                        const uint64_t orow = (2048u * I) >> 4;  // the block's 16 rows of Rc
                        mma_product<4>(ty + 16 * I, D(sb), D(sb + kBOp), D(rc) + orow, D(rc + kBOp) + orow, id16, 1);
                    }
                    mma_commit(&bars[kBarDone + (c & 1)]);
                    EAGLE_TRACE(c, 8);
                }
            }
        }
        __syncwarp();
    } else {
        // ---- warps 0-7 ----
        // An M = 64 accumulator row j sits in lane j % 16 of quadrant j / 16; the 16x32bx2 loads
        // hand a warp's threads 0-15 those 16 lanes at one column range and threads 16-31 the
        // same lanes 16 (or 8) columns on, so every thread of warps 0-7 holds data.
        const int q = warp & 3, hf = warp >> 2, up = lane >> 4;
        const int j = 16 * q + (lane & 15);   // value column (chain and read-out)
        const int m0 = 32 * hf + 16 * up;     // key rows m0 .. m0 + 15 of this thread's state
        const uint32_t tq = tmem + ((uint32_t)(32 * q) << 16);
        const int64_t sb = (b * a.H + h) * kSS;

        // build tasks: rows (row l, eight key rows mc8 .. + 7; a warp's lanes over 8 rows x 4 groups
        // of eight) for Rc and Kc, columns (channel m, eight tokens) for Kt and V^T
        auto row_task = [&](int i, int& l, int& mc8) {  // i = 0, 1: 2 x 256 tasks
            const int task = i * kSeqMath + tid;
            const int wl = task & 31, wt = task >> 5;
            l = 8 * (wt & 7) + (wl & 7);
            mc8 = 8 * (4 * (wt >> 3) + (wl >> 3));
        };
        auto col_task = [&](int i, int& m, int& t8) {
            const int task = i * kSeqMath + tid;
            m = task & 63;
            t8 = 8 * (task >> 6);
        };

        // the state before the first block: state_in (or zero), Ŝ^T into buffer 0
        float S[16], d16[16], d9[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            S[i] = a.state_in ? a.state_in[sb + (m0 + i) * kHead + j] : 0.f;
            d16[i] = pw[24 * kPwStride + m0 + i];
            d9[i] = pw[17 * kPwStride + m0 + i];
        }
        auto write_shat = [&](int xb) {
            unsigned char* hi = smem + kSqS + 2 * kBOp * xb;
#pragma unroll
            for (int g8 = 0; g8 < 2; ++g8) {
                float x[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) x[e] = S[8 * g8 + e] * d9[8 * g8 + e];
                const int o = 2 * bop_index<64>(j, m0 + 8 * g8);
                store_split8(hi + o, hi + kBOp + o, x);
            }
        };
        write_shat(0);
        fence_proxy_async_smem();
        mbar_arrive(&bars[kBarS0]);

        // y of a chunk: read back and written to the shared tile (once the y-store warp has read
        // the previous chunk's out of it), handed to the y-store warp
        auto read_y = [&](int64_t c) {
            if (c > 0) seq_wait(a, &bars[kBarYF], (uint32_t)((c - 1) & 1));
            uint32_t r[16];
            tm_ld16x2(tq + kColY + 64 * (uint32_t)(c & 1) + 32 * hf, r);  // tokens 32 hf + 16 up ..
#pragma unroll
            for (int i = 0; i < 16; ++i) ytile[(32 * hf + 16 * up + i) * kHead + j] = __uint_as_float(r[i]);
            fence_proxy_async_smem();
            mbar_arrive(&bars[kBarYT]);
        };

        for (int64_t c = 0; c < P; ++c) {
            const uint32_t par = (uint32_t)(c & 1);
            const int len = (int)min64(kEL, a.T - c * kEL);
            // operands of this chunk from the raw stage: Kt and V^T (columns), then Rc and Kc (rows).
            // Rc goes to the buffer of the chunk's parity (its last reader, the previous chunk but one,
            // is done: its y was read out); Kc, Kt, V^T and the A_I were last read by the previous
            // chunk's A, U and diagonal products.
            if (c > 0) seq_wait(a, &bars[kBarDiagDone], par ^ 1u);
            seq_wait(a, &bars[kBarRaw], par);
            if (tid == 0) EAGLE_TRACE(c, 10);
            const uint32_t rc = kSqRc + 2 * kBOp * (uint32_t)(c & 1);
#pragma unroll
            for (int i = 0; i < 2; ++i) {
                int m, t8;
                col_task(i, m, t8);
                const int I = t8 >> 4, bl = max(0, min(16, len - 16 * I));
                float xk[8], xv[8];
#pragma unroll
                for (int s = 0; s < 8; ++s) {
                    const int li = (t8 & 15) + s;
                    const bool in = li < bl;
                    const float p = pw[(in ? bl - 1 - li + 8 : 8) * kPwStride + m];  // d^{bl-1-li}
                    const float kx = *reinterpret_cast<const float*>(smem + kSqRaw + raw_off(1, t8 + s, m));
                    xk[s] = in ? kx * p : 0.f;
                    xv[s] = *reinterpret_cast<const float*>(smem + kSqRaw + raw_off(2, t8 + s, m));
                }
                const int o = 2 * bop_index<64>(m, t8);
                store_split8(smem + kSqKt + o, smem + kSqKt + kBOp + o, xk);
                store_split8(smem + kSqVt + o, smem + kSqVt + kBOp + o, xv);
            }
            fence_proxy_async_smem();
            tm_fence_before();
            mbar_arrive(&bars[kBarKV]);  // Kt and V^T written: U may start
            if (tid == 0) EAGLE_TRACE(c, 24);
#pragma unroll
            for (int i = 0; i < 2; ++i) {
                int l, mc8;
                row_task(i, l, mc8);
                const int li = l & 15;
                const float4* pr = reinterpret_cast<const float4*>(pw + li * kPwStride + mc8);         // d^{li-8}
                const float4* pk = reinterpret_cast<const float4*>(pw + (16 - li) * kPwStride + mc8);  // d^{8-li}
                const float4 r0 = *reinterpret_cast<const float4*>(smem + kSqRaw + raw_off(0, l, mc8));
                const float4 r1 = *reinterpret_cast<const float4*>(smem + kSqRaw + raw_off(0, l, mc8 + 4));
                const float4 k0 = *reinterpret_cast<const float4*>(smem + kSqRaw + raw_off(1, l, mc8));
                const float4 k1 = *reinterpret_cast<const float4*>(smem + kSqRaw + raw_off(1, l, mc8 + 4));
                const float4 pr0 = pr[0], pr1 = pr[1], pk0 = pk[0], pk1 = pk[1];
                const float xr[8] = {r0.x * pr0.x, r0.y * pr0.y, r0.z * pr0.z, r0.w * pr0.w,
                                     r1.x * pr1.x, r1.y * pr1.y, r1.z * pr1.z, r1.w * pr1.w};
                const float xk[8] = {k0.x * pk0.x, k0.y * pk0.y, k0.z * pk0.z, k0.w * pk0.w,
                                     k1.x * pk1.x, k1.y * pk1.y, k1.z * pk1.z, k1.w * pk1.w};
                const int o = 2 * bop_index<64>(l, mc8);
                store_split8(smem + rc + o, smem + rc + kBOp + o, xr);
                store_split8(smem + kSqKc + o, smem + kSqKc + kBOp + o, xk);
            }
            if (tid == 0) EAGLE_TRACE(c, 25);
            fence_proxy_async_smem();
            tm_fence_before();
            mbar_arrive(&bars[kBarOps]);
            if (tid == 0) EAGLE_TRACE(c, 12);

            // the diagonal blocks of A, masked to l' <= l and split (warp q: block q)
            auto diag_blocks = [&]() {
                seq_wait(a, &bars[kBarA], par);
                tm_fence_after();
                if (tid == 0) EAGLE_TRACE(c, 13);
                if (warp < 4) {
                    // row l = 16 q + (lane % 16) of block q, keys 16 q + 8 up .. + 7
                    uint32_t r[8];
                    tm_ld8x2(tq + kColA + 16 * q, r);
                    const int li = lane & 15;
                    unsigned char* hi = smem + kSqAd + 512 * q;
                    float x[8];
#pragma unroll
                    for (int s = 0; s < 8; ++s) x[s] = (8 * up + s <= li) ? __uint_as_float(r[s]) : 0.f;
                    const int o = 2 * bop_index<16>(li, 8 * up);
                    store_split8(hi + o, hi + 2048 + o, x);
                    fence_proxy_async_smem();
                }
                tm_fence_before();
                mbar_arrive(&bars[kBarDiag]);
                if (tid == 0) EAGLE_TRACE(c, 14);
            };

            // the previous chunk's y: its products ran behind this chunk's operands; once they are
            // done, the Ŝ^T buffers of blocks 1-3 are free as well
            if (c > 0) {
                seq_wait(a, &bars[kBarDone + ((c - 1) & 1)], (uint32_t)(((c - 1) >> 1) & 1));
                tm_fence_after();
                if (tid == 0) EAGLE_TRACE(c, 11);
                read_y(c - 1);
            }

            // the state from block to block: Ŝ^T of blocks 1-3 and of the next chunk's block 0 into
            // their buffers, handed over together at the end (the diagonal blocks in between, after
            // the first block's state)
            seq_wait(a, &bars[kBarU], par);
            tm_fence_after();
            if (tid == 0) EAGLE_TRACE(c, 15);
#pragma unroll 1
            for (int I2 = 0; I2 < 4; I2 += 2) {
                uint32_t u[2][16];
                tm_ld16x2_pair(tq + kColU + 64 * I2 + 32 * hf, tq + kColU + 64 * (I2 + 1) + 32 * hf, u[0], u[1]);
#pragma unroll
                for (int k2 = 0; k2 < 2; ++k2) {
                    const int I = I2 + k2;
                    const int bl = max(0, min(16, len - 16 * I));
                    if (bl == 16) {
#pragma unroll
                        for (int i = 0; i < 16; ++i) S[i] = fmaf(d16[i], S[i], __uint_as_float(u[k2][i]));
                    } else {
                        const float* dbl = pw + (bl + 8) * kPwStride + m0;  // d^{bl}
#pragma unroll
                        for (int i = 0; i < 16; ++i) S[i] = fmaf(dbl[i], S[i], __uint_as_float(u[k2][i]));
                    }
                    if (k2 == 1) tm_fence_before();
                    if (I < 3) {
                        write_shat(I + 1);
                        if (I == 2) {  // the states before blocks 1-3
                            fence_proxy_async_smem();
                            mbar_arrive(&bars[kBarS123]);
                        }
                    } else if (c + 1 < P) {
                        seq_wait(a, &bars[kBarY0], par);  // block 0's Y product has read buffer 0
                        write_shat(0);
                        fence_proxy_async_smem();
                        mbar_arrive(&bars[kBarS0]);  // the state before the next chunk's block 0
                    }
                    if (tid == 0) EAGLE_TRACE(c, 16 + I);
                    if (I == 0) diag_blocks();
                }
            }
        }
        if (a.state_out)
#pragma unroll
            for (int i = 0; i < 16; ++i) a.state_out[sb + (m0 + i) * kHead + j] = S[i];
        seq_wait(a, &bars[kBarDone + ((P - 1) & 1)], (uint32_t)(((P - 1) >> 1) & 1));
        tm_fence_after();
        read_y(P - 1);
    }
    tm_fence_before();
    __syncthreads();
    if (warp == 8) {
        tm_fence_after();
        tm_dealloc(tmem, kSeqCols);
    }
}

}  // namespace

int64_t eagle_chunks(int64_t T) { return (T + kEL - 1) / kEL; }

#ifdef WKV_TRACE
extern "C" void wkv_eagle_trace_set_buffer(void* buf) {
    unsigned long long* p = static_cast<unsigned long long*>(buf);
    cudaMemcpyToSymbol(g_eagle_trace, &p, sizeof(p));
}
#endif

bool eagle_uses_sequence_kernel(int64_t B, int64_t T, int64_t C) {
    // one block per (sequence, head) walking its chunks in order, against three launches over all
    // chunk-heads at once: the former wins unless a few heads carry long sequences
    const int64_t heads = B * (C / kHead);
    return heads >= kSeqMinHeads || eagle_chunks(T) <= kSeqMaxChunksAnyHeads;
}

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
        e = cudaFuncSetAttribute(eagle_seq_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSqSmem);
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
    if (eagle_uses_sequence_kernel(B, T, C)) {
        CUtensorMap tmy, tsr, tsk, tsv;
        if (!make_tile_map(&tmy, y, B, T, C, 0, kHead, kEL) || !make_tile_map(&tsr, r, B, T, C, 0, 32, kEL, true) ||
            !make_tile_map(&tsk, k, B, T, C, 0, 32, kEL, true) || !make_tile_map(&tsv, v, B, T, C, 0, 32, kEL, true))
            return cudaErrorInvalidValue;
        eagle_seq_tc<<<(unsigned)(B * H), kSeqThreads, kSqSmem, s>>>(a, tsr, tsk, tsv, tmy);
        return cudaGetLastError();
    }
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
