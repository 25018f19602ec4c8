// Launchers of the Eagle (RWKV-5) matrix-state kernels (wkv_eagle.cu), called by the C ABI
// after it has validated every argument.
#pragma once
#include <cstdint>

#include <cuda_runtime.h>

namespace wkvb {

// Chunks of the prefill's time-parallel form (tokens per chunk: 64).
int64_t eagle_chunks(int64_t T);

// True when the prefill of this shape runs as one launch of one block per (sequence, head)
// (eagle_seq_tc); otherwise three launches over all chunk-heads (chunk sums, state scan, outputs).
bool eagle_uses_sequence_kernel(int64_t B, int64_t T, int64_t C);

// Prefill over [B, T, C] (C a multiple of 64); ws holds B * H * eagle_chunks(T) * 64 * 64 floats.
cudaError_t launch_eagle_forward(int64_t B, int64_t T, int64_t C, const float* w, const float* r, const float* k,
                                 const float* v, const float* state_in, float* y, float* state_out, void* ws,
                                 cudaStream_t s);

// One token for N * L rows of C channels, parameters [L][C], state [N][L][C / 64][64][64].
cudaError_t launch_eagle_decode(int64_t N, int64_t L, int64_t C, const float* w, const float* r, const float* k,
                                const float* v, float* state, float* y, cudaStream_t s);

}  // namespace wkvb
