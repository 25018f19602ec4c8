// Host-side launch interface between the C ABI (wkv_abi.cu) and the kernel files.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <utility>

namespace wkvb {

// Device error codes written to the error word (first word of a status block).
enum : uint32_t { kDevOk = 0, kDevTimeoutCarry = 1, kDevTimeoutCopy = 2, kDevBadWorkspace = 3 };

// Bounded-wait limits (iterations of a poll loop that sleeps ~64 ns per miss).
constexpr uint32_t kSpinLimitDefault = 1u << 18;  // a few hundred ms of polling
// Kernels that wait for their stream predecessor in-kernel (grid_dep_wait) are launched with
// programmatic stream serialisation, so their launch and prologue overlap its tail.
constexpr bool kProgrammaticLaunch = true;

// Launches kern with programmatic stream serialisation; every kernel launched this way calls
// grid_dep_wait before its first access to global memory.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                              Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[0].val.programmaticStreamSerializationAllowed = kProgrammaticLaunch ? 1 : 0;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

struct ForwardArgs {
    int64_t B, T, C;
    int io;                 // 0 fp32, 1 bf16
    const float* w;         // [C]
    const float* u;         // [C]
    const void* k;          // [B,T,C]
    const void* v;          // [B,T,C]
    const float* state_in;  // [3][B][C] or null
    void* y;                // [B,T,C]
    float* state_out;       // [3][B][C] or null
    uint32_t* err;          // device error word (never null)
    uint32_t* dev_err;      // the library's device-wide error word (never null)
    const void* r = nullptr;  // [B,T,C] receptance for a fused output gate, or null
    uint32_t spin_limit;    // bounded waits
};

// The library's device-wide error word on the current device (null if it cannot be found):
// every kernel that gives up a bounded wait also records its code here, for
// wkv_get_device_status.
uint32_t* device_status_word();

// Records e as the host thread's last CUDA error (reported by wkv_last_cuda_error) and
// returns the WKV_ERR_CUDA status code, for entry points outside the main ABI file.
int record_cuda_error(cudaError_t e);

// ----- serial path: one thread per (b, c) -----
cudaError_t launch_forward_serial(const ForwardArgs& a, cudaStream_t s);

// ----- chunked path -----
struct ChunkGeom {
    int V;        // channels per thread
    int NW;       // warps per CTA (= chunks per tile)
    int LC;       // time steps per chunk
    bool bulk;    // rows copied with cp.async.bulk
    bool pipe;    // persistent warp-specialised kernel (wkv_forward_tmem.cu)
    int64_t Cg;   // channels per tile (32 * V)
    int64_t Ts;   // time steps per tile (NW * LC)
    int64_t groups_per_b;
    int64_t G;    // channel groups = B * groups_per_b
    int64_t S;    // time segments
    int64_t U;    // units = G * S
    size_t ws_bytes;
};

// Returns false if the configuration is unsupported (e.g. chunk length).
bool chunk_geometry(int64_t B, int64_t T, int64_t C, int io, int chunk, ChunkGeom* g);

// Workspace layout: [header 64 B][flags U x u32, padded to 16 B][agg U*Cg float4][incl U*Cg float4]
constexpr size_t kWsHeaderBytes = 64;
struct WsHeader {
    uint32_t error;       // kDev* code of the first failure (first word: the status word)
    uint32_t error_unit;
    uint32_t ticket;      // next unit to hand out (reset by the last CTA)
    uint32_t done;        // finished CTAs (reset by the last CTA)
    uint32_t epoch;       // launches completed on this workspace (advanced by the last CTA)
    uint32_t pad[11];
};

// Test hook: drop_unit >= 0 makes that unit skip publishing its carry, so that its
// successor's bounded wait runs out.
// Look-back flags carry the launch's epoch (read from the workspace header on the device,
// so a launch captured in a CUDA graph stays correct on every replay).
// Whether the kernel this geometry selects applies a receptance gate itself (ForwardArgs::r).
bool chunked_path_fuses_gate(const ChunkGeom& g);
cudaError_t launch_forward_chunked(const ForwardArgs& a, const ChunkGeom& g, void* ws, int64_t drop_unit,
                                   cudaStream_t s);

// Persistent warp-specialised variant (bulk rows, chunk 8 or 16); same workspace layout.
cudaError_t launch_token_shift3(int64_t B, int64_t T, int64_t C, const float* mu_r, const float* mu_k,
                                const float* mu_v, const float* x, const float* x_last, float* xr, float* xk, float* xv,
                                cudaStream_t s);
// y <- sigma(r) * y over n elements of dtype io (0 fp32, 1 bf16), in place
cudaError_t launch_gate(int64_t n, int io, const void* r, void* y, cudaStream_t s);

// WKV backward (fp32): gk, gv [B,T,C]; gw, gu [C] (zeroed, then accumulated); ws (zero-filled) holds
// backward_workspace_bytes(B, T, C); backward_fits says whether one launch's grid holds the shape
int64_t backward_segments(int64_t T);
bool backward_fits(int64_t B, int64_t T, int64_t C);
size_t backward_workspace_bytes(int64_t B, int64_t T, int64_t C);
cudaError_t launch_backward(int64_t B, int64_t T, int64_t C, const float* w, const float* u, const float* k,
                            const float* v, const float* gy, float* gk, float* gv, float* gw, float* gu, void* ws,
                            cudaStream_t s);

cudaError_t launch_forward_tmem(const ForwardArgs& a, const ChunkGeom& g, void* ws, int64_t drop_unit,
                                cudaStream_t s);

// ----- T == 0: state_out = state_in (or the empty state) -----
cudaError_t launch_state_passthrough(int64_t BC, const float* state_in, float* state_out, cudaStream_t s);

// ----- decode / token shift -----
cudaError_t launch_decode_step(int64_t N, int64_t L, int64_t C, const float* mu, const float* w, const float* u,
                               const float* x_t, const float* x_prev, float* xbar, const float* k,
                               const float* v, float* state, float* y, cudaStream_t s);
cudaError_t launch_token_shift(int64_t B, int64_t T, int64_t C, const float* mu, const float* x,
                               const float* x_last, float* xbar, cudaStream_t s);

}  // namespace wkvb
