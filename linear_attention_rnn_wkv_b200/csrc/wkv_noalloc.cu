// A chunked forward that needs no caller-provided workspace and allocates nothing.
//
// Who this is for: code that may not call cudaMalloc at all -- for example a caller
// running inside another framework's memory pool or under a strict memory budget, an
// embedding that must not grow device memory after start-up, or a host thread that is
// not allowed to make allocation calls while other work runs.  Such callers still
// own their inputs and outputs; only the chunked path's scratch (tile flags and carry
// records) moves into a fixed array that lives in this library.
//
// The scratch is one file-scope device array of kNoAllocScratchBytes (32 MiB).  Every
// GPU that loads the library holds it until the process exits.  All calls on a device
// share it, and it keeps the previous call's contents, so:
//  * two calls that can run at the same time on the GPU (different streams without an
//    ordering between them) race on it and give wrong results; order such calls;
//  * each call clears the header words that must start at zero (error word and the
//    tile-ticket and completion counters) before its kernel runs; the flags need no
//    clearing because every launch tags them with a new epoch kept in the header.
// Host code cannot use the array's name as a device address (in host code it names a
// host-side stand-in), so the first call on each device looks up the real address
// with cudaGetSymbolAddress while that device is current and caches it.  Make that
// first call outside any stream capture.  A device-side wait that runs out (possible
// only when calls overlap) is recorded in the array's header, which the next call
// clears, and in the library's device-wide error word, which wkv_get_device_status
// reports (and clears).
#include <mutex>

#include "wkv.h"
#include "wkv_device.cuh"
#include "wkv_internal.h"

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(32) << 20;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_setup_mutex;
void* g_scratch_addr[kMaxDevices] = {nullptr};

// Device address of the scratch array for the current device (set up once per device).
cudaError_t scratch_for_current_device(void** out, cudaStream_t stream) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    if (!g_scratch_addr[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return e;
        // start from an all-zero array once (header, epoch and flags)
        e = cudaMemsetAsync(p, 0, kNoAllocScratchBytes, stream);
        if (e != cudaSuccess) return e;
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
    return cudaSuccess;
}

}  // namespace

extern "C" wkv_status wkv_forward_chunked_noalloc(int64_t B, int64_t T, int64_t C, wkv_dtype io, const float* w,
                                                  const float* u, const void* k, const void* v,
                                                  const float* state_in, void* y, float* state_out,
                                                  cudaStream_t stream) {
    using namespace wkvb;
    if (B < 0 || T < 0 || C < 0) return WKV_ERR_INVALID_ARG;
    if (io != WKV_F32 && io != WKV_BF16) return WKV_ERR_UNSUPPORTED;
    if (B == 0 || C == 0) return WKV_OK;  // no channels: nothing to compute
    if (B > INT64_MAX / C || B * C > INT64_MAX / 3) return WKV_ERR_INVALID_ARG;
    if (T > 0 && B * C > INT64_MAX / T) return WKV_ERR_INVALID_ARG;
    auto al = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; };
    if (!w || !u) return WKV_ERR_INVALID_ARG;
    if (!al(w) || !al(u) || !al(state_in) || !al(state_out)) return WKV_ERR_MISALIGNED;
    if (T == 0) {
        // no tokens: the state passes through (state_in, or the empty state), as in wkv_forward_ex
        if (!state_out) return WKV_OK;
        const cudaError_t e = launch_state_passthrough(B * C, state_in, state_out, stream);
        return e == cudaSuccess ? WKV_OK : (wkv_status)record_cuda_error(e);
    }
    if (!k || !v || !y) return WKV_ERR_INVALID_ARG;
    if (!al(k) || !al(v) || !al(y)) return WKV_ERR_MISALIGNED;

    // the default tile if its scratch fits, else the longer tile (fewer records)
    ChunkGeom g;
    bool ok = chunk_geometry(B, T, C, (int)io, 0, &g) && g.ws_bytes <= kNoAllocScratchBytes;
    if (!ok) ok = chunk_geometry(B, T, C, (int)io, 16, &g) && g.ws_bytes <= kNoAllocScratchBytes;
    if (!ok || g.U > INT32_MAX) return WKV_ERR_INVALID_ARG;  // needs more than the fixed 32 MiB scratch

    void* scratch = nullptr;
    cudaError_t e = scratch_for_current_device(&scratch, stream);
    if (e != cudaSuccess) return (wkv_status)record_cuda_error(e);
    // error word, failing unit, ticket and completion counters must start at zero; keep the epoch
    e = cudaMemsetAsync(scratch, 0, 4 * sizeof(uint32_t), stream);
    if (e != cudaSuccess) return (wkv_status)record_cuda_error(e);

    ForwardArgs a;
    a.B = B;
    a.T = T;
    a.C = C;
    a.io = (int)io;
    a.w = w;
    a.u = u;
    a.k = k;
    a.v = v;
    a.state_in = state_in;
    a.y = y;
    a.state_out = state_out;
    a.err = static_cast<uint32_t*>(scratch);
    a.dev_err = device_status_word();
    if (!a.dev_err) return (wkv_status)record_cuda_error(cudaGetLastError());
    a.spin_limit = kSpinLimitDefault;
    e = launch_forward_chunked(a, g, scratch, -1, stream);
    return e == cudaSuccess ? WKV_OK : (wkv_status)record_cuda_error(e);
}
