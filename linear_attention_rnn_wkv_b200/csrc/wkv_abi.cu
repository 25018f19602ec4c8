// C ABI of the WKV library: argument validation, path choice, launches.
// Declarations and the contract of every entry point are in include/wkv.h.
#include <atomic>
#include <cstdint>
#include <cstring>

#include "wkv.h"
#include "wkv_device.cuh"
#include "wkv_eagle_internal.h"
#include "wkv_internal.h"
#include "wkv_path_table.h"

#include <cmath>

namespace {

using namespace wkvb;

thread_local int g_last_cuda_error = 0;

// Library-owned status block: words 0-1 are the error code and failing unit of launches
// that run without a workspace (the serial path); word 2 is the device-wide error word
// every kernel also records its first timeout in (wkv_get_device_status).
__device__ uint32_t g_status_block[4];

wkv_status cuda_fail(cudaError_t e) {
    g_last_cuda_error = (int)e;
    return WKV_ERR_CUDA;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool mul_ok(int64_t a, int64_t b, int64_t* out) {
    if (a < 0 || b < 0) return false;
    if (a != 0 && b > INT64_MAX / a) return false;
    *out = a * b;
    return true;
}

bool sizes_ok(int64_t A, int64_t B, int64_t C, int64_t* total) {
    int64_t ab;
    return mul_ok(A, B, &ab) && mul_ok(ab, C, total);
}

uint32_t* status_word() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return nullptr;
    static uint32_t* cache[64] = {nullptr};
    if (dev < 0 || dev >= 64) return nullptr;
    if (!cache[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_status_block) != cudaSuccess) return nullptr;
        cache[dev] = static_cast<uint32_t*>(p);
    }
    return cache[dev];
}

}  // namespace

uint32_t* wkvb::device_status_word() {
    uint32_t* w = status_word();
    return w ? w + 2 : nullptr;
}

int wkvb::record_cuda_error(cudaError_t e) { return (int)cuda_fail(e); }

namespace {

// Index of the grid value nearest to x on a log scale (ties to the larger).
template <int N>
int nearest_log(const long long (&grid)[N], int64_t x) {
    int best = 0;
    double bd = 1e300;
    const double lx = log2((double)(x > 0 ? x : 1));
    for (int i = 0; i < N; ++i) {
        const double d = fabs(log2((double)grid[i]) - lx);
        if (d <= bd) {
            bd = d;
            best = i;
        }
    }
    return best;
}

// The path (and chunk length) WKV_PATH_AUTO takes: the measured winner at the nearest grid
// point of the tuning table (wkv_path_table.h: I/O dtype, channels B*C, tokens T); a point
// too large to have been measured takes the nearest measured point with fewer tokens.
wkv_path auto_path(int64_t B, int64_t T, int64_t C, wkv_dtype io, int* chunk = nullptr) {
    const int d = io == WKV_BF16 ? 1 : 0;
    const int ib = nearest_log(kTuneBC, B * C);
    int it = nearest_log(kTuneT, T);
    while (it > 0 && kTunePath[d][ib][it] == 0) --it;
    const int code = kTunePath[d][ib][it];
    if (chunk) *chunk = code == 8 ? 8 : 16;
    return code == 1 ? WKV_PATH_SERIAL : WKV_PATH_CHUNKED;
}

wkv_status forward_impl(int64_t B, int64_t T, int64_t C, wkv_dtype io, const float* w, const float* u,
                        const void* k, const void* v, const float* state_in, void* y, float* state_out,
                        void* workspace, size_t ws_bytes, wkv_path path, int chunk, uint32_t spin_limit,
                        int64_t drop_unit, cudaStream_t stream, const void* r = nullptr) {
    int64_t n = 0, BC = 0;
    if (!sizes_ok(B, T, C, &n) || !mul_ok(B, C, &BC) || BC > INT64_MAX / 3) return WKV_ERR_INVALID_ARG;
    if (io != WKV_F32 && io != WKV_BF16) return WKV_ERR_UNSUPPORTED;
    if (path != WKV_PATH_AUTO && path != WKV_PATH_SERIAL && path != WKV_PATH_CHUNKED) return WKV_ERR_UNSUPPORTED;
    if (chunk != 0 && chunk != 4 && chunk != 8 && chunk != 16) return WKV_ERR_UNSUPPORTED;
    if (BC == 0) return WKV_OK;
    if (!w || !u) return WKV_ERR_INVALID_ARG;
    if (!aligned16(w) || !aligned16(u) || !aligned16(state_in) || !aligned16(state_out) || !aligned16(workspace))
        return WKV_ERR_MISALIGNED;
    if (T == 0) {
        if (!state_out) return WKV_OK;
        cudaError_t e = launch_state_passthrough(BC, state_in, state_out, stream);
        return e == cudaSuccess ? WKV_OK : cuda_fail(e);
    }
    if (!k || !v || !y) return WKV_ERR_INVALID_ARG;
    if (!aligned16(k) || !aligned16(v) || !aligned16(y) || !aligned16(r)) return WKV_ERR_MISALIGNED;

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
    a.spin_limit = spin_limit;

    if (path == WKV_PATH_AUTO) {
        int tuned_chunk = 16;
        path = auto_path(B, T, C, io, &tuned_chunk);
        if (chunk == 0) chunk = tuned_chunk;
    }
    if (path == WKV_PATH_SERIAL) {
        a.err = workspace && ws_bytes >= kWsHeaderBytes ? &static_cast<WsHeader*>(workspace)->error : status_word();
        a.dev_err = device_status_word();
        if (!a.err || !a.dev_err) return cuda_fail(cudaGetLastError());
        const int64_t grid = B * ((C + 127) / 128);
        if (grid > INT32_MAX) return WKV_ERR_UNSUPPORTED;
        cudaError_t e = launch_forward_serial(a, stream);
        if (e == cudaSuccess && r) e = launch_gate(n, (int)io, r, y, stream);
        return e == cudaSuccess ? WKV_OK : cuda_fail(e);
    }
    ChunkGeom g;
    if (!chunk_geometry(B, T, C, (int)io, chunk, &g)) return WKV_ERR_UNSUPPORTED;
    if (g.U > INT32_MAX) return WKV_ERR_UNSUPPORTED;
    if (!workspace || ws_bytes < g.ws_bytes) return WKV_ERR_INVALID_ARG;
    a.err = &static_cast<WsHeader*>(workspace)->error;
    a.dev_err = device_status_word();
    if (!a.dev_err) return cuda_fail(cudaGetLastError());
    // the tensor-memory kernel applies the gate as it writes y; other kernels are followed
    // by an elementwise gate pass over y
    const bool fused = r && chunked_path_fuses_gate(g);
    a.r = fused ? r : nullptr;
    cudaError_t e = launch_forward_chunked(a, g, workspace, drop_unit, stream);
    if (e == cudaSuccess && r && !fused) e = launch_gate(n, (int)io, r, y, stream);
    return e == cudaSuccess ? WKV_OK : cuda_fail(e);
}

bool f32_args_ok(std::initializer_list<const void*> ps) {
    for (const void* p : ps)
        if (!aligned16(p)) return false;
    return true;
}

}  // namespace

extern "C" {

size_t wkv_forward_workspace_size(int64_t B, int64_t T, int64_t C, wkv_dtype io) {
    int64_t n = 0;
    if (!sizes_ok(B, T, C, &n) || n == 0) return kWsHeaderBytes;
    size_t best = kWsHeaderBytes;
    for (int chunk : {0, 4, 8, 16}) {
        ChunkGeom g;
        if (chunk_geometry(B, T, C, (int)io, chunk, &g) && g.ws_bytes > best) best = g.ws_bytes;
    }
    return best;
}

wkv_status wkv_workspace_init(void* workspace, size_t ws_bytes, cudaStream_t stream) {
    if (!workspace) return ws_bytes == 0 ? WKV_OK : WKV_ERR_INVALID_ARG;
    if (!aligned16(workspace)) return WKV_ERR_MISALIGNED;
    cudaError_t e = cudaMemsetAsync(workspace, 0, ws_bytes, stream);
    return e == cudaSuccess ? WKV_OK : cuda_fail(e);
}

wkv_status wkv_forward(int64_t B, int64_t T, int64_t C, wkv_dtype io, const float* w, const float* u, const void* k,
                       const void* v, void* y, float* state_out, void* workspace, size_t ws_bytes,
                       cudaStream_t stream) {
    return forward_impl(B, T, C, io, w, u, k, v, nullptr, y, state_out, workspace, ws_bytes, WKV_PATH_AUTO, 0,
                        kSpinLimitDefault, -1, stream);
}

wkv_status wkv_forward_ex(int64_t B, int64_t T, int64_t C, wkv_dtype io, const float* w, const float* u,
                          const void* k, const void* v, const float* state_in, void* y, float* state_out,
                          void* workspace, size_t ws_bytes, wkv_path path, int chunk, cudaStream_t stream) {
    return forward_impl(B, T, C, io, w, u, k, v, state_in, y, state_out, workspace, ws_bytes, path, chunk,
                        kSpinLimitDefault, -1, stream);
}

wkv_status wkv_forward_gated(int64_t B, int64_t T, int64_t C, wkv_dtype io, const float* w, const float* u,
                             const void* k, const void* v, const void* r, const float* state_in, void* y,
                             float* state_out, void* workspace, size_t ws_bytes, wkv_path path, int chunk,
                             cudaStream_t stream) {
    int64_t n = 0;
    if (!sizes_ok(B, T, C, &n)) return WKV_ERR_INVALID_ARG;
    if (n > 0 && T > 0 && !r) return WKV_ERR_INVALID_ARG;
    return forward_impl(B, T, C, io, w, u, k, v, state_in, y, state_out, workspace, ws_bytes, path, chunk,
                        kSpinLimitDefault, -1, stream, r);
}

wkv_status token_shift_mix3(int64_t B, int64_t T, int64_t C, const float* mu_r, const float* mu_k, const float* mu_v,
                            const float* x, const float* x_last, float* xr, float* xk, float* xv, cudaStream_t stream) {
    int64_t n = 0;
    if (!sizes_ok(B, T, C, &n)) return WKV_ERR_INVALID_ARG;
    if (n == 0) return WKV_OK;
    if (!mu_r || !mu_k || !mu_v || !x || !xr || !xk || !xv) return WKV_ERR_INVALID_ARG;
    if (!f32_args_ok({mu_r, mu_k, mu_v, x, x_last, xr, xk, xv})) return WKV_ERR_MISALIGNED;
    cudaError_t e = launch_token_shift3(B, T, C, mu_r, mu_k, mu_v, x, x_last, xr, xk, xv, stream);
    return e == cudaSuccess ? WKV_OK : cuda_fail(e);
}

size_t wkv_backward_workspace_size(int64_t B, int64_t T, int64_t C) {
    int64_t n = 0;
    if (!sizes_ok(B, T, C, &n) || n > INT64_MAX / 64) return 0;
    // a 64-byte header; per (b, group of 128 steps, c) the published forward record (4 tagged
    // 64-bit words) and adjoint sums with their reference (5 words)
    return backward_workspace_bytes(B, T, C);
}

wkv_status wkv_backward(int64_t B, int64_t T, int64_t C, const float* w, const float* u, const float* k,
                        const float* v, const float* gy, float* gk, float* gv, float* gw, float* gu, void* workspace,
                        size_t ws_bytes, cudaStream_t stream) {
    int64_t n = 0;
    if (!sizes_ok(B, T, C, &n) || n > INT64_MAX / 64) return WKV_ERR_INVALID_ARG;
    if (C == 0) return WKV_OK;
    if (!w || !u || !gw || !gu) return WKV_ERR_INVALID_ARG;
    if (n > 0 && (!k || !v || !gy || !gk || !gv)) return WKV_ERR_INVALID_ARG;
    if (!f32_args_ok({w, u, k, v, gy, gk, gv, gw, gu, workspace})) return WKV_ERR_MISALIGNED;
    if (!backward_fits(B, T, C)) return WKV_ERR_UNSUPPORTED;
    if (n > 0 && (!workspace || ws_bytes < wkv_backward_workspace_size(B, T, C))) return WKV_ERR_INVALID_ARG;
    cudaError_t e = launch_backward(B, T, C, w, u, k, v, gy, gk, gv, gw, gu, workspace, stream);
    return e == cudaSuccess ? WKV_OK : cuda_fail(e);
}

size_t eagle_forward_workspace_size(int64_t B, int64_t T, int64_t C) {
    int64_t n = 0;
    if (!sizes_ok(B, T, C, &n) || C % 64 != 0) return 0;
    // the one-launch form needs no scratch; the three-launch form one 64 x 64 fp32 state per
    // (b, head, chunk) (the chunk's sum, then its starting state)
    if (eagle_uses_sequence_kernel(B, T, C)) return 0;
    const int64_t heads = B * (C / 64), chunks = eagle_chunks(T);
    if (chunks != 0 && heads > INT64_MAX / 16384 / chunks) return 0;
    return (size_t)heads * (size_t)chunks * 64 * 64 * sizeof(float);
}

wkv_status eagle_forward(int64_t B, int64_t T, int64_t C, const float* w, const float* r, const float* k,
                         const float* v, const float* state_in, float* y, float* state_out, void* workspace,
                         size_t ws_bytes, cudaStream_t stream) {
    int64_t n = 0;
    if (!sizes_ok(B, T, C, &n) || n > INT64_MAX / 64) return WKV_ERR_INVALID_ARG;
    if (C % 64 != 0) return WKV_ERR_UNSUPPORTED;
    if (B == 0 || C == 0) return WKV_OK;
    if (!w) return WKV_ERR_INVALID_ARG;
    if (n > 0 && (!r || !k || !v || !y)) return WKV_ERR_INVALID_ARG;
    if (!f32_args_ok({w, r, k, v, state_in, y, state_out, workspace})) return WKV_ERR_MISALIGNED;
    // grids: (chunks, heads, B) for the chunk kernels, 16 blocks of 256 per head for the scan
    // TMA coordinates are 32-bit
    if (B > 65535 || C / 64 > 65535 || T > INT32_MAX || C > INT32_MAX || B * (C / 64) > INT32_MAX / 16)
        return WKV_ERR_UNSUPPORTED;
    const size_t need = eagle_forward_workspace_size(B, T, C);
    if (n > 0 && need > 0 && (!workspace || ws_bytes < need)) return WKV_ERR_INVALID_ARG;
    cudaError_t e = launch_eagle_forward(B, T, C, w, r, k, v, state_in, y, state_out, workspace, stream);
    return e == cudaSuccess ? WKV_OK : cuda_fail(e);
}

int eagle_forward_launches(int64_t B, int64_t T, int64_t C) {
    int64_t n = 0;
    if (!sizes_ok(B, T, C, &n) || C % 64 != 0) return 0;
    return eagle_uses_sequence_kernel(B, T, C) ? 1 : 3;
}

wkv_status eagle_decode_step(int64_t N, int64_t L, int64_t C, const float* w, const float* r, const float* k,
                             const float* v, float* state_inout, float* y, cudaStream_t stream) {
    int64_t n = 0;
    if (!sizes_ok(N, L, C, &n) || n > INT64_MAX / 64) return WKV_ERR_INVALID_ARG;
    if (C % 64 != 0) return WKV_ERR_UNSUPPORTED;
    if (n == 0) return WKV_OK;
    if (!w || !r || !k || !v || !state_inout || !y) return WKV_ERR_INVALID_ARG;
    if (!f32_args_ok({w, r, k, v, state_inout, y})) return WKV_ERR_MISALIGNED;
    if (n / 64 > INT32_MAX) return WKV_ERR_UNSUPPORTED;  // one block per (row, head)
    cudaError_t e = launch_eagle_decode(N, L, C, w, r, k, v, state_inout, y, stream);
    return e == cudaSuccess ? WKV_OK : cuda_fail(e);
}

wkv_status wkv_forward_status(void* workspace, size_t ws_bytes, cudaStream_t stream) {
    cudaError_t e = cudaStreamSynchronize(stream);
    if (e != cudaSuccess) return cuda_fail(e);
    uint32_t* word = nullptr;
    if (workspace) {
        if (ws_bytes < kWsHeaderBytes) return WKV_ERR_INVALID_ARG;
        word = &static_cast<WsHeader*>(workspace)->error;
    } else {
        word = status_word();
        if (!word) return cuda_fail(cudaGetLastError());
    }
    uint32_t code = 0;
    e = cudaMemcpy(&code, word, sizeof(code), cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return cuda_fail(e);
    if (code == kDevOk) return WKV_OK;
    // clear the error; a workspace is zero-filled whole (counters, epoch and flags restart
    // together, so no flag of an earlier launch can match a later epoch)
    if (workspace) {
        e = cudaMemset(workspace, 0, ws_bytes);
    } else {
        const uint32_t zero[2] = {0, 0};
        e = cudaMemcpy(word, zero, sizeof(zero), cudaMemcpyHostToDevice);
    }
    if (e != cudaSuccess) return cuda_fail(e);
    return WKV_ERR_TIMEOUT;
}

wkv_status wkv_get_device_status(cudaStream_t stream) {
    cudaError_t e = cudaStreamSynchronize(stream);
    if (e != cudaSuccess) return cuda_fail(e);
    uint32_t* word = device_status_word();
    if (!word) return cuda_fail(cudaGetLastError());
    uint32_t code = 0;
    e = cudaMemcpy(&code, word, sizeof(code), cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return cuda_fail(e);
    if (code == kDevOk) return WKV_OK;
    const uint32_t zero = 0;
    e = cudaMemcpy(word, &zero, sizeof(zero), cudaMemcpyHostToDevice);
    if (e != cudaSuccess) return cuda_fail(e);
    return WKV_ERR_TIMEOUT;
}

wkv_status wkv_decode_step(int64_t N, int64_t L, int64_t C, const float* w, const float* u, const float* k,
                           const float* v, float* state_inout, float* y, cudaStream_t stream) {
    int64_t n = 0;
    if (!sizes_ok(N, L, C, &n) || n > INT64_MAX / 3) return WKV_ERR_INVALID_ARG;
    if (n == 0) return WKV_OK;
    if (!w || !u || !k || !v || !state_inout || !y) return WKV_ERR_INVALID_ARG;
    if (!f32_args_ok({w, u, k, v, state_inout, y})) return WKV_ERR_MISALIGNED;
    cudaError_t e = launch_decode_step(N, L, C, nullptr, w, u, nullptr, nullptr, nullptr, k, v, state_inout, y,
                                       stream);
    return e == cudaSuccess ? WKV_OK : cuda_fail(e);
}

wkv_status wkv_decode_step_fused(int64_t N, int64_t L, int64_t C, const float* mu, const float* w, const float* u,
                                 const float* x_t, const float* x_prev, float* xbar, const float* k, const float* v,
                                 float* state_inout, float* y, cudaStream_t stream) {
    int64_t n = 0;
    if (!sizes_ok(N, L, C, &n) || n > INT64_MAX / 3) return WKV_ERR_INVALID_ARG;
    if (n == 0) return WKV_OK;
    if (!mu || !w || !u || !x_t || !x_prev || !xbar || !k || !v || !state_inout || !y) return WKV_ERR_INVALID_ARG;
    if (!f32_args_ok({mu, w, u, x_t, x_prev, xbar, k, v, state_inout, y})) return WKV_ERR_MISALIGNED;
    cudaError_t e = launch_decode_step(N, L, C, mu, w, u, x_t, x_prev, xbar, k, v, state_inout, y, stream);
    return e == cudaSuccess ? WKV_OK : cuda_fail(e);
}

wkv_status token_shift_mix(int64_t B, int64_t T, int64_t C, const float* mu, const float* x, const float* x_last,
                           float* xbar, cudaStream_t stream) {
    int64_t n = 0;
    if (!sizes_ok(B, T, C, &n)) return WKV_ERR_INVALID_ARG;
    if (n == 0) return WKV_OK;
    if (!mu || !x || !xbar) return WKV_ERR_INVALID_ARG;
    if (!f32_args_ok({mu, x, x_last, xbar})) return WKV_ERR_MISALIGNED;
    cudaError_t e = launch_token_shift(B, T, C, mu, x, x_last, xbar, stream);
    return e == cudaSuccess ? WKV_OK : cuda_fail(e);
}

const char* wkv_status_string(wkv_status status) {
    switch (status) {
        case WKV_OK: return "WKV_OK";
        case WKV_ERR_INVALID_ARG: return "WKV_ERR_INVALID_ARG";
        case WKV_ERR_MISALIGNED: return "WKV_ERR_MISALIGNED";
        case WKV_ERR_UNSUPPORTED: return "WKV_ERR_UNSUPPORTED";
        case WKV_ERR_CUDA: return "WKV_ERR_CUDA";
        case WKV_ERR_TIMEOUT: return "WKV_ERR_TIMEOUT";
    }
    return "WKV_ERR_UNKNOWN";
}

int wkv_last_cuda_error(void) { return g_last_cuda_error; }

wkv_path wkv_forward_auto_path(int64_t B, int64_t T, int64_t C, wkv_dtype io) { return auto_path(B, T, C, io); }

int wkv_version(void) { return 100; }

// Test hook (not in wkv.h): a chunked forward in which `drop_unit` never publishes its
// carry and every bounded wait gives up after `spin_limit` polls.  The successor of the
// dropped unit then runs out its wait, records WKV_ERR_TIMEOUT in the workspace, and the
// launch still completes.  Used to check that the error path returns control.
wkv_status wkv_testhook_forward_drop(int64_t B, int64_t T, int64_t C, const float* w, const float* u, const float* k,
                                     const float* v, float* y, void* workspace, size_t ws_bytes,
                                     int64_t drop_unit, uint32_t spin_limit, cudaStream_t stream) {
    return forward_impl(B, T, C, WKV_F32, w, u, k, v, nullptr, y, nullptr, workspace, ws_bytes, WKV_PATH_CHUNKED,
                        0, spin_limit, drop_unit, stream);
}

}  // extern "C"
