/*
 * wkv.h -- C ABI of the B200 (sm_100a) RWKV-4 WKV library (libwkv_b200.so), with the
 * Eagle (RWKV-5) matrix-state operator at the end.
 *
 * The operator ("RWKV" transformer-math page, aicassindra.com, section "The WKV
 * operator: attention with a fixed decay"; aiwiki "RWKV", eq. 1), per channel c,
 * 0-based position t:
 *
 *   wkv_t = ( sum_{i<t} e^{-(t-1-i) w + k_i} v_i + e^{u + k_t} v_t )
 *         / ( sum_{i<t} e^{-(t-1-i) w + k_i}     + e^{u + k_t} )
 *
 * w >= 0 is the per-channel decay rate (the decay per step is e^{-w}; the pages
 * take w = exp(omega) > 0), u the per-channel bonus of the current token.
 *
 * The state of one channel is the triple (a, b, p) with true accumulators
 *   A = a e^p = sum_i e^{-(t-i) w + k_i} v_i,   B = b e^p = sum_i e^{-(t-i) w + k_i}
 * over the tokens i <= t consumed so far (same page, section "Numerical stability:
 * carry the exponent").  p is a free exponent offset: (a e^d, b e^d, p - d) is the
 * same state.  The empty state is a = b = 0, p = -1e38.  A state buffer holds three
 * planes: [3][rows][C] = (a plane, b plane, p plane), fp32.
 *
 * Conventions for every call below
 *  - Pointers are DEVICE pointers owned by the caller (e.g. torch tensors).  The
 *    library allocates nothing and keeps no per-call state.
 *  - Calls are asynchronous on `stream` (0 = legacy default stream): they validate
 *    their arguments on the host, enqueue the kernel(s) and return.
 *  - Argument errors are reported synchronously by the return value and nothing is
 *    enqueued: sizes < 0 or whose products overflow int64 -> WKV_ERR_INVALID_ARG;
 *    a required pointer that is NULL -> WKV_ERR_INVALID_ARG; a device pointer not
 *    16-byte aligned -> WKV_ERR_MISALIGNED; an unknown dtype/path ->
 *    WKV_ERR_UNSUPPORTED.  A launch failure returns WKV_ERR_CUDA
 *    (wkv_last_cuda_error() gives the cudaError_t).  Faults inside a kernel show
 *    up, as for any CUDA kernel, at the caller's next synchronisation.
 *  - A size of 0 in any dimension is a valid empty call (nothing is written,
 *    except that wkv_forward with T = 0 still writes state_out).
 *  - Tensors are dense row-major with the innermost (channel) dimension
 *    contiguous.  Any C is accepted; C a multiple of 4 (fp32) or 8 (bf16) takes the
 *    vectorised bulk-copy path.
 *  - There is no CPU fallback: every entry point runs CUDA kernels for sm_100a.
 */
#ifndef WKV_B200_H
#define WKV_B200_H

#include <stddef.h>
#include <stdint.h>

#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum wkv_status {
    WKV_OK = 0,
    WKV_ERR_INVALID_ARG = 1,  /* bad size, NULL pointer, workspace too small */
    WKV_ERR_MISALIGNED = 2,   /* a device pointer is not 16-byte aligned */
    WKV_ERR_UNSUPPORTED = 3,  /* unknown dtype, path or chunk length */
    WKV_ERR_CUDA = 4,         /* a CUDA runtime call or launch failed */
    WKV_ERR_TIMEOUT = 5       /* a device-side wait gave up (see wkv_forward_status) */
} wkv_status;

typedef enum wkv_dtype {
    WKV_F32 = 0,   /* k, v, y in fp32 */
    WKV_BF16 = 1   /* k, v, y in bf16 (y rounded to nearest even); state and w, u stay fp32 */
} wkv_dtype;

typedef enum wkv_path {
    WKV_PATH_AUTO = 0,     /* the fastest path measured at the nearest (dtype, B*C, T) grid point */
    WKV_PATH_SERIAL = 1,   /* one thread per (b, c) scanning all of T */
    WKV_PATH_CHUNKED = 2   /* time-parallel: chunk summaries, carry scan, fix-up */
} wkv_path;

/*
 * Forward (prefill) over [B, T, C].
 *
 * Computes wkv_t for every (b, t, c) (the equation above) and, if state_out is not
 * NULL, the state after the last token, which wkv_decode_step continues exactly
 * ("RWKV and Recurrent Models With Transformer Quality", multigrid.ai, section
 * "Prefill, decode, and where each form is used": prefill produces the state after
 * the last prompt token; decode steps from it).
 *
 *   w, u       [C] fp32 (w >= 0)
 *   k, v       [B, T, C] in dtype io
 *   y          [B, T, C] in dtype io (written)
 *   state_out  [3][B][C] fp32 (a, b, p) or NULL
 *   workspace  caller-owned device scratch of ws_bytes >= wkv_forward_workspace_size();
 *              it must be zero-filled once before its first use (wkv_workspace_init)
 *              and must not be used by two calls that can overlap on the GPU.
 *              It may be NULL when the size query returns 0.
 * Returns WKV_ERR_INVALID_ARG when ws_bytes is too small for the chosen path.
 */
wkv_status wkv_forward(int64_t B, int64_t T, int64_t C, wkv_dtype io, const float* w, const float* u,
                       const void* k, const void* v, void* y, float* state_out, void* workspace,
                       size_t ws_bytes, cudaStream_t stream);

/*
 * As wkv_forward, plus:
 *   state_in  [3][B][C] fp32 (a, b, p) to continue from, or NULL for the empty state
 *             (resumable / piecewise prefill; state_out may alias state_in);
 *   path      WKV_PATH_AUTO, WKV_PATH_SERIAL or WKV_PATH_CHUNKED;
 *   chunk     time steps per chunk for the chunked path (0 = default; else 4, 8 or 16
 *             steps per warp).  With WKV_PATH_AUTO and chunk 0 the chunk length comes
 *             from the same measured table as the path (8 or 16).
 */
wkv_status wkv_forward_ex(int64_t B, int64_t T, int64_t C, wkv_dtype io, const float* w, const float* u,
                          const void* k, const void* v, const float* state_in, void* y, float* state_out,
                          void* workspace, size_t ws_bytes, wkv_path path, int chunk, cudaStream_t stream);

/*
 * As wkv_forward_ex, with the receptance gate applied to the output (transformer-math page,
 * section "Receptance: the gate on the way out"): y receives sigma(r) * wkv channel by
 * channel, sigma the logistic function; the ungated wkv is not written.  The W_o projection
 * that follows the gate on the page is not part of this call.
 *   r          [B, T, C] in dtype io (required when B*T*C > 0)
 * state_out is the recurrence state (the gate acts on the output only).  The chunked kernel
 * for 16-byte rows applies the gate as it writes y (r is read once, y written once); other
 * paths run the forward and then one elementwise pass y <- sigma(r) * y.  Same status codes
 * as wkv_forward_ex; r must be 16-byte aligned.
 */
wkv_status wkv_forward_gated(int64_t B, int64_t T, int64_t C, wkv_dtype io, const float* w, const float* u,
                             const void* k, const void* v, const void* r, const float* state_in, void* y,
                             float* state_out, void* workspace, size_t ws_bytes, wkv_path path, int chunk,
                             cudaStream_t stream);

/*
 * Backward of the forward from the empty state: for a loss L = sum(gy * y) over [B, T, C],
 * the gradients of L with respect to k and v (per element) and w and u (per channel, summed
 * over batch and time).  The pages give no gradient; this is the wkv_t equation above
 * differentiated as written (with D_t its denominator, alpha_t = e^{u+k_t},
 * beta_{t,i} = e^{-(t-1-i) w + k_i}: dy_t/dv_i = beta_{t,i} / D_t, dy_t/dk_i =
 * beta_{t,i} (v_i - y_t) / D_t, dy_t/dw = -sum_i (t-1-i) beta_{t,i} (v_i - y_t) / D_t, and the
 * current token's alpha_t terms for v_t, k_t and u).
 *   w, u          [C] fp32
 *   k, v, gy      [B, T, C] fp32
 *   gk, gv        [B, T, C] fp32 (written; must not overlap the inputs)
 *   gw, gu        [C] fp32 (written: zeroed, then each block's partial sums added with atomics)
 *   workspace     caller-owned device scratch of ws_bytes >= wkv_backward_workspace_size()
 *                 (per channel and group of 128 steps the published forward record and adjoint
 *                 sums), zero-filled once before its first use (wkv_workspace_init); one
 *                 workspace must not serve two backward calls that can run at the same time
 * Time-parallel over segments of 16 steps, eight to a block, in one launch whose blocks take
 * their work in ticket order: first the groups in time order, each publishing its forward
 * record and, by a bounded look-back over the records of the groups before it, the state at
 * its end; then the groups in reverse time order, each recomputing its outputs from the state
 * entering it (the same look-back), taking the adjoint sums of the groups after it by a bounded
 * look-back and writing its gradients.  Inside a segment the forward and adjoint sums run in a
 * fixed exponent frame where the segment's exponents fit one (the per-step stabilised
 * recurrence elsewhere).  k, v are read twice, gy once; nothing per position is kept in global
 * memory.
 * A look-back that gives up is recorded in the device-wide word that wkv_get_device_status
 * reports (the gradients are then invalid).
 * Status codes as wkv_forward; WKV_ERR_UNSUPPORTED when (2 ceil(T / 128) - 1) B ceil(C / 32)
 * exceeds 2^31 - 1 (one launch's blocks).
 */
wkv_status wkv_backward(int64_t B, int64_t T, int64_t C, const float* w, const float* u, const float* k,
                        const float* v, const float* gy, float* gk, float* gv, float* gw, float* gu,
                        void* workspace, size_t ws_bytes, cudaStream_t stream);

/* Workspace bytes wkv_backward needs: 64, plus 72 per batch row, channel and 128 steps (rounded
 * up). */
size_t wkv_backward_workspace_size(int64_t B, int64_t T, int64_t C);

/* Workspace bytes wkv_forward needs for this shape (the largest over all paths). */
size_t wkv_forward_workspace_size(int64_t B, int64_t T, int64_t C, wkv_dtype io);

/* Zero-fill a workspace (once, before its first use). */
wkv_status wkv_workspace_init(void* workspace, size_t ws_bytes, cudaStream_t stream);

/*
 * Synchronises `stream`, then reports and clears the device-side error word of a
 * workspace: WKV_ERR_TIMEOUT if a chunked forward launched with it gave up waiting
 * for a predecessor's carry (its outputs are then invalid), else WKV_OK.
 */
wkv_status wkv_forward_status(void* workspace, size_t ws_bytes, cudaStream_t stream);

/*
 * Synchronises `stream`, then reports and clears the library's device-wide error word on
 * the current device: WKV_ERR_TIMEOUT if any forward launched on this device since the last
 * call gave up a bounded device-side wait (its outputs are then invalid; the workspace it
 * used also carries the error, see wkv_forward_status), else WKV_OK.  WKV_ERR_CUDA if the
 * synchronisation or the read fails (e.g. an earlier fault).  The word is shared by all
 * streams and workspaces of the device, so a report may concern another stream's launch.
 * The pages have no counterpart: this is the library's failure detection for its own waits.
 */
wkv_status wkv_get_device_status(cudaStream_t stream);

/*
 * One decode step for N sessions x L layers x C channels: for every row (n, l) and
 * channel c, emit wkv for the token (k, v) from the stored state and fold the token
 * into the state (aiwiki "RWKV": the one-token decode step; transformer-math page,
 * section "Numerical stability: carry the exponent").
 *   w, u         [L][C] fp32 (layer l's parameters)
 *   k, v, y      [N][L][C] fp32
 *   state_inout  [3][N][L][C] fp32 (a, b, p), updated in place
 * With L = 1 and N = B, state_out of wkv_forward continues the same sequences.
 */
wkv_status wkv_decode_step(int64_t N, int64_t L, int64_t C, const float* w, const float* u, const float* k,
                           const float* v, float* state_inout, float* y, cudaStream_t stream);

/*
 * Token shift (transformer-math page, section "Token shift: a two-tap causal
 * convolution"): xbar_t = mu * x_t + (1 - mu) * x_{t-1}, per channel.
 *   mu      [C] fp32
 *   x, xbar [B, T, C] fp32 (xbar must not alias x)
 *   x_last  [B][C] fp32, the token before t = 0, or NULL for zeros (causal padding)
 */
wkv_status token_shift_mix(int64_t B, int64_t T, int64_t C, const float* mu, const float* x, const float* x_last,
                           float* xbar, cudaStream_t stream);

/*
 * Token shift of the three projections in one pass (transformer-math page, section "Token
 * shift: a two-tap causal convolution": r, k and v each blend with their own mu):
 *   xr = mu_r * x_t + (1 - mu_r) * x_{t-1}, and likewise xk with mu_k, xv with mu_v.
 *   mu_r, mu_k, mu_v [C] fp32
 *   x, xr, xk, xv    [B, T, C] fp32 (outputs must not alias x or each other)
 *   x_last           [B][C] fp32, the token before t = 0, or NULL for zeros
 * x is read once; the W_r, W_k, W_v projections that follow are not part of this call.
 */
wkv_status token_shift_mix3(int64_t B, int64_t T, int64_t C, const float* mu_r, const float* mu_k,
                            const float* mu_v, const float* x, const float* x_last, float* xr, float* xk,
                            float* xv, cudaStream_t stream);

/*
 * Fused decode step: the token-shift lerp ("RWKV" transformer-math page, section "Token shift:
 * a two-tap causal convolution": xbar = mu x_t + (1 - mu) x_{t-1}) and the WKV decode step
 * (aiwiki "RWKV": the one-token decode step; the same arithmetic as wkv_decode_step) in one
 * kernel, each input and state element read once.
 *   mu, w, u      [L][C] fp32
 *   x_t, x_prev   [N][L][C] fp32: this token's input and the previous token's
 *   xbar          [N][L][C] fp32: mu * x_t + (1 - mu) * x_prev (written)
 *   k, v, y       [N][L][C] fp32: the token's key and value; y = its wkv (written)
 *   state_inout   [3][N][L][C] fp32, updated in place
 * The caller makes x_t the next call's x_prev (pointer swap, no copy).
 */
wkv_status wkv_decode_step_fused(int64_t N, int64_t L, int64_t C, const float* mu, const float* w,
                                 const float* u, const float* x_t, const float* x_prev, float* xbar,
                                 const float* k, const float* v, float* state_inout, float* y,
                                 cudaStream_t stream);

/*
 * wkv_forward_ex on the chunked path for callers that cannot allocate device memory
 * (for instance code running inside another framework's memory pool, or under a
 * budget that forbids cudaMalloc after start-up).  The pages have no counterpart: this
 * is a packaging of the same chunked kernel, not a different computation.
 *
 * Same arguments, layouts and results as wkv_forward_ex with path = WKV_PATH_CHUNKED,
 * minus the workspace: the scratch lives in a fixed 32 MiB device array inside the
 * library, which every GPU that loads the library keeps until the process exits.  The
 * call allocates nothing (no cudaMalloc, no allocating library routine).
 *  - Shapes whose scratch would exceed 32 MiB are rejected with WKV_ERR_INVALID_ARG
 *    before anything is enqueued (e.g. 8 x 1024 x 768 fp32 needs ~6.3 MB; 1 x 16384 x
 *    4096 fp32 needs more and is rejected).  B = 0 or C = 0 is a no-op; T = 0 writes
 *    state_out only (state_in, or the empty state), as wkv_forward_ex does.
 *  - All calls on a device share the array and it keeps the last call's contents; each
 *    call clears the counters that must start at zero.  Calls that can overlap on the
 *    GPU race on the array: order them (same stream, or events).
 *  - The first call on each device looks up the array's device address
 *    (cudaGetSymbolAddress) with that device current and zero-fills the array once;
 *    make that first call before any stream capture.
 *  - A device-side wait that runs out (only possible when calls overlap) is recorded
 *    in the array's header, which the next call clears, and in the library's
 *    device-wide error word, which wkv_get_device_status reports.
 *  - WKV_ERR_CUDA leaves the cause in wkv_last_cuda_error, as for the other calls.
 */
wkv_status wkv_forward_chunked_noalloc(int64_t B, int64_t T, int64_t C, wkv_dtype io, const float* w,
                                       const float* u, const void* k, const void* v, const float* state_in,
                                       void* y, float* state_out, cudaStream_t stream);

/*
 * Eagle (RWKV-5) matrix-state WKV ("RWKV (Attention-RNN Hybrid)", vanos001.github.io,
 * section "Versions: RWKV-4 -> Eagle -> Finch"), per sequence b and head h of 64 channels
 * (channels h*64 .. h*64+63), token after token:
 *
 *   S_t = diag(d) S_{t-1} + k_t v_t^T,     y_t = r_t^T S_t   (y_t[j] = sum_m r_t[m] S_t[m][j])
 *
 * S is 64 x 64 per head (row m a key channel, column j a value channel), d[m] = e^{-w[m]}
 * with w >= 0 the per-channel decay rate as for RWKV-4.  The read-out follows the update (the
 * current token enters with weight 1; the pages give Eagle no bonus term and no
 * normalisation).  A state buffer is [B][C / 64][64][64] fp32 (m, j), the empty state zeros.
 *
 * eagle_forward: prefill over [B, T, C].
 *   w              [C] fp32
 *   r, k, v        [B, T, C] fp32
 *   state_in       [B][C/64][64][64] fp32, or NULL for the empty state
 *   y              [B, T, C] fp32 (written; must not alias the inputs)
 *   state_out      [B][C/64][64][64] fp32, the state after the last token, or NULL
 *   workspace      caller-owned device scratch, ws_bytes >= eagle_forward_workspace_size()
 *                  (none when eagle_forward_workspace_size() is 0: workspace may then be NULL)
 * C must be a multiple of 64 (else WKV_ERR_UNSUPPORTED), C/64 and B at most 65535.  T = 0
 * writes state_out only (state_in, or zeros).  Two forms, chosen from the shape
 * (eagle_forward_launches):
 *   one launch: a block per (sequence, head) walks its 64-token chunks in order; per 16-token
 *     block the outputs are the state's read-out plus the block's own causal attention, and the
 *     state advances by the block's key-value sum, every product on the tensor cores (tcgen05,
 *     operands split into two tf32 parts for fp32-level error) and the state kept in fp32
 *     registers.  A head with a channel of |w| > 5.5 (decay below 0.004 per token) runs the
 *     same launch token by token on the CUDA cores instead.  Used when B * C/64 >= 24 or the
 *     sequence has at most 8 chunks.
 *   three launches, time-parallel over all chunk-heads: each chunk's own state contribution (a
 *     tensor-core product as above), a scan over the chunks per state entry, then each chunk's
 *     outputs from its starting state (fp32 CUDA cores).  For few heads with long sequences.
 * Status codes as wkv_forward.
 */
wkv_status eagle_forward(int64_t B, int64_t T, int64_t C, const float* w, const float* r, const float* k,
                         const float* v, const float* state_in, float* y, float* state_out, void* workspace,
                         size_t ws_bytes, cudaStream_t stream);

/* Workspace bytes eagle_forward needs: 0 for the one-launch form, else 16 KiB per sequence,
 * head and 64-token chunk. */
size_t eagle_forward_workspace_size(int64_t B, int64_t T, int64_t C);

/* Kernel launches eagle_forward makes for this shape: 1 (the one-launch form) or 3; 0 for an
 * invalid shape.  No device call. */
int eagle_forward_launches(int64_t B, int64_t T, int64_t C);

/*
 * Eagle decode: one token for N sessions x L layers (section "O(N) Inference
 * Characteristics": one matrix-vector product against the fixed-size state per token).
 *   w              [L][C] fp32 (layer l's decay rates)
 *   r, k, v, y     [N][L][C] fp32 (y written)
 *   state_inout    [N][L][C/64][64][64] fp32, updated in place
 * C must be a multiple of 64.  With L = 1 and N = B, state_out of eagle_forward continues
 * the same sequences.
 */
wkv_status eagle_decode_step(int64_t N, int64_t L, int64_t C, const float* w, const float* r, const float* k,
                             const float* v, float* state_inout, float* y, cudaStream_t stream);

/* Human-readable name of a status code (static string). */
const char* wkv_status_string(wkv_status status);

/* The cudaError_t of the last WKV_ERR_CUDA returned on this host thread (0 if none). */
int wkv_last_cuda_error(void);

/* The path WKV_PATH_AUTO picks for this shape (WKV_PATH_SERIAL or WKV_PATH_CHUNKED): the
 * fastest one measured on a B200 at the grid point nearest to (dtype, B*C, T) on a log scale
 * (csrc/wkv_path_table.h, written by the package's tuning script, tune.py). */
wkv_path wkv_forward_auto_path(int64_t B, int64_t T, int64_t C, wkv_dtype io);

/* Library version, major * 10000 + minor * 100 + patch. */
int wkv_version(void);

#ifdef __cplusplus
}
#endif

#endif /* WKV_B200_H */
