/*
 * moe_ffn.h -- C ABI of the B200 (sm_100a) top-k mixture-of-experts FFN layer.
 *
 * The operation (one decode or prefill step of a Qwen3.5/3.6-style MoE FFN):
 *
 *   l[t,e]  = sum_h x[t,h] * Wr[e,h]  (+ bias[e])            router GEMV (bf16)
 *   idx[t]  = the k largest l[t,:] (ties: lower expert first), by descending logit
 *   w[t,r]  = exp(l[t,idx_r]) / sum_j exp(l[t,idx_j])         softmax over the k chosen
 *   z[t]    = sum_h x[t,h] * g[h],  gs[t] = sigmoid(z[t])      shared-expert gate
 *   E_e(x)  = W2_e ( silu(W13_e[:I] x) * W13_e[I:] x )         SwiGLU expert, FP8 weights
 *   out[t]  = sum_r w[t,r] E_{idx_r}(x_t) + gs[t] E_shared(x_t) (+ residual[t]),
 *             rounded once to bf16.
 *
 * Passages it follows: the "Qwen3.6-35B-A3B-FP8 on NVIDIA GB10" blueprint page
 * (Kernels table: dense_gemv_bf16 router, moe_topk_softmax, gate_up and
 * silu_down FP8 expert kernels with the shared expert fused, weighted-sum
 * blend; Precision table: fp8/block128x128 weights against bf16 and f32
 * activations, f32,i32 top-k outputs); the "colibri #1992" PR page (frame A2:
 * the shared expert together with its gate; a warp per output row with 16-byte
 * lane loads and the activation in shared memory for decode GEMVs); the
 * "Neurarch Qwen3-8B" page (SwiGLU gate_proj/up_proj [I,H], down_proj [H,I]).
 *
 * Dimensions: H, I and Is must be multiples of 128; 1 <= k <= min(E, 32);
 * E <= 1024.
 *
 * Layouts (all row-major, reduction dimension contiguous, device memory):
 *   x, residual, out     bf16 [rows, H]
 *   router_w             bf16 [E, H]
 *   shared_gate          bf16 [H]
 *   router_bias          fp32 [E]                       (nullable)
 *   expert_w8            e4m3 bytes, E slabs of 3*I*H:  [W13 (2I x H) | W2 (H x I)];
 *                        W13 holds the gate rows, then the up rows
 *   expert_scales        fp32, E slabs of (2I/128)(H/128) + (H/128)(I/128):
 *                        [s13 (2I/128 x H/128) | s2 (H/128 x I/128)];
 *                        weight value = e4m3(code) * scale of its 128x128 block
 *   shared_w             one slab of the same layout with Is in place of I
 *   topk_idx / topk_w    int32 / fp32 [rows, k], descending weight
 *   shared_gate_sig      fp32 [rows]
 *
 * Ownership and execution: the caller owns every buffer and the stream.  The
 * library allocates no device memory; it uses the caller's workspace
 * (moe_workspace_bytes) and keeps one host-side table of per-device
 * properties.  Every call is asynchronous on `stream` (a cudaStream_t; NULL
 * = the legacy default stream) and returns after enqueueing.  Device
 * pointers must be 16-byte aligned.  `out` may alias `residual`; no other
 * output may alias an input.  A workspace serves one stream at a time: calls
 * that overlap on the device must use different workspaces.  A fresh
 * workspace must be zero-filled once (moe_workspace_init) before its first
 * use; the library leaves it reusable after every call it completes.
 *
 * Errors: every call returns a status (MOE_OK = 0, else a negative code).
 * Argument errors are detected on the host before anything is enqueued.
 * A CUDA error is sticky, as a lost device is in the pages' CUDA chain: after
 * MOE_ECUDA every call returns MOE_ECUDA until moe_reset_status() (after
 * which the workspace must be re-initialised).
 */
#ifndef MOE_FFN_H
#define MOE_FFN_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

#define MOE_OK 0
#define MOE_EINVAL -1        /* null pointer, misaligned pointer, rows < 0, bad path */
#define MOE_EUNSUPPORTED -2  /* H, I or Is not a multiple of 128, k > E, k > 32, E > 1024 */
#define MOE_EWORKSPACE -3    /* workspace smaller than moe_workspace_bytes(d, rows) */
#define MOE_ECUDA -4         /* a CUDA launch or runtime error (sticky) */
#define MOE_ETIMEOUT -5      /* a bounded wait inside a kernel ran out (device status word) */

#define MOE_PATH_AUTO 0      /* by rows: MOE_AUTO_DECODE_MAX_ROWS, MOE_AUTO_NARROW_MAX_PAIRS below */
#define MOE_PATH_DECODE 1    /* one persistent kernel per MOE_DECODE_MAX_ROWS rows: bf16 x and f32 h against FP8 weights */
#define MOE_PATH_PREFILL 2   /* token permute -> tcgen05 FP8 grouped GEMMs -> unpermute */
#define MOE_PATH_PREFILL_NARROW 3  /* the same pipeline with the grouped GEMMs tiled as 128 weight rows (the
                                     MMA's M) x up to 32 rows of one expert (its N): for few rows per expert;
                                     MOE_EUNSUPPORTED when H, I or Is exceeds 4096 */
#define MOE_DECODE_MAX_ROWS 4        /* rows per decode-step launch; more rows run as several launches */
#define MOE_AUTO_DECODE_MAX_ROWS 3    /* MOE_PATH_AUTO: the decode kernels up to this many rows; then the
                                         narrow grouped GEMMs while rows * k <= MOE_AUTO_NARROW_MAX_PAIRS * E
                                         (an expert's average routed rows), then the 128-row token tiles;
                                         the switch points were measured on B200 with every path timed on
                                         the 35B-A3B- and 397B-A17B-shaped layers */
#define MOE_AUTO_NARROW_MAX_PAIRS 32

typedef struct moe_dims {
    int32_t hidden;       /* H  */
    int32_t n_experts;    /* E  */
    int32_t top_k;        /* k  */
    int32_t inter;        /* I  : routed expert intermediate size */
    int32_t shared_inter; /* Is : shared expert intermediate size */
} moe_dims;

/* One expert's weights in the slab layout above (used for the shared expert). */
typedef struct moe_fp8_expert {
    const uint8_t *w8;    /* 3*Is*H e4m3 codes */
    const float *scales;  /* (2Is/128)(H/128) + (H/128)(Is/128) fp32 scales */
} moe_fp8_expert;

/* One NVFP4 expert (the shared one): packed e2m1 codes [W13 (2Is x H/2) |
 * W2 (H x Is/2)] (element 2j of a row in the low nibble of byte j), e4m3
 * block scale codes [W13 (2Is x H/16) | W2 (H x Is/16)] (one per 16
 * consecutive elements of a row), fp32 tensor scales [2] (W13, W2). */
typedef struct moe_nvfp4_expert {
    const uint8_t *w4;
    const uint8_t *sf;
    const float *gs;
} moe_nvfp4_expert;

/* Bytes of workspace needed by any call with rows <= max_rows on either path.
 * Returns 0 for invalid or unsupported dims or max_rows < 0. */
MOE_API size_t moe_workspace_bytes(const moe_dims *d, int32_t max_rows);

/* Zero-fill a workspace on `stream` (needed once per fresh workspace). */
MOE_API int moe_workspace_init(void *ws, size_t ws_bytes, void *stream);

/* Router GEMV, shared-gate sigmoid and top-k softmax for `rows` rows of x.
 * Defined by the "Qwen3.6-35B-A3B-FP8 on NVIDIA GB10" blueprint page, Kernels
 * table (the router as a bf16 dense GEMV, gemv::dense_gemv_bf16, feeding
 * moe_topk::moe_topk_softmax) and its Precision table (top-k node output
 * f32,i32); the shared-expert gate after the "colibri #1992" PR page, frame
 * A2.  Arithmetic: bf16 x and router rows, fp32 products and sums.
 * Outputs topk_idx [rows, k] (int32), topk_w [rows, k] (fp32, renormalised
 * over the k chosen, descending) and shared_gate_sig [rows] (fp32).
 * router_bias may be NULL.  rows == 0 is a no-op (pointers may then be NULL).
 * Errors: MOE_EINVAL (null or misaligned pointer, rows < 0), MOE_EUNSUPPORTED
 * (dims), MOE_EWORKSPACE (ws_bytes < moe_workspace_bytes(d, rows)), MOE_ECUDA. */
MOE_API int moe_router_topk(const moe_dims *d, const uint16_t *x, int32_t rows,
                    const uint16_t *router_w, const float *router_bias,
                    const uint16_t *shared_gate, int32_t *topk_idx, float *topk_w,
                    float *shared_gate_sig, void *ws, size_t ws_bytes, void *stream);

/* The whole layer step: out = sum_r w_r E_{idx_r}(x) + sigmoid(g.x) E_shared(x)
 * (+ residual), bf16 [rows, H].  Defined by the "Qwen3.6-35B-A3B-FP8 on
 * NVIDIA GB10" blueprint page, Kernels table (router GEMV, top-k softmax,
 * FP8 gate/up with the shared expert, SiLU and down, weighted-sum blend) and
 * Precision table (fp8 block128x128 weights against bf16 activations for
 * gate/up and f32 activations for down); the SwiGLU form after the
 * "Neurarch Qwen3-8B" page (swiglu block).  residual and router_bias may be
 * NULL.  Chooses the path by rows, as MOE_PATH_AUTO describes (moe_auto_path
 * tells which).  rows == 0 is a no-op (pointers may then be NULL).
 * Errors: as moe_router_topk, plus MOE_EINVAL when out aliases x. */
MOE_API int moe_ffn_forward(const moe_dims *d, const uint16_t *x, int32_t rows,
                    const uint16_t *router_w, const uint8_t *expert_w8,
                    const float *expert_scales, const moe_fp8_expert *shared_w,
                    const uint16_t *shared_gate, uint16_t *out, const uint16_t *residual,
                    const float *router_bias, void *ws, size_t ws_bytes, void *stream);

/* moe_ffn_forward with an explicit path (MOE_PATH_*) and optional copies of
 * the routing it used (each nullable): topk_idx [rows, k], topk_w [rows, k],
 * shared_gate_sig [rows].  The decode path accepts any rows but is sized for
 * rows <= MOE_DECODE_MAX_ROWS. */
MOE_API int moe_ffn_forward_path(const moe_dims *d, const uint16_t *x, int32_t rows,
                         const uint16_t *router_w, const uint8_t *expert_w8,
                         const float *expert_scales, const moe_fp8_expert *shared_w,
                         const uint16_t *shared_gate, uint16_t *out, const uint16_t *residual,
                         const float *router_bias, void *ws, size_t ws_bytes, void *stream,
                         int32_t path, int32_t *topk_idx, float *topk_w,
                         float *shared_gate_sig);

/* The layer behind its RMSNorm, with the residual join:
 *   x   = bf16( (resid / sqrt(mean_h resid^2 + eps)) * norm_w ),
 *   out = resid + [sum_r w_r E_{idx_r}(x) + sigmoid(g.x) E_shared(x)],  rounded once to bf16.
 * After the "Qwen3.6-35B-A3B-FP8 on NVIDIA GB10" blueprint page, Kernels table
 * (norm::rms_norm / norm::residual_add_rms_norm: the bf16 norm output feeds
 * the router GEMV of the MoE block) and the "Neurarch Qwen3-8B" page (an
 * RMSNorm over the hidden size before each SwiGLU block).  The mean square,
 * the scaling and the product with norm_w are computed in double and
 * rounded once to bf16.  On the decode path the norm runs inside the one
 * decode-step kernel, so a stack of layers is one launch per layer; on the
 * grouped-GEMM paths a norm kernel runs first.  resid bf16 [rows, H],
 * norm_w bf16 [H], eps >= 0 (the pages give none; Qwen models use 1e-6);
 * out may alias resid (an in-place update of the residual stream).  path is
 * a MOE_PATH_* (MOE_PATH_AUTO as moe_ffn_forward chooses).  Workspace:
 * moe_workspace_bytes(d, rows).  Errors as moe_ffn_forward, MOE_EINVAL also
 * for a null or misaligned norm_w or eps < 0. */
MOE_API int moe_ffn_forward_norm(const moe_dims *d, const uint16_t *resid, int32_t rows,
                         const uint16_t *norm_w, float eps, const uint16_t *router_w,
                         const uint8_t *expert_w8, const float *expert_scales,
                         const moe_fp8_expert *shared_w, const uint16_t *shared_gate, uint16_t *out,
                         const float *router_bias, void *ws, size_t ws_bytes, void *stream,
                         int32_t path);

/* Number of kernels one moe_ffn_forward_path call launches for these dims,
 * rows and path (MOE_PATH_AUTO resolved as moe_ffn_forward does); 0 for
 * invalid arguments or rows == 0. */
MOE_API int32_t moe_kernel_launches(const moe_dims *d, int32_t rows, int32_t path);

/* The path (MOE_PATH_DECODE, MOE_PATH_PREFILL or MOE_PATH_PREFILL_NARROW) that
 * moe_ffn_forward and MOE_PATH_AUTO take for these dims and rows; host only,
 * no device call; MOE_EINVAL for invalid dims or rows < 0. */
MOE_API int32_t moe_auto_path(const moe_dims *d, int32_t rows);

/* moe_ffn_forward_path for per-kernel timing: records events[0] on `stream`
 * before the first kernel and events[j] after kernel j-1 (each a caller-owned
 * cudaEvent_t created with timing enabled), and launches the kernels without
 * programmatic dependent launch so that consecutive events bracket exactly
 * one kernel.  n_events must be at least moe_kernel_launches(d, rows, path)
 * + 1, else MOE_EINVAL.  Results are identical to moe_ffn_forward_path. */
MOE_API int moe_ffn_forward_timed(const moe_dims *d, const uint16_t *x, int32_t rows,
                          const uint16_t *router_w, const uint8_t *expert_w8,
                          const float *expert_scales, const moe_fp8_expert *shared_w,
                          const uint16_t *shared_gate, uint16_t *out, const uint16_t *residual,
                          const float *router_bias, void *ws, size_t ws_bytes, void *stream,
                          int32_t path, void *const *events, int32_t n_events);

/* Device-side status of a workspace: synchronises `stream`, then reads the
 * status word the kernels keep in the workspace (MOE_OK, or MOE_ETIMEOUT if
 * a bounded wait inside a kernel ran out; the outputs of that call are then
 * incomplete and the workspace must be re-initialised).  Returns MOE_ECUDA
 * if the copy itself fails. */
MOE_API int moe_device_status(const void *ws, size_t ws_bytes, void *stream);

/* Test hook for the bounded waits: launches one CTA that waits on an
 * mbarrier nothing completes, gives up after limit_us microseconds (clamped
 * to [1, 2000000]) and records MOE_ETIMEOUT in the workspace status word, so
 * that moe_device_status reports it.  The GPU context stays usable. */
MOE_API int moe_debug_wait_timeout(void *ws, size_t ws_bytes, int32_t limit_us, void *stream);

/* moe_ffn_forward for callers that cannot allocate device memory (their
 * device memory belongs to a host application's allocator, or they must not
 * take an allocation path mid-run).  No counterpart on the reference pages:
 * it is a library-service entry point.  Instead of a caller workspace it
 * uses a scratch array built into the library, moe_static_scratch_bytes()
 * large (16 MiB), of which every GPU that loads the library holds one copy
 * until the process exits.  Calls whose moe_workspace_bytes(d, rows) exceeds
 * it fail with MOE_EWORKSPACE before anything is enqueued.  The call
 * allocates nothing (no cudaMalloc, no cudaFree, no allocating library
 * routine); it clears the array's counters on `stream` before launching,
 * all but the status word (see moe_static_device_status).  The first call
 * on a device (and the first after its context was re-created) looks up the
 * array's device address, so make it before any stream capture.  All calls
 * on a device share the one array: calls that overlap on the GPU race and
 * must not be issued (serialise them on one stream).  Arguments, results and
 * host-side errors are those of moe_ffn_forward; a failed address lookup or
 * clear returns MOE_ECUDA and sets the sticky status. */
MOE_API int moe_ffn_forward_static(const moe_dims *d, const uint16_t *x, int32_t rows,
                           const uint16_t *router_w, const uint8_t *expert_w8,
                           const float *expert_scales, const moe_fp8_expert *shared_w,
                           const uint16_t *shared_gate, uint16_t *out, const uint16_t *residual,
                           const float *router_bias, void *stream);

/* Device-side status of moe_ffn_forward_static's scratch array (no
 * counterpart on the reference pages): synchronises `stream`, then reads the
 * array's status word.  MOE_OK, or MOE_ETIMEOUT if a bounded wait inside a
 * kernel of an earlier static call ran out (the outputs of that call are
 * incomplete).  A non-OK word stays set across static calls until this
 * function reports it, and is cleared once reported.  Returns MOE_ECUDA
 * (sticky) if the read itself fails. */
MOE_API int moe_static_device_status(void *stream);

/* Test hook: moe_debug_wait_timeout against the static scratch array, so
 * that moe_static_device_status reports MOE_ETIMEOUT. */
MOE_API int moe_debug_wait_timeout_static(int32_t limit_us, void *stream);

/* Size in bytes of the scratch array moe_ffn_forward_static uses. */
MOE_API size_t moe_static_scratch_bytes(void);

/* moe_ffn_forward with x and out in host memory: the step a serving loop
 * makes when its tokens live on the host.  x [rows, H] and out [rows, H]
 * (bf16, 16-byte aligned) must be pinned host memory that the device can
 * address (cudaHostAlloc / cudaHostRegister; a pinned torch tensor): a first
 * kernel reads x into the workspace over the host link, the forward's
 * kernels then run as in moe_ffn_forward (path MOE_PATH_AUTO, no residual)
 * and store out straight into the host buffer.  The caller keeps ownership
 * of x and out; out is complete once the stream has passed the call (as for
 * any kernel output: synchronise or wait on an event before reading it).
 * The operation is moe_ffn_forward's (the blueprint page's Kernels table).
 * Errors: as moe_ffn_forward, plus MOE_EINVAL when x or out is not pinned,
 * device-addressable host memory. */
MOE_API int moe_ffn_forward_host(const moe_dims *d, const uint16_t *x_host, int32_t rows,
                         const uint16_t *router_w, const uint8_t *expert_w8,
                         const float *expert_scales, const moe_fp8_expert *shared_w,
                         const uint16_t *shared_gate, uint16_t *out_host,
                         const float *router_bias, void *ws, size_t ws_bytes, void *stream);

/* moe_ffn_forward with NVFP4 experts: the 397B-A17B checkpoint's expert
 * format ("The Config That Launched a Thousand GPUs: Inspecting
 * Qwen3.5-397B-A17B-NVFP4" page, modelopt NVFP4; the format is its public
 * definition): weight = e2m1(code) * e4m3(block scale) * tensor scale.  The
 * operation is the blueprint page's Kernels chain (router GEMV, top-k
 * softmax, gate/up with the shared expert, SiLU and down, weighted blend)
 * at its Precision table's arithmetic (bf16 x for gate/up, f32 h for down,
 * fp32 sums).  Layout: E contiguous expert slabs; expert_w4 [E][3*I*H/2]
 * packed codes ([W13 (2I x H/2) | W2 (H x I/2)], element 2j of a row in the
 * low nibble of byte j), expert_sf [E][3*I*H/16] e4m3 scale codes ([W13 (2I x
 * H/16) | W2 (H x I/16)]), expert_gs [E][2] fp32 (W13, W2); the shared expert
 * likewise (moe_nvfp4_expert).  The router, gate, bias, residual and out are
 * those of moe_ffn_forward; workspace as moe_workspace_bytes(d, rows).  A
 * decode-sized path: the weights stream once per row and routed pair, rows
 * in chunks of up to 4.  Errors: as moe_ffn_forward (pointers 16-byte
 * aligned, expert_gs and shared->gs 4-byte aligned). */
MOE_API int moe_ffn_forward_nvfp4(const moe_dims *d, const uint16_t *x, int32_t rows,
                          const uint16_t *router_w, const uint8_t *expert_w4,
                          const uint8_t *expert_sf, const float *expert_gs,
                          const moe_nvfp4_expert *shared, const uint16_t *shared_gate,
                          uint16_t *out, const uint16_t *residual, const float *router_bias,
                          void *ws, size_t ws_bytes, void *stream);

/* Sticky status: MOE_OK, or MOE_ECUDA after a CUDA error. */
MOE_API int moe_status(void);
/* Clear the sticky status (also clears a pending CUDA error of this thread). */
MOE_API void moe_reset_status(void);
/* Static, human-readable text for a status code. */
MOE_API const char *moe_status_string(int status);

/* Host-side fault injection, after the pages' fake device loss: the n-th
 * next call (n >= 1) fails with MOE_ECUDA before enqueueing anything, as if
 * a launch had failed, and sets the sticky status.  n = 0 disarms.  Nothing
 * runs on the device. */
MOE_API void moe_debug_inject_fault(int32_t n);

#ifdef __cplusplus
}
#endif

#endif /* MOE_FFN_H */
