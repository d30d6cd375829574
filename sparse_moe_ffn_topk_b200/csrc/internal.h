// internal.h -- host-side pieces shared by the C ABI and the kernel launchers.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "moe_ffn.h"

namespace moe {

constexpr int kMaxTopK = 32;
constexpr int kMaxExperts = 1024;
constexpr int kStepMaxRows = 4;           // decode step kernel: rows per launch; more rows run as several launches
constexpr int kStepMaxLd = (kMaxExperts + 1 + 3) / 4 * 4;  // router logits a row (E + 1, in fours), at most
constexpr int kCtrRouter = 0;           // last-arriver counter over the router's token groups
constexpr int kCtrStatus = 1;           // device status word: 0, or a MOE_* error a kernel recorded
constexpr int kMaxRouterGroups = 1024;
constexpr int kCtrStepEpoch = 8;        // decode step kernel: calls so far (the logits' tag is epoch + 1)
constexpr int kCtrStepExit = 9;         // decode step kernel: CTAs of the running call that have read the epoch
constexpr int kCtrStepReady = 16;       // decode step kernel: two sets (by epoch parity) of kStepReadyHalf ints: per
                                        // down expert (shared, then the routed list), units done, StepShape::rdy apart
constexpr int kCtrStepDiag = 2048;      // decode step kernel: per CTA, where a wait ran out (0: none); the trace
                                        // build's marks reach 2048 + 256 + 16 * CTAs
constexpr int kStepReadyHalf = (kCtrStepDiag - kCtrStepReady) / 2;
constexpr int kCtrStepLogits = 6144;    // decode step kernel: the router logits as tagged 8-byte words [rows][ld]: a
                                        // fixed place that only these words and zeros ever occupy
constexpr int kCtrRouterGroup = kCtrStepLogits + 2 * kStepMaxRows * kStepMaxLd;  // router kernel: per token group, the
                                        // CTAs done (a range of its own: the decode step leaves its unit counts set)
constexpr int kCounters = kCtrRouterGroup + kMaxRouterGroups;  // int32 words at the head of the workspace
static_assert(kCtrStepLogits % 2 == 0, "the tagged logits are 8-byte words");
static_assert(kCtrStepDiag + 256 + 16 * 236 <= kCtrStepLogits, "the trace build's marks stay below the tagged logits");
constexpr int kMaxBlendBlocks = 2048;   // H / 8 limit
constexpr int kSmallRouterRows = 64;    // the grouped-GEMM path routes up to this many rows with the router kernel

// The decode step kernel (decode_step.cu).
constexpr int kStepWarps = 8;             // consumer warps; plus one producer warp
constexpr int kStepThreads = (kStepWarps + 1) * 32;
constexpr int kStepMaxExpertsPerItem = 2; // down experts per ring item

inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// Decode-path workspace, carved from the caller's buffer: the router's
// logits and routing for all rows; h for one decode-step launch.
struct DecodeLayout {
    size_t counters, logits, topk_idx, topk_w, gsig, hterm, hsc, total;
    int ld;
};

inline DecodeLayout decode_layout(const moe_dims &d, int64_t rows)
{
    DecodeLayout L{};
    const int64_t E = d.n_experts, K = d.top_k, I = d.inter, Is = d.shared_inter;
    const int64_t imax = I > Is ? I : Is;
    const int64_t hrows = rows < kStepMaxRows ? rows : kStepMaxRows;
    size_t o = 0;
    auto take = [&](size_t bytes) { size_t at = o; o = align_up(o + bytes, 256); return at; };
    L.ld = (int)((E + 1 + 3) / 4 * 4);
    L.counters = take(sizeof(int32_t) * kCounters);
    L.logits = take(sizeof(float) * rows * L.ld);  // the router kernel's (the decode step's are in the counters)
    L.topk_idx = take(sizeof(int32_t) * rows * K);
    L.topk_w = take(sizeof(float) * rows * K);
    L.gsig = take(sizeof(float) * rows);
    L.hterm = take((size_t)8 * hrows * (K + 1) * imax);
    L.hsc = take(sizeof(float) * hrows * (K + 1) * (imax / 32));
    L.total = o;
    return L;
}

// ------------------------------------------------------------ C ABI plumbing
// Sticky status gate of every entry: MOE_ECUDA after an earlier CUDA error or
// when the host fault knob fires, else MOE_OK.
int enter();
// MOE_OK, or MOE_ECUDA (and the sticky status set) if `e` or the thread's
// last CUDA error is an error.
int finish(cudaError_t e);
// Host-side argument checks of a forward call, apart from the workspace.
int check_forward_args(const moe_dims *d, const uint16_t *x, int32_t rows, const uint16_t *router_w,
                       const uint8_t *expert_w8, const float *expert_scales, const moe_fp8_expert *shared_w,
                       const uint16_t *shared_gate, const uint16_t *out, const uint16_t *residual,
                       const float *router_bias, int32_t path, const int32_t *topk_idx_out,
                       const float *topk_w_out, const float *shared_gate_sig_out, bool out_may_alias_x);
// The layer step on a checked workspace of at least workspace_bytes(d, rows)
// bytes, after enter() returned MOE_OK.
int run_forward(const moe_dims *d, const uint16_t *x, int32_t rows, const uint16_t *router_w,
                const uint8_t *expert_w8, const float *expert_scales, const moe_fp8_expert *shared_w,
                const uint16_t *shared_gate, uint16_t *out, const uint16_t *residual, const float *router_bias,
                void *ws, void *stream, int32_t path, int32_t *topk_idx_out, float *topk_w_out,
                float *shared_gate_sig_out, const uint16_t *norm_w, double eps);

// Device properties cached per device.
struct DeviceInfo {
    int sm_count = 0;
    int cc_major = 0, cc_minor = 0;
    size_t max_smem_optin = 0;
};
const DeviceInfo &device_info();

// ------------------------------------------------------------ decode path
struct RouterLaunch {
    const moe_dims *d;
    const uint16_t *x;
    int32_t rows;
    const uint16_t *router_w;
    const float *router_bias;
    const uint16_t *shared_gate;
    int32_t *topk_idx;
    float *topk_w;
    float *gsig;
    float *logits;   // workspace
    int32_t *counters;
};
cudaError_t launch_router_topk(const RouterLaunch &a, cudaStream_t s);

// Shape of one decode-step launch (rows <= kStepMaxRows).
struct StepShape {
    bool ok;
    int grid, ns, gu_wp, gu_pieces, dn_tpi, dn_tpi_s, dn_epi, nt_max, rr_per_item;
    int x_stride;
    uint32_t o_uni, o_xb, o_xfac, o_y, o_sm, o_bar, o_gsc, o_dsc, o_cand, o_xB;
    int nb, nbuf, tbuf, tcols, rdy;
    bool cand2;
    int max_units;
    size_t smem;
};
StepShape step_shape(const moe_dims &d, int rows, int sms);
// Rows one decode-step launch takes for these dims (0: the dims do not fit).
int step_rows_per_launch(const moe_dims &d, int sms);

struct StepLaunch {
    const moe_dims *d;
    const uint16_t *x;       // the layer input, or the residual rows when norm_w is set
    const uint16_t *norm_w;  // null, or the RMSNorm weight: x = bf16(rmsnorm(x) * norm_w)
    double eps;
    int32_t rows;
    const uint16_t *router_w;
    const float *router_bias;
    const uint16_t *shared_gate;
    const uint8_t *expert_w8;
    const float *expert_scales;
    const uint8_t *shared_w8;
    const float *shared_scales;
    const uint16_t *residual;
    uint16_t *out;
    int32_t *topk_idx;
    float *topk_w;
    float *gsig;
    float *logits;
    int logits_ld;
    unsigned char *hterm;  // [rows * (K + 1)][inter / 32][256]: h as e5m2 terms (the down MMAs' B layout)
    float *hsc;            // [rows * (K + 1)][inter / 32]: each chunk's power of two
    int32_t *counters;
};
cudaError_t launch_decode_step(const StepLaunch &a, cudaStream_t s);
// nvfp4.cu: the layer with NVFP4 experts (router, then per chunk of rows
// gate/up and down + blend).
struct Nvfp4Launch {
    const moe_dims *d;
    const uint16_t *x;
    int32_t rows;
    const uint16_t *router_w;
    const float *router_bias;
    const uint16_t *shared_gate;
    const uint8_t *w4, *sf;   // experts: packed e2m1 codes, e4m3 block scales
    const float *gs;          // [E][2]
    const uint8_t *sw4, *ssf; // the shared expert
    const float *sgs;
    const uint16_t *residual;
    uint16_t *out;
    int32_t *topk_idx;        // workspace
    float *topk_w, *gsig, *logits, *h;
    int32_t *counters;
};
cudaError_t launch_nvfp4_forward(const Nvfp4Launch &a, cudaStream_t s);
int nvfp4_rows_per_chunk(const moe_dims &d);
int nvfp4_kernel_launches(const moe_dims &d, int32_t rows);
// host_io.cu: bytes (a multiple of 16) from pinned host memory (its device
// address) to dst, by a kernel.
cudaError_t launch_host_rows_in(const void *src_dev, void *dst, size_t bytes, cudaStream_t s);

// x = bf16(rmsnorm(resid) * norm_w) for `rows` rows (one CTA per row).
cudaError_t launch_rmsnorm(const uint16_t *resid, const uint16_t *norm_w, double eps, int H, int rows, uint16_t *x,
                           cudaStream_t s);

// One CTA waits on an mbarrier that nothing completes, for at most limit_ns,
// then records MOE_ETIMEOUT in counters[kCtrStatus].
cudaError_t launch_wait_probe(int32_t *counters, uint64_t limit_ns, cudaStream_t s);

// ------------------------------------------------------------ prefill path
// Bytes of workspace for `rows` rows on either path (with or without the norm).
size_t workspace_bytes(const moe_dims &d, int64_t rows);
// Offset of the normed-x buffer [rows][H] bf16 (the norm entry on the grouped path).
size_t norm_buffer_offset(const moe_dims &d, int64_t rows);
// Whether the prefill path is built into this library.
bool prefill_available();
// Kernels one prefill call launches.
int prefill_kernel_launches(const moe_dims &d, int64_t rows);
// The prefill path (router GEMM, permute, grouped FP8 GEMMs, unpermute).
// Returns a MOE_* status; launch errors come back as MOE_ECUDA.
int prefill_forward(const moe_dims &d, const uint16_t *x, int32_t rows, const uint16_t *router_w,
                    const uint8_t *expert_w8, const float *expert_scales, const uint8_t *shared_w8,
                    const float *shared_scales, const uint16_t *shared_gate, uint16_t *out,
                    const uint16_t *residual, const float *router_bias, void *ws, cudaStream_t s,
                    int32_t *topk_idx_out, float *topk_w_out, float *gsig_out, bool narrow);
// Whether the narrow grouped GEMMs (weight rows as M, up to 32 rows of a group
// as N) take these dims.
bool narrow_supported(const moe_dims &d);

}  // namespace moe
