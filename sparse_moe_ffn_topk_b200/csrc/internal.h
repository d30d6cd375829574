// internal.h -- host-side pieces shared by the C ABI and the kernel launchers.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "moe_ffn.h"

namespace moe {

constexpr int kMaxTopK = 32;
constexpr int kMaxExperts = 1024;
constexpr int kCounters = 4096;         // int32 counters at the head of the workspace
constexpr int kCtrRouter = 0;           // last-arriver counter over the router's token groups
constexpr int kCtrStatus = 1;           // device status word: 0, or a MOE_* error a kernel recorded
constexpr int kCtrRouterGroup = 16;     // [16, 16 + kMaxRouterGroups): per token-group counters
constexpr int kMaxRouterGroups = 1024;
constexpr int kCtrBlend = 2048;         // first of the down/blend per-row-block counters
constexpr int kMaxBlendBlocks = kCounters - kCtrBlend;
constexpr int kDescPairs = 8;           // pair ids a stage descriptor carries

inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// Decode-path workspace, carved from the caller's buffer.
struct DecodeLayout {
    size_t counters, logits, xq, xsc, topk_idx, topk_w, gsig, h_routed, h_shared, yslot, total;
};

// Tile shapes of the decode kernels for given dims and rows.
struct DecodeShape {
    int router_rows, router_groups, router_group_tokens, logits_ld;
    size_t router_smem;
    int gu_pairs, tok, gu_stages;
    size_t gu_smem;
    int dn_rows, dn_stages;
    size_t dn_smem;
    // down by output block (few rows): experts per stage; 0 = the item-based down kernel
    int ds_ue;
    // gate_up prefetches the active experts' down weights into L2
    bool l2_w2;
};
DecodeShape decode_shape(const moe_dims &d, int64_t rows);

inline DecodeLayout decode_layout(const moe_dims &d, int64_t rows)
{
    DecodeLayout L{};
    const int64_t E = d.n_experts, K = d.top_k, H = d.hidden, I = d.inter, Is = d.shared_inter;
    size_t o = 0;
    auto take = [&](size_t bytes) { size_t at = o; o = align_up(o + bytes, 256); return at; };
    L.counters = take(sizeof(int32_t) * kCounters);
    L.logits = take(sizeof(float) * rows * ((E + 1 + 3) / 4 * 4));
    L.xq = take((size_t)rows * 2 * H);
    L.xsc = take(sizeof(float) * rows * (H / 128));
    L.topk_idx = take(sizeof(int32_t) * rows * K);
    L.topk_w = take(sizeof(float) * rows * K);
    L.gsig = take(sizeof(float) * rows);
    L.h_routed = take(sizeof(float) * rows * K * I);
    L.h_shared = take(sizeof(float) * rows * Is);
    L.yslot = take(sizeof(float) * rows * (K + 1) * H);
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
                       const float *topk_w_out, const float *shared_gate_sig_out);
// The layer step on a checked workspace of at least workspace_bytes(d, rows)
// bytes, after enter() returned MOE_OK.
int run_forward(const moe_dims *d, const uint16_t *x, int32_t rows, const uint16_t *router_w,
                const uint8_t *expert_w8, const float *expert_scales, const moe_fp8_expert *shared_w,
                const uint16_t *shared_gate, uint16_t *out, const uint16_t *residual, const float *router_bias,
                void *ws, void *stream, int32_t path, int32_t *topk_idx_out, float *topk_w_out,
                float *shared_gate_sig_out);

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
    uint8_t *xq;     // workspace: x as hi/lo e4m3 (nullptr: not needed)
    float *xsc;
    int32_t *counters;
};
cudaError_t launch_router_topk(const RouterLaunch &a, cudaStream_t s);

struct ExpertsLaunch {
    const moe_dims *d;
    const uint16_t *x;
    const uint8_t *xq;
    const float *xsc;
    int32_t rows;
    const uint8_t *expert_w8;
    const float *expert_scales;
    const uint8_t *shared_w8;
    const float *shared_scales;
    const uint16_t *residual;
    uint16_t *out;
    const int32_t *topk_idx;
    const float *topk_w;
    const float *gsig;
    float *h_routed;
    float *h_shared;
    float *yslot;
    int32_t *counters;
};
cudaError_t launch_decode_experts(const ExpertsLaunch &a, cudaStream_t s);

// One CTA waits on an mbarrier that nothing completes, for at most limit_ns,
// then records MOE_ETIMEOUT in counters[kCtrStatus].
cudaError_t launch_wait_probe(int32_t *counters, uint64_t limit_ns, cudaStream_t s);

// ------------------------------------------------------------ prefill path
// Bytes of workspace for `rows` rows on either path.
size_t workspace_bytes(const moe_dims &d, int64_t rows);
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
