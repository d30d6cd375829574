// router.cu -- the router kernel (bf16 router GEMV, shared-gate dot, top-k
// softmax) for moe_router_topk and for the grouped-GEMM path at up to 64
// rows, and the bounded-wait probe.
//
// router_topk_kernel: grid (router-row blocks, token groups).  Each CTA
// bulk-copies its slice of router rows into shared memory before it waits on
// the kernel that produced x (programmatic dependent launch), one warp per
// router row, bf16 x and weights with fp32 products and sums ("Qwen3.6-35B-
// A3B-FP8 on NVIDIA GB10" blueprint page, Kernels table: the router as a bf16
// dense GEMV feeding moe_topk_softmax).  The last CTA of each token group to
// finish runs the group's top-k (no CTA waits for another).
//
// Every wait is bounded (kWaitLimitNs); a wait that runs out records
// MOE_ETIMEOUT in the workspace status word and the CTA leaves.
#include <math.h>

#include <algorithm>
#include <mutex>
#include <vector>

#include "common.cuh"
#include "internal.h"
#include "launch.h"
#include "tcgen05.cuh"
#include "topk.cuh"

namespace moe {

// ------------------------------------------------------------------ helpers

__device__ __forceinline__ float dot8_bf16(uint4 w, uint4 x)
{
    float a = bf16_lo(w.x) * bf16_lo(x.x);
    float b = bf16_hi(w.x) * bf16_hi(x.x);
    a = fmaf(bf16_lo(w.y), bf16_lo(x.y), a);
    b = fmaf(bf16_hi(w.y), bf16_hi(x.y), b);
    a = fmaf(bf16_lo(w.z), bf16_lo(x.z), a);
    b = fmaf(bf16_hi(w.z), bf16_hi(x.z), b);
    a = fmaf(bf16_lo(w.w), bf16_lo(x.w), a);
    b = fmaf(bf16_hi(w.w), bf16_hi(x.w), b);
    return a + b;
}

__host__ __device__ __forceinline__ size_t align16(size_t v) { return (v + 15) & ~(size_t)15; }


// ---------------------------------------------------------------- router

constexpr int kRouterMaxRows = 4;   // router rows per CTA (one per warp)
constexpr int kRouterTok = 8;       // activation rows staged per pass

struct RouterParams {
    const uint16_t *x;
    int rows, H, E, K;
    int ld;            // logits row stride (floats, a multiple of 4)
    int rows_per_cta;  // router rows (warps) per CTA
    int group_tokens;  // activation rows per token group (gridDim.y groups)
    const uint16_t *wr;
    const float *bias;
    const uint16_t *g;
    float *logits;     // [rows, ld]; column E holds the shared-gate logit
    int32_t *topk_idx;
    float *topk_w;
    float *gsig;
    int32_t *counters;
};


// One row's top-k from the router's logits in the workspace (one warp).
template <int EPL>
__device__ void topk_row(const RouterParams &p, int t)
{
    topk_select<EPL>(p.logits + (size_t)t * p.ld, p.E, p.K, p.topk_idx + (size_t)t * p.K, p.topk_w + (size_t)t * p.K,
                     p.gsig + t);
}

__device__ void topk_rows(const RouterParams &p, int t_begin, int t_end)
{
    const int warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
    for (int t = t_begin + warp; t < t_end; t += nwarps) {
        if (p.E <= 32) topk_row<1>(p, t);
        else if (p.E <= 64) topk_row<2>(p, t);
        else if (p.E <= 128) topk_row<4>(p, t);
        else if (p.E <= 256) topk_row<8>(p, t);
        else if (p.E <= 512) topk_row<16>(p, t);
        else topk_row<32>(p, t);
    }
}

// Exclusive prefix sum over the block of one value per thread; returns the
// block total in *total.  scratch: >= 32 ints of shared memory.
__device__ int block_exclusive_scan(int v, int *scratch, int *total)
{
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nwarps = blockDim.x >> 5;
    int incl = v;
#pragma unroll
    for (int o = 1; o < kWarp; o <<= 1) {
        const int y = __shfl_up_sync(0xFFFFFFFFu, incl, o);
        if (lane >= o) incl += y;
    }
    if (lane == kWarp - 1) scratch[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        const int w = (lane < nwarps) ? scratch[lane] : 0;
        int wi = w;
#pragma unroll
        for (int o = 1; o < kWarp; o <<= 1) {
            const int y = __shfl_up_sync(0xFFFFFFFFu, wi, o);
            if (lane >= o) wi += y;
        }
        if (lane < nwarps) scratch[lane] = wi - w;
        if (lane == kWarp - 1) scratch[kWarp] = wi;
    }
    __syncthreads();
    const int r = scratch[warp] + incl - v;
    *total = scratch[kWarp];
    __syncthreads();
    return r;
}

// grid = (router-row blocks, token groups).  Shared memory: [rows_per_cta
// router rows, bf16][kRouterTok activation rows, bf16].
__global__ void __launch_bounds__(kRouterMaxRows * kWarp) router_topk_kernel(RouterParams p)
{
    extern __shared__ __align__(128) unsigned char smem[];
    __shared__ __align__(8) uint64_t bar_w, bar_x;
    __shared__ int s_last, s_abort;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int row0 = blockIdx.x * p.rows_per_cta;
    const int nrows = min(p.rows_per_cta, p.E + 1 - row0);   // rows of this CTA; the gate row is index E
    const int nrouter = max(0, min(nrows, p.E - row0));      // of which rows of Wr
    const int t_begin = blockIdx.y * p.group_tokens;
    const int t_end = min(p.rows, t_begin + p.group_tokens);
    const size_t rowb = (size_t)p.H * 2;
    unsigned char *wsm = smem;
    unsigned char *xs = smem + (size_t)p.rows_per_cta * rowb;

    // The router weights are layer constants: fetch them before waiting on
    // the kernel that produced x.
    if (threadIdx.x == 0) {
        s_abort = 0;
        mbar_init(&bar_w, 1);
        mbar_init(&bar_x, 1);
        fence_mbar_init();
        mbar_arrive_expect_tx(&bar_w, (uint32_t)(nrows * rowb));
        if (nrouter > 0) bulk_g2s(wsm, p.wr + (size_t)row0 * p.H, (uint32_t)(nrouter * rowb), &bar_w);
        if (nrouter < nrows) bulk_g2s(wsm + nrouter * rowb, p.g, (uint32_t)rowb, &bar_w);
    }
    const bool active = warp < nrows;
    const float b = (active && row0 + warp < p.E && p.bias) ? p.bias[row0 + warp] : 0.f;
    if (threadIdx.x == 0) MOE_TRACE(0, 0);
    pdl_wait();
    pdl_trigger();
    __syncthreads();
    if (!mbar_wait(&bar_w, 0, kWaitLimitNs)) s_abort = 1;
    if (threadIdx.x == 0) MOE_TRACE(0, 1);

    const uint4 *wrow = reinterpret_cast<const uint4 *>(wsm + warp * rowb);
    const uint4 *xsv = reinterpret_cast<const uint4 *>(xs);
    const int hv = p.H / 8;
    int pass = 0;
    for (int t0 = t_begin; t0 < t_end; t0 += kRouterTok, ++pass) {
        const int nt = min(kRouterTok, t_end - t0);
        __syncthreads();  // previous pass done with xs
        if (threadIdx.x == 0) {
            mbar_arrive_expect_tx(&bar_x, (uint32_t)(nt * rowb));
            bulk_g2s(xs, p.x + (size_t)t0 * p.H, (uint32_t)(nt * rowb), &bar_x);
        }
        if (!mbar_wait(&bar_x, pass & 1, kWaitLimitNs)) s_abort = 1;
        __syncthreads();
        if (s_abort) break;
        if (!active) continue;
        for (int t = 0; t < nt; ++t) {
            float acc = 0.f;
            for (int c = lane; c < hv; c += kWarp) acc += dot8_bf16(wrow[c], xsv[t * hv + c]);
            acc = warp_sum(acc);
            if (lane == 0) p.logits[(size_t)(t0 + t) * p.ld + row0 + warp] = acc + b;
        }
    }
    __syncthreads();
    if (s_abort) {  // the same decision in every thread of the CTA
        if (threadIdx.x == 0) set_status(p.counters, MOE_ETIMEOUT);
        return;
    }

    // The last CTA of this token group to finish runs the group's top-k (no
    // CTA waits for another).
    if (threadIdx.x == 0) MOE_TRACE(0, 2);
    if (threadIdx.x == 0) {
        const int prev = atomic_add_acq_rel_gpu(p.counters + kCtrRouterGroup + blockIdx.y, 1);
        s_last = (prev == (int)gridDim.x - 1);
    }
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    if (threadIdx.x == 0) MOE_TRACE(0, 3);
    topk_rows(p, t_begin, t_end);
    __syncthreads();
    if (threadIdx.x == 0) MOE_TRACE(0, 4);
    if (threadIdx.x == 0) p.counters[kCtrRouterGroup + blockIdx.y] = 0;
}

// ------------------------------------------------------------ RMSNorm

// One CTA per row: x = bf16((r / sqrt(mean r^2 + eps)) * w), the mean square
// and the product in double, rounded once to bf16 (the decode step kernel
// computes its fused norm the same way).  Used in front of the grouped-GEMM
// path; the decode step kernel fuses the norm into its first phase.
struct NormParams {
    const uint16_t *resid;
    const uint16_t *norm_w;
    double eps;
    int H;
    uint16_t *x;
};

__global__ void __launch_bounds__(256) rmsnorm_kernel(NormParams p)
{
    const uint16_t *resid = p.resid, *norm_w = p.norm_w;
    const double eps = p.eps;
    const int H = p.H;
    uint16_t *x = p.x;
    __shared__ double red[8];
    __shared__ double s_inv;
    const int t = blockIdx.x, warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    pdl_wait();
    const uint16_t *r = resid + (size_t)t * H;
    double ss = 0.0;
    for (int h = threadIdx.x; h < H; h += blockDim.x) {
        const double v = (double)bf16_bits_to_f32(r[h]);
        ss = fma(v, v, ss);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xFFFFFFFFu, ss, o);
    if (lane == 0) red[warp] = ss;
    __syncthreads();
    if (threadIdx.x == 0) {
        double tot = 0.0;
        for (int w = 0; w < (int)(blockDim.x >> 5); ++w) tot += red[w];
        s_inv = 1.0 / sqrt(tot / (double)H + eps);
    }
    __syncthreads();
    pdl_trigger();
    for (int h = threadIdx.x; h < H; h += blockDim.x)
        x[(size_t)t * H + h] =
            f64_to_bf16_rn(((double)bf16_bits_to_f32(r[h]) * s_inv) * (double)bf16_bits_to_f32(norm_w[h]));
}

// ------------------------------------------------------------ wait probe

// One thread waits on an mbarrier that expects an arrival nobody makes, with
// the same bounded wait the kernels use, and records the timeout.
__global__ void wait_probe_kernel(int32_t *counters, uint64_t limit_ns)
{
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x != 0) return;
    mbar_init(&bar, 1);
    fence_mbar_init();
    if (!mbar_wait(&bar, 0, limit_ns)) set_status(counters, MOE_ETIMEOUT);
}

// ------------------------------------------------------------- launchers

namespace {

std::mutex g_mu;

// Blocks per SM of a kernel at a dynamic shared-memory size, per device.  On
// first use on a device the kernel's dynamic shared-memory limit is set to
// the most the device allows (the attribute sets the limit, it does not
// raise it, so it is set once and never lowered).
template <typename P>
int occupancy(void (*kernel)(P), int block, size_t smem)
{
    struct Entry {
        const void *fn;
        int device;
        size_t smem;
        int blocks;
    };
    static std::vector<Entry> cache;
    static std::vector<std::pair<const void *, int>> configured;
    int dev = 0;
    cudaGetDevice(&dev);
    std::lock_guard<std::mutex> lk(g_mu);
    for (const Entry &e : cache)
        if (e.fn == (const void *)kernel && e.device == dev && e.smem == smem) return e.blocks;
    bool done = false;
    for (const auto &c : configured) done |= (c.first == (const void *)kernel && c.second == dev);
    if (!done) {
        cudaFuncAttributes fa{};
        cudaFuncGetAttributes(&fa, kernel);
        const size_t optin = device_info().max_smem_optin;
        if (optin > fa.sharedSizeBytes)
            cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)(optin - fa.sharedSizeBytes));
        // The largest shared-memory carveout, so that a gate_up and a down CTA
        // (different kernels) can be resident on one SM together.
        cudaFuncSetAttribute(kernel, cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared);
        configured.push_back({(const void *)kernel, dev});
    }
    int b = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&b, kernel, block, smem) != cudaSuccess) b = 0;
    cache.push_back({(const void *)kernel, dev, smem, b});
    return b;
}

}  // namespace

// Router launch shape: router rows per CTA (<= 32 KB of them), token groups.
struct RouterShape {
    int rows_per_cta, groups, group_tokens, ld;
    size_t smem;
};
RouterShape router_shape(const moe_dims &d, int64_t rows)
{
    RouterShape s{};
    const int H = d.hidden, E = d.n_experts;
    rows = std::max<int64_t>(rows, 1);
    s.rows_per_cta = std::max(1, std::min(kRouterMaxRows, 32768 / H));
    s.groups = (int)std::min<int64_t>((rows + kRouterTok - 1) / kRouterTok, kMaxRouterGroups);
    s.group_tokens = (int)((rows + s.groups - 1) / s.groups);
    s.smem = std::max<size_t>((size_t)(s.rows_per_cta + kRouterTok) * H * 2, (size_t)(3 * E + 33) * 4);
    s.ld = (E + 1 + 3) / 4 * 4;
    return s;
}

cudaError_t launch_rmsnorm(const uint16_t *resid, const uint16_t *norm_w, double eps, int H, int rows, uint16_t *x,
                           cudaStream_t s)
{
    NormParams p{resid, norm_w, eps, H, x};
    return launch_kernel(rmsnorm_kernel, dim3(rows), dim3(256), 0, s, p);
}

cudaError_t launch_wait_probe(int32_t *counters, uint64_t limit_ns, cudaStream_t s)
{
    wait_probe_kernel<<<1, 32, 0, s>>>(counters, limit_ns);
    return cudaGetLastError();
}

cudaError_t launch_router_topk(const RouterLaunch &a, cudaStream_t s)
{
    const moe_dims &d = *a.d;
    const RouterShape sh = router_shape(d, a.rows);
    RouterParams p;
    p.x = a.x;
    p.rows = a.rows;
    p.H = d.hidden;
    p.E = d.n_experts;
    p.K = d.top_k;
    p.ld = sh.ld;
    p.rows_per_cta = sh.rows_per_cta;
    p.group_tokens = sh.group_tokens;
    p.wr = a.router_w;
    p.bias = a.router_bias;
    p.g = a.shared_gate;
    p.logits = a.logits;
    p.topk_idx = a.topk_idx;
    p.topk_w = a.topk_w;
    p.gsig = a.gsig;
    p.counters = a.counters;
    const dim3 grid((d.n_experts + 1 + sh.rows_per_cta - 1) / sh.rows_per_cta,
                    (a.rows + sh.group_tokens - 1) / sh.group_tokens);
    if (occupancy(router_topk_kernel, sh.rows_per_cta * kWarp, sh.smem) < 1)
        return cudaErrorInvalidConfiguration;
    return launch_kernel(router_topk_kernel, grid, dim3(sh.rows_per_cta * kWarp), sh.smem, s, p);
}

}  // namespace moe
