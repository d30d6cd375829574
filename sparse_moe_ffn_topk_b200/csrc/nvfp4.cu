// nvfp4.cu -- the layer step with NVFP4 experts (moe_ffn_forward_nvfp4).
//
// The 397B-A17B checkpoint stores its experts as NVFP4 ("The Config That
// Launched a Thousand GPUs: Inspecting Qwen3.5-397B-A17B-NVFP4" page; the
// format is its public definition): e2m1 codes packed two to a byte (element
// 2j in the low nibble of byte j), one e4m3 scale per 16 consecutive
// elements of a row, one fp32 scale per matrix; a weight is e2m1(code) *
// e4m3(scale) * tensor scale.  The step is the FP8 layer's (the blueprint
// page's Kernels chain) with that dequantisation, at the Precision table's
// arithmetic: bf16 x for gate/up and fp32 h for down, every product e2m1 x
// activation exact inside an fp32 multiply-add, sums in fp32, each 16-element
// block's sum times its e4m3 scale, each dot product times the tensor scale.
//
// Kernels: the router and top-k (router.cu) into the workspace; then, per
// chunk of rows, gate/up (one warp per (pair, intermediate row): the gate
// and the up row against x in shared memory, 16-byte lane loads of codes,
// h = silu(gate) * up in fp32 to the workspace) and down + blend (one warp
// per output row over every pair of the chunk's rows, h in shared memory;
// rank order, then the shared expert times its sigmoid gate, then the
// residual, one rounding to bf16).  The weights stream once per (row, pair):
// a decode-sized path.
#include <cuda_runtime.h>

#include <algorithm>

#include "common.cuh"
#include "internal.h"
#include "launch.h"

namespace moe {
namespace {

constexpr int kNvWarps = 8;  // warps per CTA of both kernels

struct NvGuParams {
    const uint16_t *x;        // [rows, H] bf16 (the chunk's first row)
    const int32_t *topk_idx;  // [rows, K] (the chunk's first row)
    const uint8_t *w4;        // experts' packed codes
    const uint8_t *sf;        // experts' e4m3 block scales
    const float *gs;          // [E][2]
    const uint8_t *sw4, *ssf; // the shared expert
    const float *sgs;
    float *h;                 // [pairs][imax]
    int H, K, I, Is, imax;
};

struct NvDownParams {
    const int32_t *topk_idx;  // the chunk's first row
    const float *topk_w;
    const float *gsig;
    const uint8_t *w4, *sf;
    const float *gs;
    const uint8_t *sw4, *ssf;
    const float *sgs;
    const float *h;           // [pairs][imax]
    const uint16_t *residual; // nullable, the chunk's first row
    uint16_t *out;            // the chunk's first row
    int rows, H, K, I, Is, imax;
};

// Eight e2m1 codes (a word, lowest nibble first) -> fp32, exactly (e2m1 ->
// f16 -> f32).
__device__ __forceinline__ void e2m1x8_to_f32(uint32_t w, float (&f)[8])
{
    uint32_t h0, h1, h2, h3;
    asm("{ .reg .b8 a, b, c, d; mov.b32 {a, b, c, d}, %4;"
        " cvt.rn.f16x2.e2m1x2 %0, a; cvt.rn.f16x2.e2m1x2 %1, b;"
        " cvt.rn.f16x2.e2m1x2 %2, c; cvt.rn.f16x2.e2m1x2 %3, d; }"
        : "=r"(h0), "=r"(h1), "=r"(h2), "=r"(h3)
        : "r"(w));
    const uint32_t hh[4] = {h0, h1, h2, h3};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 v = __half22float2(*reinterpret_cast<const __half2 *>(&hh[i]));
        f[2 * i] = v.x;
        f[2 * i + 1] = v.y;
    }
}

// Two e4m3 codes (low byte first) -> fp32.
__device__ __forceinline__ float2 e4m3x2_to_f32(uint32_t two)
{
    uint32_t h;
    asm("{ .reg .b16 l, u; mov.b32 {l, u}, %1; cvt.rn.f16x2.e4m3x2 %0, l; }" : "=r"(h) : "r"(two));
    return __half22float2(*reinterpret_cast<const __half2 *>(&h));
}

// Sum over a 16-byte chunk (32 codes, two scale blocks) of code * act, each
// block's sum times its scale.
__device__ __forceinline__ float chunk_dot(uint4 w, uint32_t sf2, const float *act)
{
    const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
    float blk[2] = {0.f, 0.f};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        float f[8];
        e2m1x8_to_f32(ws[i], f);
        const float4 a0 = *reinterpret_cast<const float4 *>(act + 8 * i);
        const float4 a1 = *reinterpret_cast<const float4 *>(act + 8 * i + 4);
        float s = blk[i >> 1];
        s = fmaf(f[0], a0.x, s);
        s = fmaf(f[1], a0.y, s);
        s = fmaf(f[2], a0.z, s);
        s = fmaf(f[3], a0.w, s);
        s = fmaf(f[4], a1.x, s);
        s = fmaf(f[5], a1.y, s);
        s = fmaf(f[6], a1.z, s);
        s = fmaf(f[7], a1.w, s);
        blk[i >> 1] = s;
    }
    const float2 sc = e4m3x2_to_f32(sf2);
    return fmaf(blk[1], sc.y, blk[0] * sc.x);
}

// Gate/up: CTA (jb, p): pair p = (row t, rank r; r = K: the shared expert),
// warps j = 8 jb + w: h[p][j] = silu(gate_j . x_t) * (up_j . x_t).
__global__ void __launch_bounds__(kNvWarps * 32) nvfp4_gate_up_kernel(const NvGuParams p)
{
    extern __shared__ float xs[];  // [H]
    pdl_wait();                    // the routing, and x when a predecessor wrote it
    pdl_trigger();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int pair = blockIdx.y, t = pair / (p.K + 1), r = pair - t * (p.K + 1);
    const bool shared = r == p.K;
    const int Iu = shared ? p.Is : p.I;
    const int j = blockIdx.x * kNvWarps + warp;
    for (int i = threadIdx.x; i < p.H; i += blockDim.x) xs[i] = bf16_bits_to_f32(p.x[(size_t)t * p.H + i]);
    __syncthreads();
    if (j >= Iu) return;
    const int e = shared ? 0 : __ldg(p.topk_idx + (size_t)t * p.K + r);
    const size_t slab4 = (size_t)3 * Iu * p.H / 2, slabf = (size_t)3 * Iu * p.H / 16;
    const uint8_t *w4 = shared ? p.sw4 : p.w4 + (size_t)e * slab4;
    const uint8_t *sf = shared ? p.ssf : p.sf + (size_t)e * slabf;
    const float gs13 = shared ? __ldg(p.sgs) : __ldg(p.gs + 2 * (size_t)e);
    const uint8_t *wg = w4 + (size_t)j * (p.H / 2), *wu = w4 + (size_t)(Iu + j) * (p.H / 2);
    const uint8_t *fg = sf + (size_t)j * (p.H / 16), *fu = sf + (size_t)(Iu + j) * (p.H / 16);
    float g = 0.f, u = 0.f;
    for (int c = lane; c < p.H / 32; c += 32) {  // 16-byte chunks of 32 codes
        const uint4 qg = __ldg(reinterpret_cast<const uint4 *>(wg) + c);
        const uint4 qu = __ldg(reinterpret_cast<const uint4 *>(wu) + c);
        const uint32_t sg = *reinterpret_cast<const uint16_t *>(fg + 2 * c);
        const uint32_t su = *reinterpret_cast<const uint16_t *>(fu + 2 * c);
        g += chunk_dot(qg, sg, xs + 32 * c);
        u += chunk_dot(qu, su, xs + 32 * c);
    }
    g = warp_sum(g) * gs13;
    u = warp_sum(u) * gs13;
    if (lane == 0) p.h[(size_t)pair * p.imax + j] = siluf_(g) * u;
}

// Down + blend: warp w of CTA b takes output rows n = 8 b + w + 8 G k; per
// row t of the chunk, y_p[n] = (W2_e[n] . h[p]) * gs2 for its k pairs and the
// shared expert, out[t][n] = bf16(sum_r w_r y_r + gsig y_s (+ residual)).
__global__ void __launch_bounds__(kNvWarps * 32) nvfp4_down_blend_kernel(const NvDownParams p)
{
    extern __shared__ float hs[];  // [pairs][imax]
    pdl_wait();                    // h from the gate/up kernel
    pdl_trigger();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int np = p.rows * (p.K + 1);
    for (int i = threadIdx.x; i < np * p.imax / 4; i += blockDim.x)
        reinterpret_cast<float4 *>(hs)[i] = __ldcg(reinterpret_cast<const float4 *>(p.h) + i);
    __syncthreads();
    for (int n = blockIdx.x * kNvWarps + warp; n < p.H; n += gridDim.x * kNvWarps) {
        for (int t = 0; t < p.rows; ++t) {
            float acc = 0.f;
            for (int r = 0; r <= p.K; ++r) {
                const bool shared = r == p.K;
                const int Iu = shared ? p.Is : p.I;
                const int e = shared ? 0 : __ldg(p.topk_idx + (size_t)t * p.K + r);
                const size_t slab4 = (size_t)3 * Iu * p.H / 2, slabf = (size_t)3 * Iu * p.H / 16;
                const uint8_t *w2 = (shared ? p.sw4 : p.w4 + (size_t)e * slab4) + (size_t)Iu * p.H +
                                    (size_t)n * (Iu / 2);
                const uint8_t *f2 = (shared ? p.ssf : p.sf + (size_t)e * slabf) + (size_t)Iu * p.H / 8 +
                                    (size_t)n * (Iu / 16);
                const float gs2 = shared ? __ldg(p.sgs + 1) : __ldg(p.gs + 2 * (size_t)e + 1);
                const float *hp = hs + (size_t)(t * (p.K + 1) + r) * p.imax;
                float s = 0.f;
                for (int b = lane; b < Iu / 16; b += 32) {  // 8-byte blocks of 16 codes, one scale each
                    const uint2 q = __ldg(reinterpret_cast<const uint2 *>(w2) + b);
                    float f[8];
                    float blk = 0.f;
                    e2m1x8_to_f32(q.x, f);
#pragma unroll
                    for (int i = 0; i < 8; ++i) blk = fmaf(f[i], hp[16 * b + i], blk);
                    e2m1x8_to_f32(q.y, f);
#pragma unroll
                    for (int i = 0; i < 8; ++i) blk = fmaf(f[i], hp[16 * b + 8 + i], blk);
                    s = fmaf(blk, e4m3x2_to_f32(f2[b]).x, s);
                }
                const float y = warp_sum(s) * gs2;
                acc = fmaf(shared ? __ldg(p.gsig + t) : __ldg(p.topk_w + (size_t)t * p.K + r), y, acc);
            }
            if (lane == 0) {
                const size_t o = (size_t)t * p.H + n;
                if (p.residual) acc += bf16_bits_to_f32(p.residual[o]);
                p.out[o] = f32_to_bf16_bits(acc);
            }
        }
    }
}

}  // namespace

int nvfp4_rows_per_chunk(const moe_dims &d)
{
    // h of a chunk's pairs in one CTA's shared memory (up to 160 KB), at most 4 rows
    const size_t per_row = (size_t)(d.top_k + 1) * std::max(d.inter, d.shared_inter) * 4;
    return (int)std::max<size_t>(1, std::min<size_t>(4, (size_t)160 * 1024 / per_row));
}

cudaError_t launch_nvfp4_forward(const Nvfp4Launch &a, cudaStream_t s)
{
    const moe_dims &d = *a.d;
    const int H = d.hidden, K = d.top_k, I = d.inter, Is = d.shared_inter, imax = std::max(I, Is);
    RouterLaunch ra;
    ra.d = a.d;
    ra.x = a.x;
    ra.rows = a.rows;
    ra.router_w = a.router_w;
    ra.router_bias = a.router_bias;
    ra.shared_gate = a.shared_gate;
    ra.topk_idx = a.topk_idx;
    ra.topk_w = a.topk_w;
    ra.gsig = a.gsig;
    ra.logits = a.logits;
    ra.counters = a.counters;
    cudaError_t e = launch_router_topk(ra, s);
    if (e != cudaSuccess) return e;
    static bool configured[64] = {};  // per device: the kernels' shared memory above 48 KB
    int dev = 0;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (!configured[dev]) {
        e = cudaFuncSetAttribute(nvfp4_down_blend_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 160 * 1024);
        if (e != cudaSuccess) return e;
        e = cudaFuncSetAttribute(nvfp4_gate_up_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 64 * 1024);
        if (e != cudaSuccess) return e;
        configured[dev] = true;
    }
    const int rc = nvfp4_rows_per_chunk(d);
    for (int t0 = 0; t0 < a.rows; t0 += rc) {
        const int n = std::min(rc, a.rows - t0);
        NvGuParams g;
        g.x = a.x + (size_t)t0 * H;
        g.topk_idx = a.topk_idx + (size_t)t0 * K;
        g.w4 = a.w4;
        g.sf = a.sf;
        g.gs = a.gs;
        g.sw4 = a.sw4;
        g.ssf = a.ssf;
        g.sgs = a.sgs;
        g.h = a.h;
        g.H = H;
        g.K = K;
        g.I = I;
        g.Is = Is;
        g.imax = imax;
        e = launch_kernel(nvfp4_gate_up_kernel, dim3((imax + kNvWarps - 1) / kNvWarps, n * (K + 1)),
                          dim3(kNvWarps * 32), (size_t)H * 4, s, g);
        if (e != cudaSuccess) return e;
        NvDownParams dp;
        dp.topk_idx = a.topk_idx + (size_t)t0 * K;
        dp.topk_w = a.topk_w + (size_t)t0 * K;
        dp.gsig = a.gsig + t0;
        dp.w4 = a.w4;
        dp.sf = a.sf;
        dp.gs = a.gs;
        dp.sw4 = a.sw4;
        dp.ssf = a.ssf;
        dp.sgs = a.sgs;
        dp.h = a.h;
        dp.residual = a.residual ? a.residual + (size_t)t0 * H : nullptr;
        dp.out = a.out + (size_t)t0 * H;
        dp.rows = n;
        dp.H = H;
        dp.K = K;
        dp.I = I;
        dp.Is = Is;
        dp.imax = imax;
        const int grid = std::min(4 * device_info().sm_count, (H + kNvWarps - 1) / kNvWarps);
        e = launch_kernel(nvfp4_down_blend_kernel, dim3(grid), dim3(kNvWarps * 32),
                          (size_t)n * (K + 1) * imax * 4, s, dp);
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

int nvfp4_kernel_launches(const moe_dims &d, int32_t rows)
{
    if (rows <= 0) return 0;
    const int rc = nvfp4_rows_per_chunk(d);
    return 1 + 2 * ((rows + rc - 1) / rc);
}

}  // namespace moe
