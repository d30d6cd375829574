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

constexpr int kNvWarps = 8;   // warps per CTA of the gate/up kernel
constexpr int kNvDnWarps = 16; // of the down kernel (one CTA an SM: h is staged once per SM)

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
// block's sum times its scale; act[k * stride] is the chunk's k-th
// activation (a transposed layout: consecutive lanes read consecutive words).
__device__ __forceinline__ float chunk_dot(uint4 w, uint32_t sf2, const float *act, int stride)
{
    const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
    float blk[2] = {0.f, 0.f};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        float f[8];
        e2m1x8_to_f32(ws[i], f);
        float s = blk[i >> 1];
#pragma unroll
        for (int k = 0; k < 8; ++k) s = fmaf(f[k], act[(8 * i + k) * stride], s);
        blk[i >> 1] = s;
    }
    const float2 sc = e4m3x2_to_f32(sf2);
    return fmaf(blk[1], sc.y, blk[0] * sc.x);
}

// Gate/up: CTA (jb, p): pair p = (row t, rank r; r = K: the shared expert),
// warps j = 8 jb + w: h[p][j] = silu(gate_j . x_t) * (up_j . x_t).
__global__ void __launch_bounds__(kNvWarps * 32) nvfp4_gate_up_kernel(const NvGuParams p)
{
    extern __shared__ float xs[];  // [32][H/32 + 1]: x[32 c + k] at xs[k * xst + c]
    pdl_wait();                    // the routing, and x when a predecessor wrote it
    pdl_trigger();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int pair = blockIdx.y, t = pair / (p.K + 1), r = pair - t * (p.K + 1);
    const bool shared = r == p.K;
    const int Iu = shared ? p.Is : p.I;
    const int j = blockIdx.x * kNvWarps + warp;
    const int xst = p.H / 32 + 1;
#pragma unroll 2
    for (int i = threadIdx.x; i < p.H / 8; i += blockDim.x) {  // 8 values a thread and step
        const uint4 v = __ldg(reinterpret_cast<const uint4 *>(p.x + (size_t)t * p.H) + i);
        const uint32_t vw[4] = {v.x, v.y, v.z, v.w};
        const int c = i >> 2, k0 = (i & 3) * 8;
#pragma unroll
        for (int m = 0; m < 4; ++m) {
            xs[(k0 + 2 * m) * xst + c] = bf16_bits_to_f32(vw[m] & 0xFFFFu);
            xs[(k0 + 2 * m + 1) * xst + c] = bf16_bits_to_f32(vw[m] >> 16);
        }
    }
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
    constexpr int kC = 4;  // 16-byte chunks (32 codes) a lane loads before using any
    for (int c0 = 0; c0 < p.H / 32; c0 += 32 * kC) {
        uint4 qg[kC], qu[kC];
        uint32_t sg[kC], su[kC];
#pragma unroll
        for (int i = 0; i < kC; ++i) {
            const int c = c0 + lane + 32 * i;
            if (c < p.H / 32) {
                qg[i] = __ldg(reinterpret_cast<const uint4 *>(wg) + c);
                qu[i] = __ldg(reinterpret_cast<const uint4 *>(wu) + c);
                sg[i] = __ldg(reinterpret_cast<const uint16_t *>(fg) + c);
                su[i] = __ldg(reinterpret_cast<const uint16_t *>(fu) + c);
            }
        }
#pragma unroll
        for (int i = 0; i < kC; ++i) {
            const int c = c0 + lane + 32 * i;
            if (c < p.H / 32) {
                g += chunk_dot(qg[i], sg[i], xs + c, xst);
                u += chunk_dot(qu[i], su[i], xs + c, xst);
            }
        }
    }
    g = warp_sum(g) * gs13;
    u = warp_sum(u) * gs13;
    if (lane == 0) p.h[(size_t)pair * p.imax + j] = siluf_(g) * u;
}

// Down + blend: warp w of CTA b takes output rows n = 16 b + w + 16 G k; per
// row t of the chunk, out[t][n] = bf16(sum_r w_r gs2_r (W2_r[n] . h_r) +
// gsig gs2_s (W2_s[n] . h_s) (+ residual)).
__global__ void __launch_bounds__(kNvDnWarps * 32) nvfp4_down_blend_kernel(const NvDownParams p)
{
    // h of every pair, transposed by 16-value blocks: h[p][16 b + i] at
    // hs[p * hpst + i * hst + b], so that the lanes (b = lane, lane + 32, ...)
    // read consecutive words
    extern __shared__ float hs[];
    pdl_wait();                    // h from the gate/up kernel
    pdl_trigger();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int np = p.rows * (p.K + 1);
    const int hst = p.imax / 16 + 1, hpst = 16 * hst;
#pragma unroll 4
    for (int i = threadIdx.x; i < np * p.imax / 4; i += blockDim.x) {
        const float4 v = __ldcg(reinterpret_cast<const float4 *>(p.h) + i);
        const int pr = (4 * i) / p.imax, o = 4 * i - pr * p.imax, b = o >> 4, k = o & 15;
        float *d = hs + (size_t)pr * hpst + b;
        d[k * hst] = v.x;
        d[(k + 1) * hst] = v.y;
        d[(k + 2) * hst] = v.z;
        d[(k + 3) * hst] = v.w;
    }
    __syncthreads();
    // Per output row and row of x: each lane's share of every pair's dot
    // product (16-code blocks b = lane, lane + 32, ...), times the pair's
    // blend weight and tensor scale, summed over the pairs in rank order
    // (the shared expert last); then one warp sum.  The loads of a group of
    // pairs are all issued before any is used.
    constexpr int kG = 4;  // pairs a group
    for (int n = blockIdx.x * kNvDnWarps + warp; n < p.H; n += gridDim.x * kNvDnWarps) {
        for (int t = 0; t < p.rows; ++t) {
            float acc = 0.f;
            for (int r0 = 0; r0 <= p.K; r0 += kG) {
                uint2 q[kG][2];
                uint32_t f[kG][2];
                float wgt[kG];
                int nb[kG];
                const float *hp[kG];
#pragma unroll
                for (int g = 0; g < kG; ++g) {
                    const int r = r0 + g;
                    nb[g] = 0;
                    if (r > p.K) continue;
                    const bool shared = r == p.K;
                    const int Iu = shared ? p.Is : p.I;
                    const int e = shared ? 0 : __ldg(p.topk_idx + (size_t)t * p.K + r);
                    const size_t slab4 = (size_t)3 * Iu * p.H / 2, slabf = (size_t)3 * Iu * p.H / 16;
                    const uint8_t *w2 = (shared ? p.sw4 : p.w4 + (size_t)e * slab4) + (size_t)Iu * p.H +
                                        (size_t)n * (Iu / 2);
                    const uint8_t *f2 = (shared ? p.ssf : p.sf + (size_t)e * slabf) + (size_t)Iu * p.H / 8 +
                                        (size_t)n * (Iu / 16);
                    const float gs2 = shared ? __ldg(p.sgs + 1) : __ldg(p.gs + 2 * (size_t)e + 1);
                    wgt[g] = (shared ? __ldg(p.gsig + t) : __ldg(p.topk_w + (size_t)t * p.K + r)) * gs2;
                    hp[g] = hs + (size_t)(t * (p.K + 1) + r) * hpst;
                    nb[g] = Iu / 16;
#pragma unroll
                    for (int k = 0; k < 2; ++k) {
                        const int b = lane + 32 * k;
                        if (b < nb[g]) {
                            q[g][k] = __ldg(reinterpret_cast<const uint2 *>(w2) + b);
                            f[g][k] = __ldg(f2 + b);
                        }
                    }
                }
#pragma unroll
                for (int g = 0; g < kG; ++g) {
                    if (!nb[g]) continue;
                    float sum = 0.f;
#pragma unroll
                    for (int k = 0; k < 2; ++k) {
                        const int b = lane + 32 * k;
                        if (b >= nb[g]) continue;
                        float v[8], blk = 0.f;
                        e2m1x8_to_f32(q[g][k].x, v);
#pragma unroll
                        for (int i = 0; i < 8; ++i) blk = fmaf(v[i], hp[g][i * hst + b], blk);
                        e2m1x8_to_f32(q[g][k].y, v);
#pragma unroll
                        for (int i = 0; i < 8; ++i) blk = fmaf(v[i], hp[g][(8 + i) * hst + b], blk);
                        sum = fmaf(blk, e4m3x2_to_f32(f[g][k]).x, sum);
                    }
                    // blocks beyond 64 a row (inter above 1024): the same, one at a time
                    for (int b = lane + 64; b < nb[g]; b += 32) {
                        const int r = r0 + g;
                        const bool shared = r == p.K;
                        const int Iu = shared ? p.Is : p.I;
                        const int e = shared ? 0 : __ldg(p.topk_idx + (size_t)t * p.K + r);
                        const uint8_t *w2 = (shared ? p.sw4 : p.w4 + (size_t)e * ((size_t)3 * Iu * p.H / 2)) +
                                            (size_t)Iu * p.H + (size_t)n * (Iu / 2);
                        const uint8_t *f2 = (shared ? p.ssf : p.sf + (size_t)e * ((size_t)3 * Iu * p.H / 16)) +
                                            (size_t)Iu * p.H / 8 + (size_t)n * (Iu / 16);
                        const uint2 qq = __ldg(reinterpret_cast<const uint2 *>(w2) + b);
                        float v[8], blk = 0.f;
                        e2m1x8_to_f32(qq.x, v);
#pragma unroll
                        for (int i = 0; i < 8; ++i) blk = fmaf(v[i], hp[g][i * hst + b], blk);
                        e2m1x8_to_f32(qq.y, v);
#pragma unroll
                        for (int i = 0; i < 8; ++i) blk = fmaf(v[i], hp[g][(8 + i) * hst + b], blk);
                        sum = fmaf(blk, e4m3x2_to_f32(__ldg(f2 + b)).x, sum);
                    }
                    acc = fmaf(wgt[g], sum, acc);
                }
            }
            acc = warp_sum(acc);
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
    const size_t per_row = (size_t)(d.top_k + 1) * 16 * (std::max(d.inter, d.shared_inter) / 16 + 1) * 4;
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
                          dim3(kNvWarps * 32), (size_t)32 * (H / 32 + 1) * 4, s, g);
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
        const int grid = std::min(device_info().sm_count, (H + kNvDnWarps - 1) / kNvDnWarps);
        e = launch_kernel(nvfp4_down_blend_kernel, dim3(grid), dim3(kNvDnWarps * 32),
                          (size_t)n * (K + 1) * 16 * (imax / 16 + 1) * 4, s, dp);
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
