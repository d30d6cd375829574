// decode.cu -- decode path (rows <= a few dozen): weight-streaming GEMVs.
//
// Three launches chained with programmatic dependent launch:
//   1. router_topk_kernel: bf16 router GEMV + shared-gate dot, one warp per
//      router row with the row held in registers and the activation rows in
//      shared memory; the last CTA to finish runs the top-k softmax and
//      builds the per-expert row lists (expert dedup across rows).
//   2. gate_up_kernel: for every (active expert, chunk of 16 gate/up row
//      pairs) work item, a warp per row pair streams both FP8 rows with
//      16-byte lane loads, applies the 128x128 block scales in registers and
//      writes h = silu(gate) * up in fp32.
//   3. down_blend_kernel: for every (active expert, 32 output rows) item, a
//      warp per output row streams the FP8 down row against h (shared
//      memory), scales by the routing weight (or the shared gate) and writes
//      one partial per routed slot; the last item to finish a 32-row chunk
//      blends the k partials in rank order plus the shared partial (plus the
//      residual) and rounds once to bf16.
//
// The pages' kernels are the prior art: the GB10 blueprint's per-layer MoE
// chain (router GEMV, top-k softmax, gate_up with the shared expert fused,
// silu+down, weighted blend; fp8/block128x128 weights read against bf16 and
// f32 activations) and the colibri PR's decode GEMV (one warp per output row,
// 16 bytes per lane, the activation in shared memory).
#include <math.h>

#include <algorithm>
#include <mutex>

#include "common.cuh"
#include "internal.h"

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

// 4 e4m3 codes (one word) against 4 bf16 activations (two words).
__device__ __forceinline__ void fma4_e4m3_bf16(uint32_t w, uint32_t x01, uint32_t x23, float &a, float &b)
{
    float2 f0 = e4m3x2_to_f32x2(static_cast<uint16_t>(w & 0xFFFFu));
    float2 f1 = e4m3x2_to_f32x2(static_cast<uint16_t>(w >> 16));
    a = fmaf(f0.x, bf16_lo(x01), a);
    b = fmaf(f0.y, bf16_hi(x01), b);
    a = fmaf(f1.x, bf16_lo(x23), a);
    b = fmaf(f1.y, bf16_hi(x23), b);
}

// 16 e4m3 codes against 16 bf16 activations (two 16-byte words).
__device__ __forceinline__ float dot16_e4m3_bf16(uint4 w, uint4 xa, uint4 xb)
{
    float a = 0.f, b = 0.f;
    fma4_e4m3_bf16(w.x, xa.x, xa.y, a, b);
    fma4_e4m3_bf16(w.y, xa.z, xa.w, a, b);
    fma4_e4m3_bf16(w.z, xb.x, xb.y, a, b);
    fma4_e4m3_bf16(w.w, xb.z, xb.w, a, b);
    return a + b;
}

__device__ __forceinline__ void fma4_e4m3_f32(uint32_t w, float4 h, float &a, float &b)
{
    float2 f0 = e4m3x2_to_f32x2(static_cast<uint16_t>(w & 0xFFFFu));
    float2 f1 = e4m3x2_to_f32x2(static_cast<uint16_t>(w >> 16));
    a = fmaf(f0.x, h.x, a);
    b = fmaf(f0.y, h.y, b);
    a = fmaf(f1.x, h.z, a);
    b = fmaf(f1.y, h.w, b);
}

__device__ __forceinline__ uint32_t ordered_key(float f)
{
    uint32_t u = __float_as_uint(f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// ---------------------------------------------------------------- router

constexpr int kRouterWarps = 16;  // router rows per CTA (one per warp)
constexpr int kRouterTok = 8;     // activation rows staged per pass

struct RouterParams {
    const uint16_t *x;
    int rows, H, E, K;
    const uint16_t *wr;
    const float *bias;
    const uint16_t *g;
    float *logits;
    int32_t *topk_idx;
    float *topk_w;
    float *gsig;
    int32_t *counters;
    int32_t *plan;
};

// Top-k of every row (warp per row), run by the last router CTA.  Logits are
// compared as order-preserving 32-bit keys; 0 marks a taken (or absent)
// expert and a NaN logit gets key 1, so every round selects a valid,
// untaken expert even on non-finite input.  Equal keys go to the lower
// expert index.
__device__ void router_topk_rows(const RouterParams &p)
{
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int t = warp; t < p.rows; t += kRouterWarps) {
        const float *lrow = p.logits + (size_t)t * (p.E + 1);
        uint32_t v[kMaxExperts / kWarp];
#pragma unroll
        for (int i = 0; i < kMaxExperts / kWarp; ++i) {
            const int e = lane + kWarp * i;
            const float l = (e < p.E) ? __ldcg(lrow + e) : 0.f;
            v[i] = (e < p.E) ? (isnan(l) ? 1u : max(ordered_key(l), 2u)) : 0u;
        }
        int my_e = 0;
        float my_v = 0.f;
        for (int r = 0; r < p.K; ++r) {
            uint32_t bk = 0;
            int be = 0x7FFFFFFF;
#pragma unroll
            for (int i = 0; i < kMaxExperts / kWarp; ++i)
                if (v[i] > bk) { bk = v[i]; be = lane + kWarp * i; }
            const uint32_t kmax = __reduce_max_sync(0xFFFFFFFFu, bk);
            const int emin = (int)__reduce_min_sync(0xFFFFFFFFu, bk == kmax ? (uint32_t)be : 0x7FFFFFFFu);
#pragma unroll
            for (int i = 0; i < kMaxExperts / kWarp; ++i)
                if (lane + kWarp * i == emin) v[i] = 0u;
            if (lane == r) { my_e = emin; my_v = __ldcg(lrow + emin); }
        }
        const float top = __shfl_sync(0xFFFFFFFFu, my_v, 0);
        const float ev = (lane < p.K) ? expf(my_v - top) : 0.f;
        const float sum = warp_sum(ev);
        if (lane < p.K) {
            p.topk_idx[(size_t)t * p.K + lane] = my_e;
            p.topk_w[(size_t)t * p.K + lane] = ev / sum;
        }
        if (lane == 0) p.gsig[t] = sigmoidf_(__ldcg(lrow + p.E));
    }
}

// Per-expert lists of routed pairs (pair id = t*K + r), active experts in
// ascending id, pairs within an expert in ascending pair id.
__device__ void router_build_plan(const RouterParams &p, int *cnt, int *cursor)
{
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int E = p.E, P = p.rows * p.K;
    int32_t *n_active = p.plan;
    int32_t *act_e = p.plan + 1;
    int32_t *act_off = act_e + E;
    int32_t *pairs = act_off + E + 1;
    for (int e = threadIdx.x; e < E; e += blockDim.x) cnt[e] = 0;
    __syncthreads();
    for (int i = threadIdx.x; i < P; i += blockDim.x) atomicAdd(&cnt[__ldcg(p.topk_idx + i)], 1);
    __syncthreads();
    if (warp == 0) {
        int run = 0, nact = 0;
        for (int e0 = 0; e0 < E; e0 += kWarp) {
            const int e = e0 + lane;
            const int c = (e < E) ? cnt[e] : 0;
            int incl = c;
#pragma unroll
            for (int o = 1; o < kWarp; o <<= 1) {
                const int y = __shfl_up_sync(0xFFFFFFFFu, incl, o);
                if (lane >= o) incl += y;
            }
            const int excl = run + incl - c;
            const uint32_t act = __ballot_sync(0xFFFFFFFFu, c > 0);
            const int apos = nact + __popc(act & ((1u << lane) - 1u));
            if (c > 0) {
                act_e[apos] = e;
                act_off[apos] = excl;
                cursor[e] = excl;
            }
            run += __shfl_sync(0xFFFFFFFFu, incl, kWarp - 1);
            nact += __popc(act);
        }
        if (lane == 0) {
            act_off[nact] = run;
            n_active[0] = nact;
        }
        __syncwarp();
        for (int p0 = 0; p0 < P; p0 += kWarp) {
            const int i = p0 + lane;
            const int e = (i < P) ? __ldcg(p.topk_idx + i) : -1;
            const uint32_t m = __match_any_sync(0xFFFFFFFFu, e);
            const int rank = __popc(m & ((1u << lane) - 1u));
            const int base = (i < P) ? cursor[e] : 0;
            __syncwarp();
            if (i < P) {
                pairs[base + rank] = i;
                if (lane == __ffs(m) - 1) cursor[e] = base + __popc(m);
            }
            __syncwarp();
        }
    }
}

template <int KC>  // 16-byte bf16 chunks per lane per segment: segment = KC*256 columns
__global__ void __launch_bounds__(kRouterWarps * kWarp) router_topk_kernel(RouterParams p)
{
    extern __shared__ __align__(16) unsigned char smem[];
    __shared__ int s_last;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int row = blockIdx.x * kRouterWarps + warp;  // rows 0..E-1: router; row E: shared gate
    const bool active = row <= p.E;
    const uint16_t *wrow = (row < p.E) ? p.wr + (size_t)row * p.H : p.g;
    constexpr int kSeg = KC * 256;
    const int nseg = (p.H + kSeg - 1) / kSeg;

    // The router weights are layer constants: fetch them before waiting on
    // the kernel that produced x.
    uint4 w[KC];
#pragma unroll
    for (int c = 0; c < KC; ++c) {
        const int col = c * 256 + lane * 8;
        w[c] = (active && col < p.H) ? ld_stream_v4(wrow + col) : make_uint4(0, 0, 0, 0);
    }
    const float b = (active && row < p.E && p.bias) ? p.bias[row] : 0.f;
    pdl_wait();
    pdl_trigger();

    uint4 *xs = reinterpret_cast<uint4 *>(smem);
    const int hv = p.H / 8;
    for (int t0 = 0; t0 < p.rows; t0 += kRouterTok) {
        const int nt = min(kRouterTok, p.rows - t0);
        __syncthreads();
        const uint4 *xg = reinterpret_cast<const uint4 *>(p.x + (size_t)t0 * p.H);
        for (int i = threadIdx.x; i < nt * hv; i += blockDim.x) xs[i] = xg[i];
        __syncthreads();
        if (!active) continue;
        float acc[kRouterTok];
#pragma unroll
        for (int t = 0; t < kRouterTok; ++t) acc[t] = 0.f;
        for (int s = 0; s < nseg; ++s) {
            if (nseg > 1 && !(s == 0 && t0 == 0)) {
#pragma unroll
                for (int c = 0; c < KC; ++c) {
                    const int col = s * kSeg + c * 256 + lane * 8;
                    w[c] = (col < p.H) ? ld_stream_v4(wrow + col) : make_uint4(0, 0, 0, 0);
                }
            }
#pragma unroll
            for (int t = 0; t < kRouterTok; ++t) {
                if (t < nt) {
#pragma unroll
                    for (int c = 0; c < KC; ++c) {
                        const int col = s * kSeg + c * 256 + lane * 8;
                        if (col < p.H) acc[t] += dot8_bf16(w[c], xs[t * hv + col / 8]);
                    }
                }
            }
        }
#pragma unroll
        for (int t = 0; t < kRouterTok; ++t) {
            if (t < nt) {
                const float v = warp_sum(acc[t]);
                if (lane == 0) p.logits[(size_t)(t0 + t) * (p.E + 1) + row] = v + b;
            }
        }
    }

    // Last CTA to finish runs the top-k (no CTA waits for another).
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence();
        const int prev = atomicAdd(&p.counters[kCtrRouter], 1);
        s_last = (prev == (int)gridDim.x - 1);
    }
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    router_topk_rows(p);
    if (p.plan) {
        __syncthreads();
        int *cnt = reinterpret_cast<int *>(smem);
        router_build_plan(p, cnt, cnt + p.E);
    }
    __syncthreads();
    if (threadIdx.x == 0) p.counters[kCtrRouter] = 0;
}

// -------------------------------------------------------------- gate_up

constexpr int kGuWarps = 8;
constexpr int kGuPairsPerWarp = 2;
constexpr int kGuPairs = kGuWarps * kGuPairsPerWarp;  // row pairs per work item
constexpr int kGuTok = 8;                             // activation rows staged per pass

struct ExpertParams {
    const uint16_t *x;
    int rows, H, E, K, I, Is;
    const uint8_t *w8;
    const float *sc;
    const uint8_t *sw8;
    const float *ssc;
    const int32_t *plan;
    const float *topk_w;
    const float *gsig;
    float *h_routed;
    float *h_shared;
    float *yslot;
    const uint16_t *residual;
    uint16_t *out;
    int32_t *counters;
};

struct ItemView {
    const uint8_t *slab;   // expert slab (codes)
    const float *scales;   // expert scales
    const int32_t *pairs;  // routed pair ids, or nullptr for the shared expert
    int n;                 // rows routed to this expert
    int inter;             // I or Is
    int chunk;
};

__device__ __forceinline__ ItemView item_view(const ExpertParams &p, int item, int nch_r, int n_active)
{
    ItemView v;
    const int32_t *act_e = p.plan + 1;
    const int32_t *act_off = act_e + p.E;
    const int32_t *pairs = act_off + p.E + 1;
    if (item < n_active * nch_r) {
        const int u = item / nch_r;
        const int e = act_e[u];
        v.chunk = item - u * nch_r;
        v.inter = p.I;
        v.slab = p.w8 + (size_t)e * 3 * p.I * p.H;
        v.scales = p.sc + (size_t)e * ((2 * p.I / 128) * (p.H / 128) + (p.H / 128) * (p.I / 128));
        v.pairs = pairs + act_off[u];
        v.n = act_off[u + 1] - act_off[u];
    } else {
        v.chunk = item - n_active * nch_r;
        v.inter = p.Is;
        v.slab = p.sw8;
        v.scales = p.ssc;
        v.pairs = nullptr;
        v.n = p.rows;
    }
    return v;
}

// Shared-memory layout of a staged bf16 activation row: 16-byte units of
// the row are stored so that, for each 512-column chunk c and half j, lane L
// reads unit (c, j, L) at position c*64 + j*32 + L (conflict-free).
template <int KC>
__global__ void __launch_bounds__(kGuWarps * kWarp) gate_up_kernel(ExpertParams p)
{
    extern __shared__ __align__(16) unsigned char smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    pdl_wait();
    pdl_trigger();
    const int n_active = p.plan[0];
    const int nch_r = p.I / kGuPairs, nch_s = p.Is / kGuPairs;
    const int n_items = n_active * nch_r + nch_s;
    const int nck = (p.H + 511) / 512;   // 512-column chunks per row
    const int row_units = nck * 64;      // staged 16-byte units per row
    const int hb = p.H / 128;
    constexpr int kSeg = KC * 512;
    const int nseg = (p.H + kSeg - 1) / kSeg;
    uint4 *xs = reinterpret_cast<uint4 *>(smem);

    for (int item = blockIdx.x; item < n_items; item += gridDim.x) {
        const ItemView v = item_view(p, item, nch_r, n_active);
        const int Iu = v.inter;
        for (int tok0 = 0; tok0 < v.n; tok0 += kGuTok) {
            const int nt = min(kGuTok, v.n - tok0);
            __syncthreads();
            for (int i = threadIdx.x; i < nt * (p.H / 8); i += blockDim.x) {
                const int t = i / (p.H / 8), q = i - t * (p.H / 8);
                const int tok = v.pairs ? v.pairs[tok0 + t] / p.K : tok0 + t;
                const int c = q >> 6, r = q & 63;
                xs[t * row_units + c * 64 + (r & 1) * 32 + (r >> 1)] =
                    reinterpret_cast<const uint4 *>(p.x + (size_t)tok * p.H)[q];
            }
            __syncthreads();
#pragma unroll 1
            for (int qp = 0; qp < kGuPairsPerWarp; ++qp) {
                const int j = v.chunk * kGuPairs + qp * kGuWarps + warp;  // gate row j, up row Iu + j
                const uint8_t *rg = v.slab + (size_t)j * p.H;
                const uint8_t *ru = v.slab + (size_t)(Iu + j) * p.H;
                const float *sg = v.scales + (j / 128) * hb;
                const float *su = v.scales + ((Iu + j) / 128) * hb;
                float ag[kGuTok], au[kGuTok];
#pragma unroll
                for (int t = 0; t < kGuTok; ++t) ag[t] = au[t] = 0.f;
                for (int s = 0; s < nseg; ++s) {
                    uint4 wg[KC], wu[KC];
                    float cg[KC], cu[KC];
#pragma unroll
                    for (int c = 0; c < KC; ++c) {
                        const int col = s * kSeg + c * 512 + lane * 16;
                        const bool in = col < p.H;
                        wg[c] = in ? ld_stream_v4(rg + col) : make_uint4(0, 0, 0, 0);
                        wu[c] = in ? ld_stream_v4(ru + col) : make_uint4(0, 0, 0, 0);
                        cg[c] = in ? sg[col >> 7] : 0.f;
                        cu[c] = in ? su[col >> 7] : 0.f;
                    }
#pragma unroll
                    for (int t = 0; t < kGuTok; ++t) {
                        if (t < nt) {
#pragma unroll
                            for (int c = 0; c < KC; ++c) {
                                const int col = s * kSeg + c * 512 + lane * 16;
                                if (col < p.H) {
                                    const int cc = s * KC + c;
                                    const uint4 xa = xs[t * row_units + cc * 64 + lane];
                                    const uint4 xb = xs[t * row_units + cc * 64 + 32 + lane];
                                    ag[t] = fmaf(cg[c], dot16_e4m3_bf16(wg[c], xa, xb), ag[t]);
                                    au[t] = fmaf(cu[c], dot16_e4m3_bf16(wu[c], xa, xb), au[t]);
                                }
                            }
                        }
                    }
                }
#pragma unroll
                for (int t = 0; t < kGuTok; ++t) {
                    if (t < nt) {
                        const float g = warp_sum(ag[t]);
                        const float u = warp_sum(au[t]);
                        if (lane == 0) {
                            const float h = siluf_(g) * u;
                            if (v.pairs)
                                p.h_routed[(size_t)v.pairs[tok0 + t] * Iu + j] = h;
                            else
                                p.h_shared[(size_t)(tok0 + t) * Iu + j] = h;
                        }
                    }
                }
            }
        }
    }
}

// ------------------------------------------------------------ down+blend

constexpr int kDnWarps = 8;
constexpr int kDnRowsPerWarp = kDownRowsPerItem / kDnWarps;  // 4
constexpr int kDnSlots = 8;                                  // h rows staged per pass

// Staged fp32 h rows: float4 units, for 512-column chunk c and quarter j,
// lane L reads unit (c, j, L) at position c*128 + j*32 + L.
template <int KC>
__global__ void __launch_bounds__(kDnWarps * kWarp) down_blend_kernel(ExpertParams p)
{
    extern __shared__ __align__(16) unsigned char smem[];
    __shared__ int s_last;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    pdl_wait();
    pdl_trigger();
    const int n_active = p.plan[0];
    const int n_chunks = p.H / kDownRowsPerItem;
    const int n_items = (n_active + 1) * n_chunks;
    constexpr int kSeg = KC * 512;
    float4 *hs = reinterpret_cast<float4 *>(smem);

    for (int item = blockIdx.x; item < n_items; item += gridDim.x) {
        const int u = item / n_chunks;       // expert-major: neighbouring items stream neighbouring rows
        const int chunk = item - u * n_chunks;
        const ItemView v = item_view(p, u < n_active ? u : n_active, 1, n_active);
        const int Iu = v.inter;
        const int nck = (Iu + 511) / 512;
        const int row_units = nck * 128;
        const int ib = Iu / 128;
        const int nseg = (Iu + kSeg - 1) / kSeg;
        const float *hsrc = v.pairs ? p.h_routed : p.h_shared;
        for (int s0 = 0; s0 < v.n; s0 += kDnSlots) {
            const int ns = min(kDnSlots, v.n - s0);
            __syncthreads();
            for (int i = threadIdx.x; i < ns * (Iu / 4); i += blockDim.x) {
                const int sl = i / (Iu / 4), q = i - sl * (Iu / 4);
                const int slot = v.pairs ? v.pairs[s0 + sl] : s0 + sl;
                const int c = q >> 7, r = q & 127;
                hs[sl * row_units + c * 128 + (r & 3) * 32 + (r >> 2)] =
                    reinterpret_cast<const float4 *>(hsrc + (size_t)slot * Iu)[q];
            }
            __syncthreads();
#pragma unroll 1
            for (int rr = 0; rr < kDnRowsPerWarp; ++rr) {
                const int n = chunk * kDownRowsPerItem + warp * kDnRowsPerWarp + rr;
                const uint8_t *row = v.slab + (size_t)2 * Iu * p.H + (size_t)n * Iu;
                const float *sc = v.scales + (2 * Iu / 128) * (p.H / 128) + (n / 128) * ib;
                float acc[kDnSlots];
#pragma unroll
                for (int t = 0; t < kDnSlots; ++t) acc[t] = 0.f;
                for (int s = 0; s < nseg; ++s) {
                    uint4 w[KC];
                    float cs[KC];
#pragma unroll
                    for (int c = 0; c < KC; ++c) {
                        const int col = s * kSeg + c * 512 + lane * 16;
                        const bool in = col < Iu;
                        w[c] = in ? ld_stream_v4(row + col) : make_uint4(0, 0, 0, 0);
                        cs[c] = in ? sc[col >> 7] : 0.f;
                    }
#pragma unroll
                    for (int t = 0; t < kDnSlots; ++t) {
                        if (t < ns) {
#pragma unroll
                            for (int c = 0; c < KC; ++c) {
                                const int col = s * kSeg + c * 512 + lane * 16;
                                if (col < Iu) {
                                    const float4 *hr = hs + t * row_units + (s * KC + c) * 128 + lane;
                                    float a = 0.f, b = 0.f;
                                    fma4_e4m3_f32(w[c].x, hr[0], a, b);
                                    fma4_e4m3_f32(w[c].y, hr[32], a, b);
                                    fma4_e4m3_f32(w[c].z, hr[64], a, b);
                                    fma4_e4m3_f32(w[c].w, hr[96], a, b);
                                    acc[t] = fmaf(cs[c], a + b, acc[t]);
                                }
                            }
                        }
                    }
                }
#pragma unroll
                for (int t = 0; t < kDnSlots; ++t) {
                    if (t < ns) {
                        const float y = warp_sum(acc[t]);
                        if (lane == 0) {
                            int yrow;
                            float wt;
                            if (v.pairs) {
                                yrow = v.pairs[s0 + t];
                                wt = p.topk_w[yrow];
                            } else {
                                yrow = p.rows * p.K + s0 + t;
                                wt = p.gsig[s0 + t];
                            }
                            p.yslot[(size_t)yrow * p.H + n] = wt * y;
                        }
                    }
                }
            }
        }
        // The last item to finish this 32-row chunk blends it.
        __syncthreads();
        if (threadIdx.x == 0) {
            __threadfence();
            const int prev = atomicAdd(&p.counters[kCtrBlend + chunk], 1);
            s_last = (prev == n_active);  // n_active routed items + 1 shared item per chunk
        }
        __syncthreads();
        if (s_last) {
            __threadfence();
            const int n0 = chunk * kDownRowsPerItem;
            for (int i = threadIdx.x; i < p.rows * kDownRowsPerItem; i += blockDim.x) {
                const int t = i / kDownRowsPerItem;
                const int n = n0 + (i - t * kDownRowsPerItem);
                float acc = 0.f;
                for (int r = 0; r < p.K; ++r) acc += __ldcg(p.yslot + (size_t)(t * p.K + r) * p.H + n);
                acc += __ldcg(p.yslot + (size_t)(p.rows * p.K + t) * p.H + n);
                if (p.residual) acc += bf16_bits_to_f32(p.residual[(size_t)t * p.H + n]);
                p.out[(size_t)t * p.H + n] = f32_to_bf16_bits(acc);
            }
            if (threadIdx.x == 0) p.counters[kCtrBlend + chunk] = 0;
        }
    }
}

// ------------------------------------------------------------- launchers

namespace {

template <typename P>
cudaError_t launch_ex(void (*kernel)(P), int grid, int block, size_t smem, cudaStream_t s, const P &p)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(block);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, p);
}

int pick_kc(int cols_per_chunk, int n)  // smallest of 1,2,4,8 chunks covering n columns, else 8
{
    const int need = (n + cols_per_chunk - 1) / cols_per_chunk;
    if (need <= 1) return 1;
    if (need <= 2) return 2;
    if (need <= 4) return 4;
    return 8;
}

struct KernelSlot {
    int device = -1;  // device the entry was measured on
    int blocks_per_sm = 1;
};

std::mutex g_mu;

template <typename P>
int occupancy(void (*kernel)(P), int block, size_t smem, KernelSlot &slot)
{
    int dev = 0;
    cudaGetDevice(&dev);
    std::lock_guard<std::mutex> lk(g_mu);
    if (slot.device != dev) {
        if (smem > 48 * 1024) cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        int b = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&b, kernel, block, smem) != cudaSuccess || b < 1) b = 1;
        slot.blocks_per_sm = b;
        slot.device = dev;
    }
    return slot.blocks_per_sm;
}

}  // namespace

cudaError_t launch_router_topk(const RouterLaunch &a, cudaStream_t s)
{
    const moe_dims &d = *a.d;
    RouterParams p;
    p.x = a.x;
    p.rows = a.rows;
    p.H = d.hidden;
    p.E = d.n_experts;
    p.K = d.top_k;
    p.wr = a.router_w;
    p.bias = a.router_bias;
    p.g = a.shared_gate;
    p.logits = a.logits;
    p.topk_idx = a.topk_idx;
    p.topk_w = a.topk_w;
    p.gsig = a.gsig;
    p.counters = a.counters;
    p.plan = a.plan;
    const int grid = (d.n_experts + 1 + kRouterWarps - 1) / kRouterWarps;
    const size_t xs = (size_t)kRouterTok * d.hidden * 2;
    const size_t plan_smem = a.plan ? (size_t)2 * d.n_experts * sizeof(int) : 0;
    const size_t smem = xs > plan_smem ? xs : plan_smem;
    const int need = (d.hidden + 255) / 256;
    void (*k)(RouterParams);
    if (need <= 2) k = router_topk_kernel<2>;
    else if (need <= 4) k = router_topk_kernel<4>;
    else if (need <= 8) k = router_topk_kernel<8>;
    else k = router_topk_kernel<16>;
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    return launch_ex(k, grid, kRouterWarps * kWarp, smem, s, p);
}

static KernelSlot g_gu_slots[9], g_dn_slots[9];

cudaError_t launch_decode_experts(const ExpertsLaunch &a, cudaStream_t s)
{
    const moe_dims &d = *a.d;
    const DeviceInfo &di = device_info();
    ExpertParams p;
    p.x = a.x;
    p.rows = a.rows;
    p.H = d.hidden;
    p.E = d.n_experts;
    p.K = d.top_k;
    p.I = d.inter;
    p.Is = d.shared_inter;
    p.w8 = a.expert_w8;
    p.sc = a.expert_scales;
    p.sw8 = a.shared_w8;
    p.ssc = a.shared_scales;
    p.plan = a.plan;
    p.topk_w = a.topk_w;
    p.gsig = a.gsig;
    p.h_routed = a.h_routed;
    p.h_shared = a.h_shared;
    p.yslot = a.yslot;
    p.residual = a.residual;
    p.out = a.out;
    p.counters = a.counters;

    const int64_t max_active = std::min<int64_t>(d.n_experts, (int64_t)a.rows * d.top_k);

    // gate_up
    {
        const int kc = pick_kc(512, d.hidden);
        void (*k)(ExpertParams) = kc == 1 ? gate_up_kernel<1> : kc == 2 ? gate_up_kernel<2>
                                : kc == 4 ? gate_up_kernel<4> : gate_up_kernel<8>;
        const size_t smem = (size_t)kGuTok * ((d.hidden + 511) / 512) * 64 * 16;
        const int bps = occupancy(k, kGuWarps * kWarp, smem, g_gu_slots[kc]);
        const int64_t items = max_active * (d.inter / kGuPairs) + d.shared_inter / kGuPairs;
        const int grid = (int)std::min<int64_t>(items, (int64_t)bps * di.sm_count);
        cudaError_t e = launch_ex(k, grid, kGuWarps * kWarp, smem, s, p);
        if (e != cudaSuccess) return e;
    }
    // down + blend
    {
        const int imax = d.inter > d.shared_inter ? d.inter : d.shared_inter;
        const int kc = pick_kc(512, imax);
        void (*k)(ExpertParams) = kc == 1 ? down_blend_kernel<1> : kc == 2 ? down_blend_kernel<2>
                                : kc == 4 ? down_blend_kernel<4> : down_blend_kernel<8>;
        const size_t smem = (size_t)kDnSlots * ((imax + 511) / 512) * 128 * 16;
        const int bps = occupancy(k, kDnWarps * kWarp, smem, g_dn_slots[kc]);
        const int64_t items = (max_active + 1) * (d.hidden / kDownRowsPerItem);
        const int grid = (int)std::min<int64_t>(items, (int64_t)bps * di.sm_count);
        cudaError_t e = launch_ex(k, grid, kDnWarps * kWarp, smem, s, p);
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace moe
