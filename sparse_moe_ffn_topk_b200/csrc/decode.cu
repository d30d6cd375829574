// decode.cu -- decode path (rows <= a few dozen): weight-streaming GEMVs.
//
// Three launches chained with programmatic dependent launch (PDL):
//   1. router_topk_kernel: bf16 router GEMV + shared-gate dot.  Each CTA
//      bulk-copies its slice of router rows into shared memory before it
//      waits on the kernel that produced x, one warp per router row; the row
//      block 0 CTA also writes x as hi/lo e4m3 rows; the last CTA of each
//      token group runs the group's top-k softmax.
//   2. gate_up_kernel: every CTA first builds the per-expert routing table
//      (expert dedup across rows) in its shared memory from the top-k.
//      Persistent CTAs then walk (expert, block of gate/up row pairs) items
//      through a ring of shared-memory stages filled by bulk copies;
//      shared-expert items come first and are fetched before the PDL wait,
//      since they do not depend on routing.  The e4m3 weight bytes feed
//      mma.m16n8k32 directly, block scales are applied per 128-wide K block
//      in registers, h = silu(gate) * up is kept in fp32.
//   3. The down product and blend, one of two kernels:
//      down_small_kernel (few rows): a CTA item is 16 output rows of every
//      active expert and the shared expert (W2 tiles by TMA), so each output
//      row is complete in one CTA and written straight to out;
//      down_blend_kernel (otherwise): (expert, block of down rows) items
//      through the same kind of ring as gate_up; one partial per routed slot
//      scaled by its routing weight (or the shared gate); the last item to
//      finish a row block blends the k partials in rank order plus the
//      shared partial (plus the residual) and rounds once to bf16.
//      Both use one arithmetic, so their results are identical bits.
//
// Prior art on the pages: the GB10 blueprint's per-layer MoE chain (router
// GEMV, top-k softmax, gate_up with the shared expert fused, silu+down,
// weighted blend; fp8/block128x128 weights read against bf16 and f32
// activations) and the colibri PR's decode GEMV (one warp per output row, 16
// bytes a lane, the activation in shared memory).  Here the weight bytes
// reach shared memory by bulk DMA instead of through registers, so the bytes
// in flight per SM are bounded by shared memory, not by registers.
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

namespace moe {

// ------------------------------------------------------------------ helpers

// 8 e4m3 codes (two words) against 8 bf16 activations (16 bytes).
__device__ __forceinline__ float dot8_e4m3_bf16(uint2 w, uint4 x)
{
    float2 f0 = e4m3x2_to_f32x2(static_cast<uint16_t>(w.x & 0xFFFFu));
    float2 f1 = e4m3x2_to_f32x2(static_cast<uint16_t>(w.x >> 16));
    float2 f2 = e4m3x2_to_f32x2(static_cast<uint16_t>(w.y & 0xFFFFu));
    float2 f3 = e4m3x2_to_f32x2(static_cast<uint16_t>(w.y >> 16));
    float a = f0.x * bf16_lo(x.x);
    float b = f0.y * bf16_hi(x.x);
    a = fmaf(f1.x, bf16_lo(x.y), a);
    b = fmaf(f1.y, bf16_hi(x.y), b);
    a = fmaf(f2.x, bf16_lo(x.z), a);
    b = fmaf(f2.y, bf16_hi(x.z), b);
    a = fmaf(f3.x, bf16_lo(x.w), a);
    b = fmaf(f3.y, bf16_hi(x.w), b);
    return a + b;
}

// 4 e4m3 codes (one word) against 4 fp32 values.
__device__ __forceinline__ float dot4_e4m3_f32(uint32_t w, float4 h)
{
    float2 f0 = e4m3x2_to_f32x2(static_cast<uint16_t>(w & 0xFFFFu));
    float2 f1 = e4m3x2_to_f32x2(static_cast<uint16_t>(w >> 16));
    float a = f0.x * h.x;
    float b = f0.y * h.y;
    a = fmaf(f1.x, h.z, a);
    b = fmaf(f1.y, h.w, b);
    return a + b;
}

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
    uint8_t *xq;       // x as hi/lo e4m3 rows [rows][2H] for the expert kernels
    float *xsc;        // their scales [rows][H/128]
    int32_t *topk_idx;
    float *topk_w;
    float *gsig;
    int32_t *counters;
};

__device__ __forceinline__ int atomic_add_acq_rel_gpu(int32_t *p, int v)
{
    int old;
    asm volatile("atom.acq_rel.gpu.global.add.s32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
    return old;
}

// Top-k of one row (one warp) on order-preserving keys.  Lane L holds the
// EPL experts L*EPL .. L*EPL+EPL-1, sorted once by descending key (a stable
// sort, so equal keys keep the lower expert first).  Each round takes the
// best head across the warp; equal heads go to the lower lane, whose
// experts all have lower indices, and the winning lane pops its head.  Key 0
// marks an absent expert and a NaN logit gets key 1, so every round picks a
// valid expert even on non-finite input.
template <int EPL>
__device__ void topk_select(const float *lrow, int E, int K, int32_t *out_idx, float *out_w, float *out_gsig)
{
    const int lane = threadIdx.x & 31;
    uint32_t v[EPL];
    int id[EPL];
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
        const int e = lane * EPL + i;
        const float l = (e < E) ? __ldcg(lrow + e) : 0.f;
        v[i] = (e < E) ? topk_key(l) : 0u;
        id[i] = e;
    }
    const float z = __ldcg(lrow + E);
    // odd-even transposition sort, descending; swaps only on a strict
    // inequality, so it is stable
#pragma unroll
    for (int pass = 0; pass < EPL; ++pass) {
#pragma unroll
        for (int j = pass & 1; j + 1 < EPL; j += 2) {
            if (v[j] < v[j + 1]) {
                const uint32_t tv = v[j];
                v[j] = v[j + 1];
                v[j + 1] = tv;
                const int ti = id[j];
                id[j] = id[j + 1];
                id[j + 1] = ti;
            }
        }
    }
    int my_e = 0;
    uint32_t my_k = 0;
    for (int r = 0; r < K; ++r) {
        const uint32_t kmax = __reduce_max_sync(0xFFFFFFFFu, v[0]);
        const int wl = __ffs(__ballot_sync(0xFFFFFFFFu, v[0] == kmax)) - 1;
        const int ew = __shfl_sync(0xFFFFFFFFu, id[0], wl);
        if (lane == wl) {
#pragma unroll
            for (int j = 0; j + 1 < EPL; ++j) {
                v[j] = v[j + 1];
                id[j] = id[j + 1];
            }
            v[EPL - 1] = 0u;
        }
        if (lane == r) {
            my_e = ew;
            my_k = kmax;
        }
    }
    if (threadIdx.x == 0) MOE_TRACE(0, 5);
    const float my_v = (my_k == 1u) ? __int_as_float(0x7FC00000) : key_value(my_k);
    const float top = __shfl_sync(0xFFFFFFFFu, my_v, 0);
    const float ev = (lane < K) ? expf(my_v - top) : 0.f;
    const float sum = warp_sum(ev);
    if (lane < K) {
        out_idx[lane] = my_e;
        out_w[lane] = ev / sum;
    }
    if (lane == 0) *out_gsig = sigmoidf_(z);
    if (threadIdx.x == 0) MOE_TRACE(0, 6);
}

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
        if (blockIdx.x == 0 && p.xq) {
            // the expert kernels' activation format: hi/lo e4m3, one scale per (row, 128 block)
            const int hb = p.H / 128;
            for (int u = warp; u < nt * hb; u += blockDim.x >> 5) {
                const int t = u / hb, kb = u - t * hb;
                const uint2 raw = reinterpret_cast<const uint2 *>(xs + (size_t)t * rowb)[kb * 32 + lane];
                const float4 v = make_float4(bf16_lo(raw.x), bf16_hi(raw.x), bf16_lo(raw.y), bf16_hi(raw.y));
                const float amax = warp_max(fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w))));
                const float sc = amax > 0.f ? amax / 448.f : 1.f;
                uint32_t hi, lo;
                quant4_hilo(v, 1.f / sc, hi, lo);
                uint32_t *dst = reinterpret_cast<uint32_t *>(p.xq + (size_t)(t0 + t) * 2 * p.H);
                dst[kb * 32 + lane] = hi;
                dst[p.H / 4 + kb * 32 + lane] = lo;
                if (lane == 0) p.xsc[(size_t)(t0 + t) * hb + kb] = sc;
            }
        }
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

// ------------------------------------------------------- expert kernels

struct ExpertParams {
    const uint16_t *x;
    const uint8_t *xq;  // activations as hi/lo e4m3: [rows][hi: H | lo: H]
    const float *xsc;   // their scales: [rows][H/128]
    int rows, H, E, K, I, Is;
    const uint8_t *w8;
    const float *sc;
    const uint8_t *sw8;
    const float *ssc;
    const int32_t *topk_idx;
    const float *topk_w;
    const float *gsig;
    float *h_routed;
    float *h_shared;
    float *yslot;
    const uint16_t *residual;
    uint16_t *out;
    int32_t *counters;
    int pairs;   // gate_up: gate/up row pairs per item (a multiple of 8, <= 32)
    int drows;   // down: rows per item (a multiple of 16, <= 64)
    int tok;     // activation / h rows staged with an item (<= kDescPairs)
    int stages;  // ring depth
    int ue;      // down by output block: experts per stage
    int l2_w2;   // gate_up: prefetch the active experts' down weights into L2
};

// What a stage holds; written by the producer before the stage's "full"
// arrival, read by the consumers after the phase completes.
struct StageDesc {
    const uint8_t *slab;
    const float *scales;
    const int32_t *pairs;  // all pair ids of the expert, or nullptr for the shared expert
    int n;                 // rows routed to the expert
    int inter;             // I or Is
    int first;             // first gate/up pair (gate_up) or first down row (down)
    int rows[kDescPairs];  // pair ids (routed) or token rows (shared) staged with the item
    float wt[kDescPairs];  // down: routing weight (or shared gate) of each staged slot
};

__device__ __forceinline__ int expert_nscales(int H, int I)
{
    return (2 * I / 128) * (H / 128) + (H / 128) * (I / 128);
}

// The routing table of one expert CTA, built in its shared memory from
// topk_idx: the active experts in ascending id, where each one's pairs
// start in the pair list, and the pair ids (t*K + r) grouped by expert.
// Every CTA builds the same table (the order of pairs within an expert may
// differ between CTAs; each pair is computed on its own, so it does not
// matter).
struct LocalPlan {
    int *cnt;       // [E] counts, then fill cursors
    int *e_of;      // [min(E, P)] active expert ids
    int *first_of;  // [min(E, P) + 1] each active expert's first pair slot
    int *pairs;     // [P]
    int *scratch;   // [kWarp + 1] scan scratch
};

__host__ __device__ __forceinline__ size_t plan_bytes(int E, int P)
{
    const int U = E < P ? E : P;
    return align16(sizeof(int) * ((size_t)E + U + (U + 1) + P + (kWarp + 1)));
}

__device__ __forceinline__ LocalPlan plan_at(unsigned char *base, int E, int P)
{
    const int U = min(E, P);
    LocalPlan lp;
    lp.cnt = reinterpret_cast<int *>(base);
    lp.e_of = lp.cnt + E;
    lp.first_of = lp.e_of + U;
    lp.pairs = lp.first_of + U + 1;
    lp.scratch = lp.pairs + P;
    return lp;
}

// All threads of the CTA.  Returns the number of active routed experts (0
// if an earlier kernel of this call recorded an error: its outputs are not
// valid).
__device__ int build_local_plan(const ExpertParams &p, const LocalPlan &lp)
{
    const int E = p.E, P = p.rows * p.K;
    auto expert_of = [&](int i) { return __ldcg(p.topk_idx + i); };
    for (int e = threadIdx.x; e < E; e += blockDim.x) lp.cnt[e] = 0;
    __syncthreads();
    for (int i = threadIdx.x; i < P; i += blockDim.x)
        atomicAdd(&lp.cnt[min(max(expert_of(i), 0), E - 1)], 1);
    __syncthreads();
    int run_off = 0, run_act = 0;
    for (int e0 = 0; e0 < E; e0 += blockDim.x) {
        const int e = e0 + threadIdx.x;
        const int c = (e < E) ? lp.cnt[e] : 0;
        int tot_off, tot_act;
        const int off = block_exclusive_scan(c, lp.scratch, &tot_off);
        const int act = block_exclusive_scan(c > 0 ? 1 : 0, lp.scratch, &tot_act);
        if (c > 0) {
            lp.e_of[run_act + act] = e;
            lp.first_of[run_act + act] = run_off + off;
            lp.cnt[e] = run_off + off;
        }
        run_off += tot_off;
        run_act += tot_act;
    }
    if (threadIdx.x == 0) lp.first_of[run_act] = run_off;
    __syncthreads();
    for (int i = threadIdx.x; i < P; i += blockDim.x) {
        const int e = min(max(expert_of(i), 0), E - 1);
        lp.pairs[atomicAdd(&lp.cnt[e], 1)] = i;
    }
    const int bad = __ldcg(p.counters + kCtrStatus);
    __syncthreads();
    return bad ? 0 : run_act;
}

// Item i: shared-expert items first (routing-independent), then the routed
// experts in table order.
__device__ __forceinline__ void describe(const ExpertParams &p, int item, int per_shared, int per_routed,
                                         int block, const LocalPlan *lp, StageDesc &d)
{
    if (item < per_shared) {
        d.slab = p.sw8;
        d.scales = p.ssc;
        d.pairs = nullptr;
        d.n = p.rows;
        d.inter = p.Is;
        d.first = item * block;
#pragma unroll
        for (int i = 0; i < kDescPairs; ++i) d.rows[i] = i;
    } else {
        const int r = item - per_shared;
        const int u = r / per_routed;
        const int e = lp->e_of[u], f0 = lp->first_of[u];
        d.slab = p.w8 + (size_t)e * 3 * p.I * p.H;
        d.scales = p.sc + (size_t)e * expert_nscales(p.H, p.I);
        d.pairs = lp->pairs + f0;
        d.n = lp->first_of[u + 1] - f0;
        d.inter = p.I;
        d.first = (r - u * per_routed) * block;
#pragma unroll
        for (int i = 0; i < kDescPairs; ++i) d.rows[i] = i < d.n ? d.pairs[i] : 0;
    }
}

// Warp roles of the expert kernels: warps 0..7 compute (consumers), warp 8
// is the producer.  Each stage has a "full" mbarrier (one producer arrival
// plus the bulk-copy bytes) and an "empty" mbarrier (one arrival per
// consumer warp).  The producer runs up to `stages` items ahead: it fetches
// an item's descriptor, issues the bulk copies of its weight rows (one per
// row, into rows padded by 16 bytes so that the tensor-core fragment loads
// hit distinct banks) and activations, loads the block scales into the
// stage and arrives.
//
// The consumers feed the e4m3 weights straight into mma.m16n8k32 as the A
// operand and the hi/lo e4m3 activations as B (up to 8 rows in the 8
// columns).  Within each 32-wide K chunk, lane t of a quad reads the 8
// bytes [8t, 8t+8) of its two rows and of its activation column; the first
// four bytes play the fragment's k = 4t..4t+3 and the next four k =
// 16+4t..19+4t, for A and B alike, so the products pair up the same
// columns.  Each 128-wide K block is summed by the tensor cores, then scaled
// by its weight and activation block scales into fp32 registers; the K
// blocks are spread over the warps and reduced through shared memory.
constexpr int kConsumerWarps = 8;
constexpr int kExpThreads = (kConsumerWarps + 1) * kWarp;
constexpr int kConsumerThreads = kConsumerWarps * kWarp;
constexpr int kMaxStages = 4;
constexpr int kRowPad = 16;   // bytes of padding after each staged row
// Cross-warp reduction area of an item with T 16-row MMA tiles.
__host__ __device__ constexpr size_t red_bytes(int T) { return (size_t)kConsumerWarps * T * kWarp * 16; }

// ------------------------------------------------------------- gate_up

// Stage layout (WS = H + 16): [16*T weight rows: tile tau's rows 0..7 are
// gate rows first+8tau.., rows 8..15 the matching up rows][tok x-hi rows]
// [tok x-lo rows][x scales: tok * H/128][gate scales: H/128][up scales: H/128]
struct GuLayout {
    int WS, T, hb;
    size_t xh, xl, xs, sw, bytes;
};
__device__ __forceinline__ GuLayout gu_layout(const ExpertParams &p)
{
    GuLayout L;
    L.WS = p.H + kRowPad;
    L.T = p.pairs / 8;
    L.hb = p.H / 128;
    L.xh = (size_t)16 * L.T * L.WS;
    L.xl = L.xh + (size_t)p.tok * L.WS;
    L.xs = L.xl + (size_t)p.tok * L.WS;
    L.sw = L.xs + (size_t)p.tok * L.hb * 4;
    L.bytes = align16(L.sw + (size_t)2 * L.hb * 4);
    return L;
}

// Producer warp, all lanes: weights (and/or activations) of a stage.
__device__ void gu_produce(const ExpertParams &p, const GuLayout &L, const StageDesc &d, unsigned char *st,
                           uint64_t *bar, uint64_t pol, bool weights, bool acts)
{
    const int lane = threadIdx.x & 31;
    const int nt = min(p.tok, d.n);
    // Scale rows (H/128 floats) travel by bulk copy on the stage's barrier
    // when they are whole 16-byte units; otherwise the lanes store them.
    const uint32_t scb = (uint32_t)L.hb * 4;
    const bool bsc = (scb % 16) == 0 && (smem_u32(st + L.sw) & 15) == 0 && (smem_u32(st + L.xs) & 15) == 0;
    if (lane == 0) {
        uint32_t bytes = 0;
        if (weights) bytes += (uint32_t)(16 * L.T * p.H) + (bsc ? 2 * scb : 0);
        if (acts) bytes += (uint32_t)(2 * nt * p.H) + (bsc ? nt * scb : 0);
        mbar_expect_tx(bar, bytes);
    }
    __syncwarp();
    if (weights) {
        for (int i = lane; i < 16 * L.T; i += kWarp) {
            const int tau = i >> 4, r = i & 15;
            const int src = r < 8 ? d.first + 8 * tau + r : d.inter + d.first + 8 * tau + r - 8;
            bulk_g2s_stream(st + (size_t)i * L.WS, d.slab + (size_t)src * p.H, (uint32_t)p.H, bar, pol);
        }
        float *sw = reinterpret_cast<float *>(st + L.sw);
        const float *sg = d.scales + (d.first / 128) * L.hb;
        const float *su = d.scales + ((d.inter + d.first) / 128) * L.hb;
        if (bsc) {
            if (lane == 0) bulk_g2s(sw, sg, scb, bar);
            if (lane == 1) bulk_g2s(sw + L.hb, su, scb, bar);
        } else {
            for (int i = lane; i < 2 * L.hb; i += kWarp) sw[i] = (i < L.hb) ? __ldg(sg + i) : __ldg(su + i - L.hb);
        }
    }
    if (acts) {
        for (int i = lane; i < 2 * nt; i += kWarp) {
            const int t = i >> 1, lo = i & 1;
            const int row = d.pairs ? d.rows[t] / p.K : d.rows[t];
            bulk_g2s(st + (lo ? L.xl : L.xh) + (size_t)t * L.WS, p.xq + (size_t)row * 2 * p.H + (size_t)lo * p.H,
                     (uint32_t)p.H, bar);
        }
        float *xs = reinterpret_cast<float *>(st + L.xs);
        if (bsc) {
            for (int t = lane; t < nt; t += kWarp) {
                const int row = d.pairs ? d.rows[t] / p.K : d.rows[t];
                bulk_g2s(xs + t * L.hb, p.xsc + (size_t)row * L.hb, scb, bar);
            }
        } else {
            for (int i = lane; i < nt * L.hb; i += kWarp) {
                const int t = i / L.hb;
                const int row = d.pairs ? d.rows[t] / p.K : d.rows[t];
                xs[i] = __ldcg(p.xsc + (size_t)row * L.hb + (i - t * L.hb));
            }
        }
    }
}

// Warm L2 with the down weights of the active experts and of the shared
// expert, 64 KB pieces spread over the CTAs (piece i goes to CTA i mod grid):
// the down kernel then reads them from L2 instead of waiting on HBM.
__device__ void prefetch_down_weights(const ExpertParams &p, const LocalPlan &lp, int n_active)
{
    const int lane = threadIdx.x & 31;
    const size_t piece = 65536, per = (size_t)p.I * p.H, per_s = (size_t)p.Is * p.H;
    const size_t pieces_r = (per + piece - 1) / piece, pieces_s = (per_s + piece - 1) / piece;
    const size_t total = (size_t)n_active * pieces_r + pieces_s;
    for (size_t i = blockIdx.x + (size_t)lane * gridDim.x; i < total; i += (size_t)gridDim.x * kWarp) {
        const uint8_t *base;
        size_t off, len;
        if (i < (size_t)n_active * pieces_r) {
            const size_t u = i / pieces_r;
            off = (i - u * pieces_r) * piece;
            len = per;
            base = p.w8 + (size_t)lp.e_of[u] * 3 * p.I * p.H + (size_t)2 * p.I * p.H;
        } else {
            off = (i - (size_t)n_active * pieces_r) * piece;
            len = per_s;
            base = p.sw8 + (size_t)2 * p.Is * p.H;
        }
        prefetch_l2(base + off, (uint32_t)(len - off < piece ? len - off : piece));
    }
}

// gate_up, producer warp: the weights of the first stages' shared-expert
// items, which do not depend on routing (fetched before the routing exists).
__device__ void gu_prefetch_shared(const ExpertParams &p, unsigned char *smem, uint64_t *full, StageDesc *desc)
{
    const int lane = threadIdx.x & 31;
    const GuLayout L = gu_layout(p);
    const int per_shared = p.Is / p.pairs, per_routed = p.I / p.pairs;
    const uint64_t pol = policy_evict_first();
    for (int q = 0; q < p.stages; ++q) {
        const int item = blockIdx.x + q * gridDim.x;
        if (item >= per_shared) break;
        if (lane == 0) describe(p, item, per_shared, per_routed, p.pairs, nullptr, desc[q]);
        __syncwarp();
        gu_produce(p, L, desc[q], smem + q * L.bytes, &full[q], pol, true, false);
    }
    __syncwarp();
}

// gate_up's item loops, once the routing table lp (n_active routed experts)
// exists: the producer warp fills the stage ring, the consumer warps compute
// h into HBM.  Every thread of the CTA calls this; it returns when the
// thread's role is done.
template <int T>
__device__ void gu_items(const ExpertParams &p, unsigned char *smem, uint64_t *full, uint64_t *empty, StageDesc *desc,
                         volatile int &s_abort, const LocalPlan &lp, int n_active)
{
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const GuLayout L = gu_layout(p);
    const int per_shared = p.Is / p.pairs, per_routed = p.I / p.pairs;
    const int S = p.stages;
    float4 *red = reinterpret_cast<float4 *>(smem + (size_t)S * L.bytes);  // [warp][tile][lane]
    const uint64_t pol = policy_evict_first();
    const int n_items = per_shared + n_active * per_routed;
    if (warp == kConsumerWarps) {
        // ------------------------------------------------------- producer
        for (int q = 0;; ++q) {
            const int item = blockIdx.x + q * gridDim.x;
            if (item >= n_items) break;
            const int s = q % S;
            if (q >= S && !mbar_wait(&empty[s], ((q / S) - 1) & 1, kWaitLimitNs)) {
                if (lane == 0) set_status(p.counters, MOE_ETIMEOUT);
                s_abort = 1;
                break;
            }
            unsigned char *st = smem + s * L.bytes;
            const bool prefetched = q < S && item < per_shared;
            if (lane == 0) {
                if (q >= S) fence_proxy_async_smem();  // consumers' generic accesses precede the copies
                if (!prefetched) describe(p, item, per_shared, per_routed, p.pairs, &lp, desc[s]);
            }
            __syncwarp();
            gu_produce(p, L, desc[s], st, &full[s], pol, !prefetched, true);
            __syncwarp();
            if (lane == 0) mbar_arrive(&full[s]);
            if (q == S - 1 && p.l2_w2) prefetch_down_weights(p, lp, n_active);  // after this CTA's first stages
        }
        if (p.l2_w2 && n_items <= (int)blockIdx.x + (S - 1) * (int)gridDim.x) prefetch_down_weights(p, lp, n_active);
        return;
    }

    // ----------------------------------------------------------- consumers
    const int g = lane >> 2, t = lane & 3;
    for (int q = 0;; ++q) {
        const int item = blockIdx.x + q * gridDim.x;
        if (item >= n_items) break;
        const int s = q % S;
        unsigned char *st = smem + s * L.bytes;
        if (!s_abort && !mbar_wait(&full[s], (q / S) & 1, kWaitLimitNs)) {
            if (lane == 0) set_status(p.counters, MOE_ETIMEOUT);
            s_abort = 1;
        }
        named_barrier(1, kConsumerThreads);  // every consumer warp sees the same abort flag
        if (q < 2 && threadIdx.x == 0) MOE_TRACE(1, 2 + 2 * q);
        const bool skip = s_abort;  // keep the loop (and its barriers) uniform after a timeout
        const StageDesc &d = desc[s];  // read in place; the producer rewrites it only after "empty"
        const int Iu = d.inter;
        const float *xsc = reinterpret_cast<const float *>(st + L.xs);
        const float *swg = reinterpret_cast<const float *>(st + L.sw);
        for (int tok0 = 0; tok0 < (skip ? 0 : d.n); tok0 += p.tok) {
            const int nt = min(p.tok, d.n - tok0);
            if (tok0 > 0) {  // more rows than a stage holds: restage the next ones in place
                named_barrier(1, kConsumerThreads);
                const int hv = p.H / 16;
                for (int i = threadIdx.x; i < 2 * nt * hv; i += kConsumerThreads) {
                    const int tr = i / (2 * hv), rem = i - tr * 2 * hv, lo = rem / hv, c = rem - lo * hv;
                    const int row = d.pairs ? d.pairs[tok0 + tr] / p.K : tok0 + tr;
                    reinterpret_cast<uint4 *>(st + (lo ? L.xl : L.xh) + (size_t)tr * L.WS)[c] =
                        __ldcg(reinterpret_cast<const uint4 *>(p.xq + (size_t)row * 2 * p.H + (size_t)lo * p.H) + c);
                }
                for (int i = threadIdx.x; i < nt * L.hb; i += kConsumerThreads) {
                    const int tr = i / L.hb;
                    const int row = d.pairs ? d.pairs[tok0 + tr] / p.K : tok0 + tr;
                    const_cast<float *>(xsc)[i] = __ldcg(p.xsc + (size_t)row * L.hb + (i - tr * L.hb));
                }
                named_barrier(1, kConsumerThreads);
            }
            float acc[T][4];
#pragma unroll
            for (int tau = 0; tau < T; ++tau) acc[tau][0] = acc[tau][1] = acc[tau][2] = acc[tau][3] = 0.f;
            const bool col_ok = g < nt;
            for (int kb = warp; kb < L.hb; kb += kConsumerWarps) {
                // all fragments of the K block first, then the MMAs: hi and lo
                // products on separate accumulator chains
                uint2 bh[4], bl[4], ra[T][4], rb[T][4];
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const int k0 = kb * 128 + c * 32 + 8 * t;
                    bh[c] = bl[c] = make_uint2(0, 0);
                    if (col_ok) {
                        bh[c] = *reinterpret_cast<const uint2 *>(st + L.xh + (size_t)g * L.WS + k0);
                        bl[c] = *reinterpret_cast<const uint2 *>(st + L.xl + (size_t)g * L.WS + k0);
                    }
#pragma unroll
                    for (int tau = 0; tau < T; ++tau) {
                        ra[tau][c] = *reinterpret_cast<const uint2 *>(st + (size_t)(16 * tau + g) * L.WS + k0);
                        rb[tau][c] = *reinterpret_cast<const uint2 *>(st + (size_t)(16 * tau + g + 8) * L.WS + k0);
                    }
                }
                float th[T][4], tl[T][4];
#pragma unroll
                for (int tau = 0; tau < T; ++tau)
#pragma unroll
                    for (int i = 0; i < 4; ++i) th[tau][i] = tl[tau][i] = 0.f;
#pragma unroll
                for (int c = 0; c < 4; ++c)
#pragma unroll
                    for (int tau = 0; tau < T; ++tau) {
                        mma_e4m3_16832(th[tau], ra[tau][c].x, rb[tau][c].x, ra[tau][c].y, rb[tau][c].y, bh[c].x, bh[c].y);
                        mma_e4m3_16832(tl[tau], ra[tau][c].x, rb[tau][c].x, ra[tau][c].y, rb[tau][c].y, bl[c].x, bl[c].y);
                    }
                const float sg = swg[kb], su = swg[L.hb + kb];
                const float x0 = (2 * t < nt) ? xsc[(2 * t) * L.hb + kb] : 0.f;
                const float x1 = (2 * t + 1 < nt) ? xsc[(2 * t + 1) * L.hb + kb] : 0.f;
#pragma unroll
                for (int tau = 0; tau < T; ++tau) {
                    acc[tau][0] = fmaf(sg * x0, th[tau][0] + tl[tau][0], acc[tau][0]);
                    acc[tau][1] = fmaf(sg * x1, th[tau][1] + tl[tau][1], acc[tau][1]);
                    acc[tau][2] = fmaf(su * x0, th[tau][2] + tl[tau][2], acc[tau][2]);
                    acc[tau][3] = fmaf(su * x1, th[tau][3] + tl[tau][3], acc[tau][3]);
                }
            }
            if (q == 0 && threadIdx.x == 0) MOE_TRACE(1, 7);
#pragma unroll
            for (int tau = 0; tau < T; ++tau)
                red[(warp * T + tau) * kWarp + lane] = make_float4(acc[tau][0], acc[tau][1], acc[tau][2], acc[tau][3]);
            named_barrier(1, kConsumerThreads);
            if (q == 0 && threadIdx.x == 0) MOE_TRACE(1, 8);
            // (tile, pair row g, column n) -> h
            for (int i = threadIdx.x; i < 64 * L.T; i += kConsumerThreads) {
                const int tau = i >> 6, gg = (i >> 3) & 7, n = i & 7;
                if (n >= nt) continue;
                const int src = gg * 4 + (n >> 1), comp = n & 1;
                float gate = 0.f, up = 0.f;
#pragma unroll
                for (int w = 0; w < kConsumerWarps; ++w) {
                    const float4 v = red[(w * L.T + tau) * kWarp + src];
                    gate += comp ? v.y : v.x;
                    up += comp ? v.w : v.z;
                }
                const float h = siluf_(gate) * up;
                const int j = d.first + 8 * tau + gg;
                if (d.pairs) {
                    const int pr = tok0 == 0 ? d.rows[n] : d.pairs[tok0 + n];
                    p.h_routed[(size_t)pr * Iu + j] = h;
                } else {
                    p.h_shared[(size_t)(tok0 + n) * Iu + j] = h;
                }
            }
            if (q == 0 && threadIdx.x == 0) MOE_TRACE(1, 9);
            named_barrier(1, kConsumerThreads);  // red is free again
            if (q == 0 && threadIdx.x == 0) MOE_TRACE(1, 10);
        }
        if (q < 2 && threadIdx.x == 0) MOE_TRACE(1, 3 + 2 * q);
        __syncwarp();  // this warp is done with the stage and its descriptor
        if (lane == 0) mbar_arrive(&empty[s]);
    }
}

template <int T>
__global__ void __launch_bounds__(kExpThreads, 1) gate_up_kernel(ExpertParams p)
{
    extern __shared__ __align__(128) unsigned char smem[];
    __shared__ __align__(8) uint64_t full[kMaxStages], empty[kMaxStages];
    __shared__ StageDesc desc[kMaxStages];
    __shared__ volatile int s_abort;
    const int warp = threadIdx.x >> 5;
    const GuLayout L = gu_layout(p);
    const int S = p.stages;
    const LocalPlan lp = plan_at(smem + (size_t)S * L.bytes + red_bytes(L.T), p.E, p.rows * p.K);

    if (threadIdx.x == 0) {
        s_abort = 0;
        for (int s = 0; s < S; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kConsumerWarps);
        }
        fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) MOE_TRACE(1, 0);
    if (warp == kConsumerWarps) gu_prefetch_shared(p, smem, full, desc);
    pdl_wait();
    pdl_trigger();
    const int n_active = build_local_plan(p, lp);
    if (threadIdx.x == 0) MOE_TRACE(1, 1);
    gu_items<T>(p, smem, full, empty, desc, s_abort, lp, n_active);
    if (threadIdx.x == 0) MOE_TRACE(1, 6);
}

// ------------------------------------------------------------ down+blend

// One K block's contribution to a down product, in the fixed arithmetic both
// down kernels share: (weight scale x h scale) x (hi product + lo product),
// each operation rounded on its own.  Components: rows g and g+8 of the
// tile, columns 2t and 2t+1.
__device__ __forceinline__ float4 down_partial(float ws, float h0, float h1, const float (&th)[4], const float (&tl)[4])
{
    const float a0 = __fmul_rn(ws, h0), a1 = __fmul_rn(ws, h1);
    return make_float4(__fmul_rn(a0, __fadd_rn(th[0], tl[0])), __fmul_rn(a1, __fadd_rn(th[1], tl[1])),
                       __fmul_rn(a0, __fadd_rn(th[2], tl[2])), __fmul_rn(a1, __fadd_rn(th[3], tl[3])));
}

// Reduction area of a down item: one float4 per lane for each (tile, K block).
__host__ __device__ constexpr size_t dn_red_bytes(int T, int ib) { return (size_t)T * (ib > 8 ? ib : 8) * kWarp * 16; }

// Stage layout (WS = Imax + 16): [drows weight rows][tok raw h rows, fp32]
// [tok h-hi rows][tok h-lo rows][h scales: tok * Imax/128][row-block scales:
// Imax/128]
struct DnLayout {
    int WS, T, imax;
    size_t hr, hh, hl, hs, sw, bytes;
};
__device__ __forceinline__ DnLayout dn_layout(const ExpertParams &p)
{
    DnLayout L;
    L.imax = max(p.I, p.Is);
    L.WS = L.imax + kRowPad;
    L.T = p.drows / 16;
    L.hr = (size_t)p.drows * L.WS;
    L.hh = L.hr + (size_t)p.tok * L.imax * 4;
    L.hl = L.hh + (size_t)p.tok * L.WS;
    L.hs = L.hl + (size_t)p.tok * L.WS;
    L.sw = L.hs + (size_t)p.tok * (L.imax / 128) * 4;
    L.bytes = align16(L.sw + (size_t)(L.imax / 128) * 4);
    return L;
}

__device__ void dn_produce(const ExpertParams &p, const DnLayout &L, StageDesc &d, unsigned char *st,
                           uint64_t *bar, uint64_t pol, bool weights, bool acts)
{
    const int lane = threadIdx.x & 31;
    const int ns = min(p.tok, d.n);
    // The row block's scales (I/128 floats) travel by bulk copy when they
    // are a whole number of 16-byte units.
    const int ib = d.inter / 128;
    const bool bsc = (ib % 4) == 0 && ((p.H / 128) % 4) == 0 && (smem_u32(st + L.sw) & 15) == 0;
    if (lane == 0) {
        uint32_t bytes = 0;
        if (weights) bytes += (uint32_t)(p.drows * d.inter) + (bsc ? (uint32_t)ib * 4 : 0);
        if (acts) bytes += (uint32_t)(ns * d.inter * 4);
        mbar_expect_tx(bar, bytes);
    }
    __syncwarp();
    if (weights) {
        const uint8_t *w2 = d.slab + (size_t)2 * d.inter * p.H + (size_t)d.first * d.inter;
        for (int i = lane; i < p.drows; i += kWarp)
            bulk_g2s_stream(st + (size_t)i * L.WS, w2 + (size_t)i * d.inter, (uint32_t)d.inter, bar, pol);
        float *sw = reinterpret_cast<float *>(st + L.sw);
        const float *src = d.scales + (2 * d.inter / 128) * (p.H / 128) + (d.first / 128) * ib;
        if (bsc) {
            if (lane == 0) bulk_g2s(sw, src, (uint32_t)ib * 4, bar);
        } else {
            for (int i = lane; i < ib; i += kWarp) sw[i] = __ldg(src + i);
        }
        if (lane < ns) d.wt[lane] = d.pairs ? __ldcg(p.topk_w + d.rows[lane]) : __ldcg(p.gsig + lane);
    }
    if (acts) {
        for (int i = lane; i < ns; i += kWarp) {
            const float *src = d.pairs ? p.h_routed + (size_t)d.rows[i] * d.inter : p.h_shared + (size_t)i * d.inter;
            bulk_g2s(st + L.hr + (size_t)i * L.imax * 4, src, (uint32_t)d.inter * 4, bar);
        }
    }
}

template <int T>
__global__ void __launch_bounds__(kExpThreads, 1) down_blend_kernel(ExpertParams p)
{
    extern __shared__ __align__(128) unsigned char smem[];
    __shared__ __align__(8) uint64_t full[kMaxStages], empty[kMaxStages];
    __shared__ StageDesc desc[kMaxStages];
    __shared__ volatile int s_abort, s_last;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const DnLayout L = dn_layout(p);
    const int per_block = p.H / p.drows;  // items per expert
    const int S = p.stages;
    float4 *red = reinterpret_cast<float4 *>(smem + (size_t)S * L.bytes);  // [tile][K block][lane]
    const LocalPlan lp = plan_at(smem + (size_t)S * L.bytes + dn_red_bytes(L.T, L.imax / 128), p.E, p.rows * p.K);

    if (threadIdx.x == 0) {
        s_abort = 0;
        for (int s = 0; s < S; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kConsumerWarps);
        }
        fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) MOE_TRACE(2, 0);
    // The router has finished when this kernel starts (its predecessor
    // waited for the router before letting this kernel launch), so the
    // routing is final: build the table and fetch the first stages' down
    // weights and scales now; only h waits for gate_up.
    const int n_active = build_local_plan(p, lp);
    const int n_items = per_block + n_active * per_block;

    if (warp == kConsumerWarps) {
        // ------------------------------------------------------- producer
        const uint64_t pol = policy_evict_first();
        for (int q = 0; q < S; ++q) {
            const int item = blockIdx.x + q * gridDim.x;
            if (item >= n_items) break;
            if (lane == 0) describe(p, item, per_block, per_block, p.drows, &lp, desc[q]);
            __syncwarp();
            dn_produce(p, L, desc[q], smem + q * L.bytes, &full[q], pol, true, false);
        }
        __syncwarp();  // the lanes' stage writes precede lane 0's arrivals
        pdl_wait();
        pdl_trigger();
        if (lane == 0) MOE_TRACE(2, 1);
        for (int q = 0;; ++q) {
            const int item = blockIdx.x + q * gridDim.x;
            if (item >= n_items) break;
            const int s = q % S;
            unsigned char *st = smem + s * L.bytes;
            if (q < S) {
                dn_produce(p, L, desc[s], st, &full[s], pol, false, true);
                __syncwarp();
                if (lane == 0) mbar_arrive(&full[s]);
                continue;
            }
            if (!mbar_wait(&empty[s], ((q / S) - 1) & 1, kWaitLimitNs)) {
                if (lane == 0) set_status(p.counters, MOE_ETIMEOUT);
                s_abort = 1;
                break;
            }
            if (lane == 0) {
                fence_proxy_async_smem();  // consumers' generic accesses precede the copies
                describe(p, item, per_block, per_block, p.drows, &lp, desc[s]);
            }
            __syncwarp();
            dn_produce(p, L, desc[s], st, &full[s], pol, true, true);
            __syncwarp();
            if (lane == 0) mbar_arrive(&full[s]);
        }
        return;
    }

    // ----------------------------------------------------------- consumers
    pdl_wait();
    pdl_trigger();
    const int g = lane >> 2, t = lane & 3;
    for (int q = 0;; ++q) {
        const int item = blockIdx.x + q * gridDim.x;
        if (item >= n_items) break;
        const int s = q % S;
        unsigned char *st = smem + s * L.bytes;
        if (!s_abort && !mbar_wait(&full[s], (q / S) & 1, kWaitLimitNs)) {
            if (lane == 0) set_status(p.counters, MOE_ETIMEOUT);
            s_abort = 1;
        }
        named_barrier(1, kConsumerThreads);  // every consumer warp sees the same abort flag
        if (q < 2 && threadIdx.x == 0) MOE_TRACE(2, 2 + 3 * q);
        const bool skip = s_abort;  // keep the loop (and its barriers) uniform after a timeout
        const StageDesc &d = desc[s];  // read in place; the producer rewrites it only after "empty"
        const int Iu = d.inter;
        const int ib = Iu / 128;
        const float *sw = reinterpret_cast<const float *>(st + L.sw);
        float *hsc = reinterpret_cast<float *>(st + L.hs);
        for (int s0 = 0; s0 < (skip ? 0 : d.n); s0 += p.tok) {
            const int ns = min(p.tok, d.n - s0);
            if (s0 > 0) {  // more slots than a stage holds: restage raw h in place
                named_barrier(1, kConsumerThreads);
                float4 *hv = reinterpret_cast<float4 *>(st + L.hr);
                const int iv = Iu / 4, rv = L.imax / 4;
                for (int i = threadIdx.x; i < ns * iv; i += kConsumerThreads) {
                    const int tr = i / iv;
                    const float *src = d.pairs ? p.h_routed + (size_t)d.pairs[s0 + tr] * Iu
                                               : p.h_shared + (size_t)(s0 + tr) * Iu;
                    hv[tr * rv + (i - tr * iv)] = __ldcg(reinterpret_cast<const float4 *>(src) + (i - tr * iv));
                }
                named_barrier(1, kConsumerThreads);
            }
            // h -> hi/lo e4m3 with one scale per (slot, 128 block): a warp per block
            for (int u = warp; u < ns * ib; u += kConsumerWarps) {
                const int tr = u / ib, kb = u - tr * ib;
                const float4 v = reinterpret_cast<const float4 *>(st + L.hr + (size_t)tr * L.imax * 4)[kb * 32 + lane];
                const float amax = warp_max(fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w))));
                const float sc = amax > 0.f ? amax / 448.f : 1.f;
                uint32_t hi, lo;
                quant4_hilo(v, 1.f / sc, hi, lo);
                reinterpret_cast<uint32_t *>(st + L.hh + (size_t)tr * L.WS)[kb * 32 + lane] = hi;
                reinterpret_cast<uint32_t *>(st + L.hl + (size_t)tr * L.WS)[kb * 32 + lane] = lo;
                if (lane == 0) hsc[tr * (L.imax / 128) + kb] = sc;
            }
            named_barrier(1, kConsumerThreads);
            if (q == 0 && threadIdx.x == 0) MOE_TRACE(2, 9);
            // (tile, K block) units over the warps; per unit all fragments first,
            // then the MMAs, hi and lo products on separate accumulator chains.
            // Each unit's scaled partial goes to its own slot of `red`; the
            // partials are then summed in K-block order, so that the result
            // does not depend on how units were spread over warps.
            const bool col_ok = g < ns;
            for (int u = warp; u < T * ib; u += kConsumerWarps) {
                const int tau = u % T, kb = u / T;
                uint2 bh[4], bl[4], ra[4], rb[4];
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const int k0 = kb * 128 + c * 32 + 8 * t;
                    bh[c] = bl[c] = make_uint2(0, 0);
                    if (col_ok) {
                        bh[c] = *reinterpret_cast<const uint2 *>(st + L.hh + (size_t)g * L.WS + k0);
                        bl[c] = *reinterpret_cast<const uint2 *>(st + L.hl + (size_t)g * L.WS + k0);
                    }
                    ra[c] = *reinterpret_cast<const uint2 *>(st + (size_t)(16 * tau + g) * L.WS + k0);
                    rb[c] = *reinterpret_cast<const uint2 *>(st + (size_t)(16 * tau + g + 8) * L.WS + k0);
                }
                float th[4] = {0.f, 0.f, 0.f, 0.f}, tl[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    mma_e4m3_16832(th, ra[c].x, rb[c].x, ra[c].y, rb[c].y, bh[c].x, bh[c].y);
                    mma_e4m3_16832(tl, ra[c].x, rb[c].x, ra[c].y, rb[c].y, bl[c].x, bl[c].y);
                }
                const float ws_ = sw[kb];
                const float h0 = (2 * t < ns) ? hsc[(2 * t) * (L.imax / 128) + kb] : 0.f;
                const float h1 = (2 * t + 1 < ns) ? hsc[(2 * t + 1) * (L.imax / 128) + kb] : 0.f;
                red[(tau * ib + kb) * kWarp + lane] = down_partial(ws_, h0, h1, th, tl);
            }
            if (q == 0 && threadIdx.x == 0) MOE_TRACE(2, 10);
            named_barrier(1, kConsumerThreads);
            if (q == 0 && threadIdx.x == 0) MOE_TRACE(2, 11);
            // (output row, slot column) -> weighted partial
            for (int i = threadIdx.x; i < 128 * L.T; i += kConsumerThreads) {
                const int tau = i >> 7, r = (i >> 3) & 15, n = i & 7;
                if (n >= ns) continue;
                const int src = (r & 7) * 4 + (n >> 1), comp = (n & 1) + (r >= 8 ? 2 : 0);
                float y = 0.f;
                for (int kb = 0; kb < ib; ++kb) {
                    const float4 v = red[(tau * ib + kb) * kWarp + src];
                    y = __fadd_rn(y, comp == 0 ? v.x : comp == 1 ? v.y : comp == 2 ? v.z : v.w);
                }
                const int row = d.first + 16 * tau + r;
                int yrow;
                float wt;
                if (d.pairs) {
                    yrow = s0 == 0 ? d.rows[n] : d.pairs[s0 + n];
                    wt = s0 == 0 ? d.wt[n] : __ldcg(p.topk_w + yrow);
                } else {
                    yrow = p.rows * p.K + s0 + n;
                    wt = s0 == 0 ? d.wt[n] : __ldcg(p.gsig + s0 + n);
                }
                p.yslot[(size_t)yrow * p.H + row] = __fmul_rn(wt, y);
            }
            if (q == 0 && threadIdx.x == 0) MOE_TRACE(2, 12);
            named_barrier(1, kConsumerThreads);  // red and the h staging are free again
        }
        if (q < 2 && threadIdx.x == 0) MOE_TRACE(2, 3 + 3 * q);
        const int chunk = d.first / p.drows;
        named_barrier(1, kConsumerThreads);  // every warp is done with the stage and its descriptor
        if (lane == 0) mbar_arrive(&empty[s]);  // the producer may refill the stage
        // Count the item; the last item of a row block blends it.
        if (threadIdx.x == 0) {
            const int prev = skip ? -1 : atomic_add_acq_rel_gpu(p.counters + kCtrBlend + chunk, 1);
            s_last = (prev == n_active);  // n_active routed items + 1 shared item per block
        }
        named_barrier(1, kConsumerThreads);
        if (s_last) {
            __threadfence();
            const int n0 = chunk * p.drows;
            for (int i = threadIdx.x; i < p.rows * p.drows; i += kConsumerThreads) {
                const int tr = i / p.drows;
                const int n = n0 + (i - tr * p.drows);
                float a = 0.f;
                for (int r = 0; r < p.K; ++r) a += __ldcg(p.yslot + (size_t)(tr * p.K + r) * p.H + n);
                a += __ldcg(p.yslot + (size_t)(p.rows * p.K + tr) * p.H + n);
                if (p.residual) a += bf16_bits_to_f32(p.residual[(size_t)tr * p.H + n]);
                p.out[(size_t)tr * p.H + n] = f32_to_bf16_bits(a);
            }
            if (threadIdx.x == 0) p.counters[kCtrBlend + chunk] = 0;
        }
        named_barrier(1, kConsumerThreads);  // s_last is read by all before the next item sets it
        if (q < 2 && threadIdx.x == 0) MOE_TRACE(2, 4 + 3 * q);
    }
    if (threadIdx.x == 0) MOE_TRACE(2, 8);
}

// ------------------------------------------------------- down, few rows

// For a few rows, the down product and blend by output block: a CTA item is
// 16 output rows (one MMA tile) for every active expert and the shared
// expert, so each output element is complete inside one CTA and is written
// straight to `out` (no per-slot partials in HBM, no cross-CTA counting).
// The item's experts are streamed through a two-stage ring `ue` at a time;
// each expert's 16 x I block arrives by TMA in 128-byte-swizzled boxes of
// 16 rows x 128 bytes (one box per 128-wide K block).  Every h row arrives
// by bulk copy and is quantised once per CTA.  The arithmetic is the one the
// item-based down kernel uses (down_partial, K blocks in order, rank-order
// blend), so the two kernels give identical bits.
struct DsLayout {
    int WS, imax, ib, ibp, ue, S_all;
    size_t sc, stage, hraw, hh, hl, hs, ys, wt, plan;
};
__host__ __device__ inline DsLayout ds_layout(int K, int I, int Is, int rows, int ue, int stages)
{
    DsLayout L;
    L.imax = I > Is ? I : Is;
    L.WS = L.imax + kRowPad;
    L.ib = L.imax / 128;
    L.ibp = (L.ib + 3) / 4 * 4;
    L.ue = ue;
    L.S_all = rows * K + rows;
    L.sc = (size_t)ue * L.ib * 2048;
    L.stage = (L.sc + (size_t)ue * L.ibp * 4 + 1023) / 1024 * 1024;
    L.hraw = (size_t)stages * L.stage;
    L.hh = L.hraw + (size_t)L.S_all * L.imax * 4;
    L.hl = L.hh + (size_t)L.S_all * L.WS;
    L.hs = L.hl + (size_t)L.S_all * L.WS;
    L.ys = L.hs + align16((size_t)L.S_all * L.ib * 4);
    L.wt = L.ys + (size_t)L.S_all * 16 * 4;
    L.plan = L.wt + align16((size_t)L.S_all * 4);
    return L;
}

struct DsParams {
    CUtensorMap w2r;  // routed down weights: (I bytes, H rows, E experts), boxes 128 B x 16 rows
    CUtensorMap w2s;  // shared expert's down weights: (Is bytes, H rows)
    ExpertParams p;
};

// Byte offset of (row r, K byte k) of a 16-row box group laid out by TMA with
// the 128-byte swizzle: box kb = k / 128 at kb * 2048; in a box, row r at
// r * 128 with its 16-byte units permuted by r mod 8.
__device__ __forceinline__ uint32_t sw128_off(int r, int k)
{
    const int kb = k >> 7, o = k & 127;
    return (uint32_t)(kb * 2048 + r * 128 + ((((o >> 4) ^ (r & 7))) << 4) + (o & 15));
}

// Producer warp: W2 rows [16 rb, +16) of experts [u0, u0 + n) of the table
// (index n_active is the shared expert) and their row-block scales.
__device__ void ds_produce(const DsParams &P, const DsLayout &L, const LocalPlan &lp, int n_active, int rb, int u0,
                           int n, unsigned char *st, uint64_t *bar, uint64_t pol)
{
    const ExpertParams &p = P.p;
    const int lane = threadIdx.x & 31;
    uint32_t bytes = 0;
    for (int j = 0; j < n; ++j) {
        const int ibu = ((u0 + j < n_active) ? p.I : p.Is) / 128;
        bytes += (uint32_t)ibu * 2048 + (ibu % 4 == 0 ? (uint32_t)ibu * 4 : 0);
    }
    if (lane == 0) mbar_expect_tx(bar, bytes);
    __syncwarp();
    for (int i = lane; i < n * L.ib; i += kWarp) {
        const int j = i / L.ib, kb = i - j * L.ib, u = u0 + j;
        const bool sh = u >= n_active;
        if (kb >= (sh ? p.Is : p.I) / 128) continue;
        unsigned char *dst = st + ((size_t)j * L.ib + kb) * 2048;
        if (sh) tma_load_2d(dst, &P.w2s, kb * 128, 16 * rb, bar, pol);
        else tma_load_3d(dst, &P.w2r, kb * 128, 16 * rb, lp.e_of[u], bar, pol);
    }
    for (int j = lane; j < n; j += kWarp) {
        const int u = u0 + j;
        const bool sh = u >= n_active;
        const int inter = sh ? p.Is : p.I, ibu = inter / 128;
        const float *src = (sh ? p.ssc : p.sc + (size_t)lp.e_of[u] * expert_nscales(p.H, p.I)) +
                           (2 * inter / 128) * (p.H / 128) + ((16 * rb) / 128) * ibu;
        float *dst = reinterpret_cast<float *>(st + L.sc) + j * L.ibp;
        if (ibu % 4 == 0) {
            bulk_g2s(dst, src, (uint32_t)ibu * 4, bar);
        } else {
            for (int k = 0; k < ibu; ++k) dst[k] = __ldg(src + k);
        }
    }
    __syncwarp();  // the lanes' scale stores precede the arrival
    if (lane == 0) mbar_arrive(bar);
}

// Producer warp: every h row (routed slots, then the shared rows) into the
// CTA's h area by bulk copy, completing `bar`.
__device__ void ds_produce_h(const ExpertParams &p, const DsLayout &L, unsigned char *smem, uint64_t *bar)
{
    const int lane = threadIdx.x & 31;
    const int PR = p.rows * p.K;
    if (lane == 0) mbar_arrive_expect_tx(bar, (uint32_t)(PR * p.I + p.rows * p.Is) * 4);
    __syncwarp();
    for (int sl = lane; sl < L.S_all; sl += kWarp) {
        const bool sh = sl >= PR;
        const float *src = sh ? p.h_shared + (size_t)(sl - PR) * p.Is : p.h_routed + (size_t)sl * p.I;
        bulk_g2s(smem + L.hraw + (size_t)sl * L.imax * 4, src, (uint32_t)(sh ? p.Is : p.I) * 4, bar);
    }
}

// The down-by-output-block item loops, once the routing table lp (n_active
// routed experts) and the slot weights wt (routing weights, then the shared
// gates: rows*K + rows floats) are in shared memory.  The producer warp
// streams W2 tiles through the stage ring and then the h rows (after
// gate_up: they wait for it here); the consumer warps quantise h once and
// write out.  Every thread of the CTA calls this.
__device__ void ds_items(const DsParams &P, unsigned char *smem, uint64_t *full, uint64_t *empty, uint64_t *hbar,
                         volatile int &s_abort, const LocalPlan &lp, int n_active, const float *wt)
{
    const ExpertParams &p = P.p;
    const int ue = p.ue, S = p.stages;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const DsLayout L = ds_layout(p.K, p.I, p.Is, p.rows, ue, S);
    const int PR = p.rows * p.K;
    float *ys = reinterpret_cast<float *>(smem + L.ys);
    float *hs = reinterpret_cast<float *>(smem + L.hs);
    const int n_exp = n_active + 1;             // + the shared expert
    const int chunks = (n_exp + ue - 1) / ue;   // stage loads per item
    const int n_items = p.H / 16;
    if (warp == kConsumerWarps) {
        // ------------------------------------------------------- producer
        const uint64_t pol = policy_evict_first();
        int q = 0;
        bool h_done = false;
        for (int item = blockIdx.x; item < n_items && !s_abort; item += gridDim.x) {
            for (int c = 0; c < chunks; ++c, ++q) {
                const int s = q % S;
                if (q == S && !h_done) {  // the first stages are in flight: now h (after gate_up)
                    h_done = true;
                    pdl_wait();
                    pdl_trigger();
                    ds_produce_h(p, L, smem, hbar);
                }
                if (q >= S && !mbar_wait(&empty[s], ((q / S) - 1) & 1, kWaitLimitNs)) {
                    if (lane == 0) set_status(p.counters, MOE_ETIMEOUT);
                    s_abort = 1;
                    break;
                }
                if (lane == 0 && q >= S) fence_proxy_async_smem();
                __syncwarp();
                ds_produce(P, L, lp, n_active, item, c * ue, min(ue, n_exp - c * ue), smem + (size_t)s * L.stage,
                           &full[s], pol);
            }
        }
        if (!h_done) {
            pdl_wait();
            pdl_trigger();
            ds_produce_h(p, L, smem, hbar);
        }
        return;
    }

    // ----------------------------------------------------------- consumers
    pdl_wait();
    pdl_trigger();
    if (threadIdx.x == 0) MOE_TRACE(2, 1);
    if (!mbar_wait(hbar, 0, kWaitLimitNs)) {
        if (lane == 0) set_status(p.counters, MOE_ETIMEOUT);
        s_abort = 1;
    }
    // every h row -> hi/lo e4m3 with a scale per (slot, 128 block): a warp per block
    {
        const int units_r = PR * (p.I / 128), units = units_r + p.rows * (p.Is / 128);
        for (int u = warp; u < units; u += kConsumerWarps) {
            int sl, kb;
            if (u < units_r) {
                sl = u / (p.I / 128);
                kb = u - sl * (p.I / 128);
            } else {
                const int w = u - units_r;
                const int t = w / (p.Is / 128);
                kb = w - t * (p.Is / 128);
                sl = PR + t;
            }
            const float4 v = reinterpret_cast<const float4 *>(smem + L.hraw + (size_t)sl * L.imax * 4)[kb * 32 + lane];
            const float amax = warp_max(fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w))));
            const float sc = amax > 0.f ? amax / 448.f : 1.f;
            uint32_t hi, lo;
            quant4_hilo(v, 1.f / sc, hi, lo);
            reinterpret_cast<uint32_t *>(smem + L.hh + (size_t)sl * L.WS)[kb * 32 + lane] = hi;
            reinterpret_cast<uint32_t *>(smem + L.hl + (size_t)sl * L.WS)[kb * 32 + lane] = lo;
            if (lane == 0) hs[sl * L.ib + kb] = sc;
        }
    }
    named_barrier(1, kConsumerThreads);
    if (threadIdx.x == 0) MOE_TRACE(2, 2);
    const int g = lane >> 2, t = lane & 3;
    int q = 0;
    for (int item = blockIdx.x; item < n_items; item += gridDim.x) {
        for (int c = 0; c < chunks; ++c, ++q) {
            const int s = q % S;
            const unsigned char *st = smem + (size_t)s * L.stage;
            if (!s_abort && !mbar_wait(&full[s], (q / S) & 1, kWaitLimitNs)) {
                if (lane == 0) set_status(p.counters, MOE_ETIMEOUT);
                s_abort = 1;
            }
            named_barrier(1, kConsumerThreads);  // every consumer warp sees the same abort flag
            if (q == 0 && threadIdx.x == 0) MOE_TRACE(2, 3);
            const int n = s_abort ? 0 : min(ue, n_exp - c * ue);
            for (int j = warp; j < n; j += kConsumerWarps) {
                const int u = c * ue + j;
                const bool sh = u >= n_active;
                const int ibu = (sh ? p.Is : p.I) / 128;
                const int f0 = sh ? 0 : lp.first_of[u];
                const int ncol = sh ? p.rows : lp.first_of[u + 1] - f0;  // <= rows <= 8
                const int sg = g < ncol ? (sh ? PR + g : lp.pairs[f0 + g]) : -1;
                const int c0 = 2 * t < ncol ? (sh ? PR + 2 * t : lp.pairs[f0 + 2 * t]) : -1;
                const int c1 = 2 * t + 1 < ncol ? (sh ? PR + 2 * t + 1 : lp.pairs[f0 + 2 * t + 1]) : -1;
                const float *wsc = reinterpret_cast<const float *>(st + L.sc) + j * L.ibp;
                const unsigned char *wj = st + (size_t)j * L.ib * 2048;
                float4 y = make_float4(0.f, 0.f, 0.f, 0.f);
                for (int kb = 0; kb < ibu; ++kb) {
                    uint2 bh[4], bl[4], ra[4], rb[4];
#pragma unroll
                    for (int cc = 0; cc < 4; ++cc) {
                        const int k0 = kb * 128 + cc * 32 + 8 * t;
                        bh[cc] = bl[cc] = make_uint2(0, 0);
                        if (sg >= 0) {
                            bh[cc] = *reinterpret_cast<const uint2 *>(smem + L.hh + (size_t)sg * L.WS + k0);
                            bl[cc] = *reinterpret_cast<const uint2 *>(smem + L.hl + (size_t)sg * L.WS + k0);
                        }
                        ra[cc] = *reinterpret_cast<const uint2 *>(wj + sw128_off(g, k0));
                        rb[cc] = *reinterpret_cast<const uint2 *>(wj + sw128_off(g + 8, k0));
                    }
                    float th[4] = {0.f, 0.f, 0.f, 0.f}, tl[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                    for (int cc = 0; cc < 4; ++cc) {
                        mma_e4m3_16832(th, ra[cc].x, rb[cc].x, ra[cc].y, rb[cc].y, bh[cc].x, bh[cc].y);
                        mma_e4m3_16832(tl, ra[cc].x, rb[cc].x, ra[cc].y, rb[cc].y, bl[cc].x, bl[cc].y);
                    }
                    const float h0 = c0 >= 0 ? hs[c0 * L.ib + kb] : 0.f;
                    const float h1 = c1 >= 0 ? hs[c1 * L.ib + kb] : 0.f;
                    const float4 v = down_partial(wsc[kb], h0, h1, th, tl);
                    y.x = __fadd_rn(y.x, v.x);
                    y.y = __fadd_rn(y.y, v.y);
                    y.z = __fadd_rn(y.z, v.z);
                    y.w = __fadd_rn(y.w, v.w);
                }
                if (c0 >= 0) {
                    ys[c0 * 16 + g] = y.x;
                    ys[c0 * 16 + g + 8] = y.z;
                }
                if (c1 >= 0) {
                    ys[c1 * 16 + g] = y.y;
                    ys[c1 * 16 + g + 8] = y.w;
                }
            }
            named_barrier(1, kConsumerThreads);  // the stage is consumed, ys is complete for these experts
            if (q == 0 && threadIdx.x == 0) MOE_TRACE(2, 4);
            if (lane == 0) mbar_arrive(&empty[s]);
        }
        // out[t][16 item + r]: the k weighted partials in rank order, then the
        // shared expert's, then the residual; one bf16 rounding
        if (!s_abort) {
            for (int i = threadIdx.x; i < p.rows * 16; i += kConsumerThreads) {
                const int tr = i >> 4, r = i & 15;
                float a = 0.f;
                for (int k = 0; k < p.K; ++k) {
                    const int sl = tr * p.K + k;
                    a = __fadd_rn(a, __fmul_rn(wt[sl], ys[sl * 16 + r]));
                }
                a = __fadd_rn(a, __fmul_rn(wt[PR + tr], ys[(PR + tr) * 16 + r]));
                const size_t o = (size_t)tr * p.H + 16 * item + r;
                if (p.residual) a = __fadd_rn(a, bf16_bits_to_f32(p.residual[o]));
                p.out[o] = f32_to_bf16_bits(a);
            }
        }
        named_barrier(1, kConsumerThreads);  // ys may be rewritten by the next item
    }
}

__global__ void __launch_bounds__(kExpThreads, 1) down_small_kernel(const __grid_constant__ DsParams P)
{
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    __shared__ __align__(8) uint64_t full[kMaxStages], empty[kMaxStages], hbar;
    __shared__ volatile int s_abort;
    const ExpertParams &p = P.p;
    unsigned char *smem =
        reinterpret_cast<unsigned char *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const DsLayout L = ds_layout(p.K, p.I, p.Is, p.rows, p.ue, p.stages);
    const LocalPlan lp = plan_at(smem + L.plan, p.E, p.rows * p.K);
    const int PR = p.rows * p.K;
    float *wt = reinterpret_cast<float *>(smem + L.wt);

    if (threadIdx.x == 0) {
        s_abort = 0;
        for (int s = 0; s < p.stages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kConsumerWarps);
        }
        mbar_init(&hbar, 1);
        fence_mbar_init();
    }
    if (warp == kConsumerWarps && lane == 0) {
        tma_prefetch_desc(&P.w2r);
        tma_prefetch_desc(&P.w2s);
    }
    __syncthreads();
    if (threadIdx.x == 0) MOE_TRACE(2, 0);
    // The router finished before this kernel could launch: the routing is final.
    const int n_active = build_local_plan(p, lp);
    for (int i = threadIdx.x; i < L.S_all; i += blockDim.x)
        wt[i] = i < PR ? __ldcg(p.topk_w + i) : __ldcg(p.gsig + i - PR);
    __syncthreads();  // every thread wrote some of wt; the consumers read all of it
    ds_items(P, smem, full, empty, &hbar, s_abort, lp, n_active, wt);
    if (threadIdx.x == 0) MOE_TRACE(2, 8);
}

#ifdef MOE_PHASE_TRACE
extern "C" __attribute__((visibility("default"))) int moe_trace_set(void *p)
{
    return (int)cudaMemcpyToSymbol(g_moe_trace, &p, sizeof(p));
}
#endif

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

DecodeShape decode_shape(const moe_dims &d, int64_t rows)
{
    DecodeShape s{};
    const int H = d.hidden, I = d.inter, Is = d.shared_inter, E = d.n_experts;
    const int imax = std::max(I, Is);
    rows = std::max<int64_t>(rows, 1);
    // router: rows_per_cta router rows (<= 32 KB) and kRouterTok activation rows per CTA
    s.router_rows = std::max(1, std::min(kRouterMaxRows, 32768 / H));
    s.router_groups = (int)std::min<int64_t>((rows + kRouterTok - 1) / kRouterTok, kMaxRouterGroups);
    s.router_group_tokens = (int)((rows + s.router_groups - 1) / s.router_groups);
    s.router_smem = std::max<size_t>((size_t)(s.router_rows + kRouterTok) * H * 2, (size_t)(3 * E + 33) * 4);
    s.logits_ld = (E + 1 + 3) / 4 * 4;
    // activation rows per item: the 8 MMA columns, fewer for wide rows
    s.tok = (int)std::min<int64_t>({(int64_t)kDescPairs, rows, std::max(1, 16384 / H)});
    // Each expert kernel has an SM to itself (measured: deeper rings of larger
    // items beat sharing an SM between a gate_up and a down CTA).
    const size_t budget = 224 * 1024 - 2048;
    const int sms = std::max(1, device_info().sm_count);
    const int64_t umax = std::min<int64_t>(E, rows * d.top_k);
    const size_t plan = plan_bytes(E, (int)(rows * d.top_k));
    const size_t ws_g = (size_t)H + kRowPad;
    auto gu_stage_of = [&](int pr) {
        return align16(16 * (pr / 8) * ws_g + 2 * s.tok * ws_g + (size_t)s.tok * (H / 128) * 4 + (size_t)2 * (H / 128) * 4);
    };
    auto gu_items = [&](int pr) { return (int64_t)(Is / pr) + umax * (I / pr); };
    // gate_up: 8..32 gate/up row pairs per item (a power of two: divides I and
    // Is); grown while an item stays <= 64 KB of weights, two stages fit and
    // every SM still gets an item
    int pairs = 8;
    while (pairs * 2 <= 32 && pairs * 2 * 2 * H <= 65536 && gu_items(pairs * 2) >= sms &&
           2 * gu_stage_of(pairs * 2) + red_bytes(pairs * 2 / 8) + plan <= budget)
        pairs *= 2;
    s.gu_pairs = pairs;
    const size_t gu_stage = gu_stage_of(pairs);
    const size_t gu_extra = red_bytes(pairs / 8) + plan;
    const int64_t gu_per_cta = (gu_items(pairs) + sms - 1) / sms;
    int gs = (int)std::min<int64_t>(std::max<int64_t>(gu_per_cta, 2), kMaxStages);
    while (gs > 1 && gs * gu_stage + gu_extra > budget) --gs;
    // down (item kernel): rows per item 16..64 (a power of two dividing H and
    // 128), ~32 KB of weights; as many stages as fit
    const size_t ws_d = (size_t)imax + kRowPad;
    int drows = 16;
    while (drows * 2 <= 64 && drows * 2 * imax <= 32768) drows *= 2;
    const size_t dn_stage = align16(drows * ws_d + (size_t)s.tok * imax * 4 + 2 * s.tok * ws_d +
                                    (size_t)s.tok * (imax / 128) * 4 + (size_t)(imax / 128) * 4);
    const size_t dn_extra = dn_red_bytes(drows / 16, imax / 128) + plan;
    const int64_t dn_per_cta = ((umax + 1) * (H / drows) + sms - 1) / sms;
    int ds = (int)std::min<int64_t>(std::max<int64_t>(dn_per_cta, 2), kMaxStages);
    while (ds > 1 && ds * dn_stage + dn_extra > budget) --ds;
    s.dn_rows = drows;
    // gate_up warms L2 with the active experts' down weights when they take
    // a small part of it
    s.l2_w2 = (umax * (int64_t)I * H + (int64_t)Is * H) <= (int64_t)48 << 20;
    s.gu_stages = gs;
    s.dn_stages = ds;
    s.gu_smem = gs * gu_stage + gu_extra;
    s.dn_smem = ds * dn_stage + dn_extra;
    s.ds_ue = 0;
    // Few rows: the down product by output block (one CTA item = 16 output
    // rows of every active expert, two stages of up to all of them), when it
    // fits; gate_up then has the SM to itself and warms L2 with the down
    // weights instead.
    if (rows <= kDescPairs) {
        const int u1 = (int)umax + 1;
        for (int ue = u1; ue >= 1; --ue) {
            const DsLayout Ls = ds_layout(d.top_k, I, Is, (int)rows, ue, 2);
            const size_t need = Ls.plan + plan + 1024;  // + alignment slack (1024-byte TMA boxes)
            if (need <= budget) {
                s.ds_ue = ue;
                s.dn_stages = 2;
                s.dn_smem = need;
                s.dn_rows = 16;
                s.l2_w2 = true;
                break;
            }
        }
    }
    return s;
}

cudaError_t launch_wait_probe(int32_t *counters, uint64_t limit_ns, cudaStream_t s)
{
    wait_probe_kernel<<<1, 32, 0, s>>>(counters, limit_ns);
    return cudaGetLastError();
}

cudaError_t launch_router_topk(const RouterLaunch &a, cudaStream_t s)
{
    const moe_dims &d = *a.d;
    const DecodeShape sh = decode_shape(d, a.rows);
    RouterParams p;
    p.x = a.x;
    p.rows = a.rows;
    p.H = d.hidden;
    p.E = d.n_experts;
    p.K = d.top_k;
    p.ld = sh.logits_ld;
    p.rows_per_cta = sh.router_rows;
    p.group_tokens = sh.router_group_tokens;
    p.wr = a.router_w;
    p.bias = a.router_bias;
    p.g = a.shared_gate;
    p.logits = a.logits;
    p.xq = a.xq;
    p.xsc = a.xsc;
    p.topk_idx = a.topk_idx;
    p.topk_w = a.topk_w;
    p.gsig = a.gsig;
    p.counters = a.counters;
    const dim3 grid((d.n_experts + 1 + sh.router_rows - 1) / sh.router_rows,
                    (a.rows + sh.router_group_tokens - 1) / sh.router_group_tokens);
    if (occupancy(router_topk_kernel, sh.router_rows * kWarp, sh.router_smem) < 1)
        return cudaErrorInvalidConfiguration;
    return launch_kernel(router_topk_kernel, grid, dim3(sh.router_rows * kWarp), sh.router_smem, s, p);
}

cudaError_t launch_decode_experts(const ExpertsLaunch &a, cudaStream_t s)
{
    const moe_dims &d = *a.d;
    const DeviceInfo &di = device_info();
    const DecodeShape sh = decode_shape(d, a.rows);
    ExpertParams p;
    p.x = a.x;
    p.xq = a.xq;
    p.xsc = a.xsc;
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
    p.topk_idx = a.topk_idx;
    p.topk_w = a.topk_w;
    p.gsig = a.gsig;
    p.h_routed = a.h_routed;
    p.h_shared = a.h_shared;
    p.yslot = a.yslot;
    p.residual = a.residual;
    p.out = a.out;
    p.counters = a.counters;
    p.tok = sh.tok;
    p.pairs = sh.gu_pairs;
    p.drows = sh.dn_rows;
    const int64_t max_active = std::min<int64_t>(d.n_experts, (int64_t)a.rows * d.top_k);

    // gate_up
    {
        p.stages = sh.gu_stages;
        p.ue = 0;
        p.l2_w2 = sh.l2_w2 ? 1 : 0;
        void (*kern)(ExpertParams) = sh.gu_pairs == 8    ? gate_up_kernel<1>
                                     : sh.gu_pairs == 16 ? gate_up_kernel<2>
                                                         : gate_up_kernel<4>;
        const int bps = occupancy(kern, kExpThreads, sh.gu_smem);
        if (bps < 1) return cudaErrorInvalidConfiguration;
        const int64_t items = (int64_t)(d.shared_inter / sh.gu_pairs) + max_active * (d.inter / sh.gu_pairs);
        const int grid = (int)std::min<int64_t>(items, (int64_t)di.sm_count);
        cudaError_t e = launch_kernel(kern, dim3(grid), dim3(kExpThreads), sh.gu_smem, s, p);
        if (e != cudaSuccess) return e;
    }
    // down + blend
    if (sh.ds_ue > 0) {
        p.stages = sh.dn_stages;
        p.ue = sh.ds_ue;
        DsParams dp;
        dp.p = p;
        const int H = d.hidden, I = d.inter, Is = d.shared_inter;
        if (!make_map(&dp.w2r, a.expert_w8 + (size_t)2 * I * H, (uint64_t)I, (uint64_t)H, (uint64_t)d.n_experts,
                      (uint64_t)I, 3 * (uint64_t)I * H, 16) ||
            !make_map(&dp.w2s, a.shared_w8 + (size_t)2 * Is * H, (uint64_t)Is, (uint64_t)H, 1, (uint64_t)Is, 0, 16))
            return cudaErrorInvalidValue;
        const int bps = occupancy(down_small_kernel, kExpThreads, sh.dn_smem);
        if (bps < 1) return cudaErrorInvalidConfiguration;
        const int grid = std::min(d.hidden / 16, di.sm_count);
        return launch_kernel(down_small_kernel, dim3(grid), dim3(kExpThreads), sh.dn_smem, s, dp);
    }
    {
        p.stages = sh.dn_stages;
        void (*kern)(ExpertParams) = sh.dn_rows == 16   ? down_blend_kernel<1>
                                     : sh.dn_rows == 32 ? down_blend_kernel<2>
                                                        : down_blend_kernel<4>;
        const int bps = occupancy(kern, kExpThreads, sh.dn_smem);
        if (bps < 1) return cudaErrorInvalidConfiguration;
        const int64_t items = (max_active + 1) * (d.hidden / sh.dn_rows);
        const int grid = (int)std::min<int64_t>(items, (int64_t)di.sm_count);
        cudaError_t e = launch_kernel(kern, dim3(grid), dim3(kExpThreads), sh.dn_smem, s, p);
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}


}  // namespace moe
