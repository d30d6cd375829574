// prefill.cu -- prefill path (rows above a few dozen): token permute ->
// expert-grouped FP8 GEMMs on the tcgen05 tensor cores -> unpermute + blend.
//
// Launch chain (programmatic dependent launch between every pair):
//   1. router_tc_kernel: logits = x Wr^T (+ bias) and the shared-gate logit
//      x g on tcgen05 (bf16, M=128 rows, N = experts), the top-k of each row
//      straight from tensor memory, softmax over the k, and each (row, rank)
//      pair's position within its expert (an atomic count per expert).
//   2. scan_kernel (one CTA): expert offsets and the table of 128-row M tiles
//      (routed experts in order, then the shared expert over all rows).
//   3. permute_kernel: each pair's x row, quantised to hi/lo e4m3 with one
//      scale per 128 block, into its expert's contiguous rows; then every
//      row again in token order for the shared expert.
//   4. gemm_kernel<GEMM1>: per M tile and 128-column block j of h,
//      [gate_j | up_j] = A (hi+lo) x W13^T on tcgen05 (M=128, N=256, K=32 per
//      instruction), each 128-wide K block promoted into fp32 registers with
//      its row scale x block scale; epilogue h = silu(gate) * up, quantised
//      to hi/lo e4m3 with one scale per (row, 128 block) for GEMM2.
//   5. gemm_kernel<GEMM2>: y = h (hi+lo) x W2^T the same way; epilogue
//      scales by the row's routing weight (or the shared gate) into one
//      partial row per (row, slot).
//   6. blend_kernel: out[t] = sum of its k partials in rank order + the
//      shared partial (+ residual), rounded once to bf16.
//
// Rows space of the GEMMs: the T*k routed pairs sorted by expert, then the T
// shared-expert rows in token order.
#include <algorithm>
#include <mutex>
#include <vector>

#include "internal.h"
#include "launch.h"
#include "tcgen05.cuh"

namespace moe {

constexpr int kBM = 128;     // rows per M tile
constexpr int kBN = 256;     // accumulator columns per tile
constexpr int kBK = 128;     // K bytes per stage (one scale block of e4m3)
constexpr int kNT = 32;      // token rows per item of the narrow grouped GEMM (its MMA's N)
constexpr int kNtMaxKb = 32; // K blocks per item its scale table holds (K <= 4096)
constexpr int kGemmStages = 3;
constexpr int kEpiWarps = 16;
constexpr int kGemmThreads = 64 + 32 * kEpiWarps;  // warp 0: TMA, warp 1: MMA + TMEM, warps 2..17: epilogue
constexpr int kEpiThreads = 32 * kEpiWarps;
constexpr uint32_t kTmemCols = 512;  // two 256-column fp32 accumulators
constexpr size_t kStageBytes = 2 * kBM * kBK + kBN * kBK;  // A hi, A lo, B
constexpr int kStgBytes = 32 * 48;  // per epilogue warp: 32 rows x 48 B staging for coalesced stores
constexpr size_t kGemmSmem =
    kGemmStages * kStageBytes + 1024 /* alignment slack */ + 4096 /* amax exchange */ + kEpiWarps * kStgBytes;

// ------------------------------------------------------------ layout

struct PrefillLayout {
    size_t counters, logits, topk_idx, topk_w, gsig, counts, offsets, rank, pos, mtiles, xp, xps, slot_w, hq, hs,
        yslot, total;
    int64_t routed, rows_total, max_mtiles;
};

inline PrefillLayout prefill_layout(const moe_dims &d, int64_t T)
{
    PrefillLayout L{};
    const int64_t E = d.n_experts, K = d.top_k, H = d.hidden, I = d.inter, Is = d.shared_inter;
    const int64_t imax = std::max(I, Is);
    L.routed = T * K;
    L.rows_total = T * K + T;
    // group tiles of kNT rows (the narrow GEMMs) outnumber those of kBM rows
    L.max_mtiles = (T * K + kNT - 1) / kNT + E + (T + kNT - 1) / kNT + 1;
    size_t o = 0;
    auto take = [&](size_t bytes) { size_t at = o; o = align_up(o + bytes, 1024); return at; };
    L.counters = take(sizeof(int32_t) * kCounters);
    // up to kSmallRouterRows rows the decode path's router (spread over
    // many CTAs) computes the routing; it needs fp32 logits rows
    L.logits = take(T <= kSmallRouterRows ? sizeof(float) * T * ((E + 1 + 3) / 4 * 4) : 0);
    L.topk_idx = take(sizeof(int32_t) * T * K);
    L.topk_w = take(sizeof(float) * T * K);
    L.gsig = take(sizeof(float) * T);
    L.counts = take(sizeof(int32_t) * (E + 1));
    L.offsets = take(sizeof(int32_t) * (E + 2));
    L.rank = take(sizeof(int32_t) * T * K);
    L.pos = take(sizeof(int32_t) * T * K);
    L.mtiles = take(sizeof(int4) * (1 + L.max_mtiles));
    // routed rows, then the T shared rows; TMA boxes are 128 rows, so each of
    // the two tensors spans at least that many rows of the buffer
    L.xp = take((size_t)(std::max<int64_t>(L.routed, kBM) + std::max<int64_t>(T, kBM)) * 2 * H);
    L.xps = take(sizeof(float) * (L.routed + T) * (H / 128));
    L.slot_w = take(sizeof(float) * L.rows_total);
    L.hq = take((size_t)std::max<int64_t>(L.rows_total, kBM) * 2 * imax);
    L.hs = take(sizeof(float) * L.rows_total * (imax / 128));
    L.yslot = take(sizeof(float) * L.rows_total * H);
    L.total = o;
    return L;
}

size_t norm_buffer_offset(const moe_dims &d, int64_t rows)
{
    return align_up(std::max(decode_layout(d, rows).total, prefill_layout(d, rows).total), 256);
}

size_t workspace_bytes(const moe_dims &d, int64_t rows)
{
    return norm_buffer_offset(d, rows) + align_up((size_t)rows * d.hidden * 2, 256);
}

bool prefill_available() { return true; }

int prefill_kernel_launches(const moe_dims &, int64_t) { return 6; }

// The narrow GEMMs keep a K block's activation scales of every item in
// shared memory: K (H for GEMM1, the intermediate sizes for GEMM2) up to
// 128 * kNtMaxKb.
bool narrow_supported(const moe_dims &d)
{
    return d.hidden <= 128 * kNtMaxKb && d.inter <= 128 * kNtMaxKb && d.shared_inter <= 128 * kNtMaxKb;
}

// ------------------------------------------------------------ count / scan / permute

struct PlanParams {
    int T, E, K, H, I, Is;
    const int32_t *topk_idx;
    const float *topk_w;
    const float *gsig;
    int32_t *counts;   // [E]
    int32_t *offsets;  // [E+1]
    int32_t *rank;     // [T*K]
    int32_t *pos;      // [T*K]
    int4 *mtiles;      // [0].x = count; entries from [1]: {group, row0, rows, a_row0}
    int tile_rows;     // rows per group tile: kBM, or kNT for the narrow GEMMs
    int count_in_scan; // counts and ranks not given by the router: scan_kernel derives them
    int perm_split;    // permute_kernel: warps per token (its k + 1 destinations split between them)
    const uint16_t *x; // [T][H] bf16
    int xp_shared0;    // first xp row of the shared expert's rows (the routed rows span at least 128)
    uint8_t *xp;
    float *xps;
    float *slot_w;
    int32_t *counters;
};

__device__ int block_scan_excl(int v, int *scratch, int *total)
{
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nwarps = blockDim.x >> 5;
    int incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xFFFFFFFFu, incl, o);
        if (lane >= o) incl += y;
    }
    if (lane == 31) scratch[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        const int w = (lane < nwarps) ? scratch[lane] : 0;
        int wi = w;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xFFFFFFFFu, wi, o);
            if (lane >= o) wi += y;
        }
        if (lane < nwarps) scratch[lane] = wi - w;
        if (lane == 31) scratch[32] = wi;
    }
    __syncthreads();
    const int r = scratch[warp] + incl - v;
    *total = scratch[32];
    __syncthreads();
    return r;
}

// One CTA of 1024 threads: expert offsets and the table of group tiles
// (after each pair's rank within its expert, when the router gave none).
__global__ void __launch_bounds__(1024) scan_kernel(PlanParams p)
{
    __shared__ int scratch[33];
    __shared__ int s_cnt[kMaxExperts];
    pdl_wait();
    pdl_trigger();
    if (p.count_in_scan) {
        for (int e = threadIdx.x; e < p.E; e += blockDim.x) s_cnt[e] = 0;
        __syncthreads();
        for (int i = threadIdx.x; i < p.T * p.K; i += blockDim.x) {
            const int e = min(max(p.topk_idx[i], 0), p.E - 1);
            p.rank[i] = atomicAdd(&s_cnt[e], 1);
        }
        __syncthreads();
    }
    int run_rows = 0, run_tiles = 0;
    for (int e0 = 0; e0 < p.E; e0 += blockDim.x) {
        const int e = e0 + threadIdx.x;
        const int c = (e < p.E) ? (p.count_in_scan ? s_cnt[e] : p.counts[e]) : 0;
        const int mt = (c + p.tile_rows - 1) / p.tile_rows;
        int tot_rows, tot_tiles;
        const int off = block_scan_excl(c, scratch, &tot_rows) + run_rows;
        const int toff = block_scan_excl(mt, scratch, &tot_tiles) + run_tiles;
        if (e < p.E) {
            p.offsets[e] = off;
            for (int i = 0; i < mt; ++i)
                p.mtiles[1 + toff + i] =
                    make_int4(e, off + i * p.tile_rows, min(p.tile_rows, c - i * p.tile_rows), off + i * p.tile_rows);
        }
        run_rows += tot_rows;
        run_tiles += tot_tiles;
    }
    if (threadIdx.x == 0) p.offsets[p.E] = run_rows;
    // the shared expert: all T rows, in token order, after the routed rows
    const int tr = p.tile_rows;
    const int smt = (p.T + tr - 1) / tr;
    for (int i = threadIdx.x; i < smt; i += blockDim.x)
        p.mtiles[1 + run_tiles + i] = make_int4(p.E, p.T * p.K + i * tr, min(tr, p.T - i * tr), i * tr);
    if (threadIdx.x == 0) p.mtiles[0] = make_int4(run_tiles + smt, run_tiles, 0, 0);
}

// A token's x row is quantised to hi/lo e4m3 (hi codes [H], then lo codes
// [H]) with one scale per 128 block, amax / 448 (x ~ s * (hi + lo)), and
// written to each of its k expert rows and to its row of the shared expert;
// each routed pair's position and blend weight are recorded.  A warp takes
// one token and perm_split-th of its k + 1 destinations (few tokens: one
// destination per warp, so that the writes spread over many warps; many
// tokens: all of them, quantising once).  Rows of up to kPermMaxBlocks * 128
// elements keep their codes in registers; wider rows quantise again for each
// destination.
constexpr int kPermMaxBlocks = 32;

__device__ __forceinline__ void permute_write(const PlanParams &p, int dst_row, int dst_scale, int kb, int lane,
                                              uint32_t hi, uint32_t lo, float sc)
{
    uint32_t *dq = reinterpret_cast<uint32_t *>(p.xp + (size_t)dst_row * 2 * p.H);
    dq[kb * 32 + lane] = hi;
    dq[p.H / 4 + kb * 32 + lane] = lo;
    if (lane == 0) p.xps[(size_t)dst_scale * (p.H / 128) + kb] = sc;
}

__global__ void __launch_bounds__(256) permute_kernel(PlanParams p)
{
    pdl_wait();
    pdl_trigger();
    const int lane = threadIdx.x & 31;
    const int P = p.T * p.K;
    const int hb = p.H / 128;
    const int D = p.K + 1;  // destinations of a token: its k routed rows, then its shared row
    const int ns = p.perm_split;
    const int dpw = (D + ns - 1) / ns;
    const int gw = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int nw = (gridDim.x * blockDim.x) >> 5;
    for (int w = gw; w < p.T * ns; w += nw) {
        const int t = w / ns;
        const int d0 = (w - t * ns) * dpw, nd = min(D, d0 + dpw) - d0;
        if (nd <= 0) continue;
        // this warp's destinations: rows of xp and of its scales
        int row[kMaxTopK + 1], srow[kMaxTopK + 1];
        for (int c = 0; c < nd; ++c) {
            const int r = d0 + c;
            if (r < p.K) {
                const int i = t * p.K + r;
                const int e = min(max(p.topk_idx[i], 0), p.E - 1);
                row[c] = srow[c] = p.offsets[e] + p.rank[i];
                if (lane == 0) {
                    p.pos[i] = row[c];
                    p.slot_w[row[c]] = p.topk_w[i];
                }
            } else {
                row[c] = p.xp_shared0 + t;
                srow[c] = P + t;
                if (lane == 0) p.slot_w[P + t] = p.gsig[t];
            }
        }
        const uint2 *src = reinterpret_cast<const uint2 *>(p.x + (size_t)t * p.H);
        if (hb <= kPermMaxBlocks) {
            uint32_t hi[kPermMaxBlocks], lo[kPermMaxBlocks];
            float scv[kPermMaxBlocks];
#pragma unroll
            for (int kb = 0; kb < kPermMaxBlocks; ++kb) {
                if (kb >= hb) break;
                const uint2 raw = __ldg(src + kb * 32 + lane);
                const float4 v = make_float4(bf16_lo(raw.x), bf16_hi(raw.x), bf16_lo(raw.y), bf16_hi(raw.y));
                const float amax = warp_max(fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w))));
                scv[kb] = amax > 0.f ? amax / 448.f : 1.f;
                quant4_hilo(v, 1.f / scv[kb], hi[kb], lo[kb]);
            }
            for (int c = 0; c < nd; ++c) {
#pragma unroll
                for (int kb = 0; kb < kPermMaxBlocks; ++kb) {
                    if (kb >= hb) break;
                    permute_write(p, row[c], srow[c], kb, lane, hi[kb], lo[kb], scv[kb]);
                }
            }
        } else {
            for (int kb = 0; kb < hb; ++kb) {
                const uint2 raw = __ldg(src + kb * 32 + lane);
                const float4 v = make_float4(bf16_lo(raw.x), bf16_hi(raw.x), bf16_lo(raw.y), bf16_hi(raw.y));
                const float amax = warp_max(fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w))));
                const float sc = amax > 0.f ? amax / 448.f : 1.f;
                uint32_t h, l;
                quant4_hilo(v, 1.f / sc, h, l);
                for (int c = 0; c < nd; ++c) permute_write(p, row[c], srow[c], kb, lane, h, l, sc);
            }
        }
    }
}

// ------------------------------------------------------------ router on tcgen05

constexpr int kRtBK = 128;                         // K bytes per stage: 64 bf16
constexpr int kRtStages = 4;
constexpr int kRtThreads = 192;                    // warp 0: TMA, warp 1: MMA + TMEM, warps 2..5: top-k
constexpr int kRtChunk = 256;                      // experts per accumulator pass
constexpr size_t kRtStageBytes = (size_t)kBM * kRtBK + (size_t)kRtChunk * kRtBK + 16 * kRtBK;  // x, Wr, g
constexpr size_t kRtSmem = kRtStages * kRtStageBytes + 1024;

struct RouterTcParams {
    CUtensorMap x;    // [T][2H bytes], boxes of 128 rows
    CUtensorMap wr;   // [E][2H bytes], boxes of nbox rows
    CUtensorMap g;    // [1][2H bytes], boxes of 16 rows (rows past the first read as zero)
    int T, E, K, H;
    int nbox;         // rows of a router box / N of the expert MMA: min(256, E rounded up to 16)
    const float *bias;
    int32_t *topk_idx;
    float *topk_w;
    float *gsig;
    int32_t *counts;  // [E], zero on entry
    int32_t *rank;    // [T*K]
    int32_t *counters;
};

// Insert (k, e) into a row's running top-k (keys descending).  The new key
// goes in front of the first key it strictly exceeds, so equal keys keep the
// lower expert first.  Every place of the new list is taken from the old list
// at once (kept, shifted down one, or the new key): KM independent selects
// instead of a chain of compare-and-swaps through k, which one thread per row
// would otherwise run at the latency of each step.
template <int KM>
__device__ __forceinline__ void topk_insert(uint32_t (&keys)[KM], int (&ids)[KM], uint32_t k, int e)
{
    bool gt[KM];
#pragma unroll
    for (int j = 0; j < KM; ++j) gt[j] = k > keys[j];  // false then true: the list is sorted
    uint32_t nk[KM];
    int ni[KM];
#pragma unroll
    for (int j = 0; j < KM; ++j) {
        const bool shift = gt[j] && j > 0 && gt[j > 0 ? j - 1 : 0];
        nk[j] = !gt[j] ? keys[j] : (shift ? keys[j > 0 ? j - 1 : 0] : k);
        ni[j] = !gt[j] ? ids[j] : (shift ? ids[j > 0 ? j - 1 : 0] : e);
    }
#pragma unroll
    for (int j = 0; j < KM; ++j) {
        keys[j] = nk[j];
        ids[j] = ni[j];
    }
}

// One CTA per 128-row tile of x (persistent over tiles).  The accumulator
// holds one pass of up to 256 experts (TMEM columns [0, 256)) and the shared
// gate logit (column 256); an epilogue thread owns one row and keeps its
// running top-k in registers across passes.
template <int KM>
__global__ void __launch_bounds__(kRtThreads, 1) router_tc_kernel(const __grid_constant__ RouterTcParams p)
{
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    __shared__ __align__(8) uint64_t full[kRtStages], empty[kRtStages], acc_full, acc_empty;
    __shared__ uint32_t tmem_base_s;
    __shared__ volatile int s_abort;
    __shared__ float s_bias[kMaxExperts];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    unsigned char *smem = reinterpret_cast<unsigned char *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);

    for (int e = threadIdx.x; e < p.E; e += blockDim.x) s_bias[e] = p.bias ? __ldg(p.bias + e) : 0.f;
    if (threadIdx.x == 0) {
        s_abort = 0;
        for (int s = 0; s < kRtStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(&acc_full, 1);
        mbar_init(&acc_empty, 4);
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(&tmem_base_s, 512);
        tmem_relinquish();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&p.x);
        tma_prefetch_desc(&p.wr);
        tma_prefetch_desc(&p.g);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = tmem_base_s;

    pdl_wait();
    pdl_trigger();
    const int n_tiles = (p.T + kBM - 1) / kBM;
    const int npass = (p.E + kRtChunk - 1) / kRtChunk;
    const int nkb = 2 * p.H / kRtBK;
    const uint32_t stage_tx = (uint32_t)(kBM * kRtBK + p.nbox * kRtBK + 16 * kRtBK);

    if (warp == 0) {
        if (lane == 0) {
            const uint64_t pol = policy_evict_last();  // x and Wr are re-read by other tiles / passes
            int it = 0;
            for (int tile = blockIdx.x; tile < n_tiles && !s_abort; tile += gridDim.x) {
                for (int ps = 0; ps < npass && !s_abort; ++ps) {
                    for (int kb = 0; kb < nkb; ++kb, ++it) {
                        const int s = it % kRtStages;
                        if (it >= kRtStages && !mbar_wait(&empty[s], ((it / kRtStages) - 1) & 1, kWaitLimitNs)) {
                            set_status(p.counters, MOE_ETIMEOUT);
                            s_abort = 1;
                            break;
                        }
                        unsigned char *st = smem + s * kRtStageBytes;
                        mbar_arrive_expect_tx(&full[s], stage_tx);
                        tma_load_2d(st, &p.x, kb * kRtBK, tile * kBM, &full[s], pol);
                        tma_load_2d(st + kBM * kRtBK, &p.wr, kb * kRtBK, ps * kRtChunk, &full[s], pol);
                        tma_load_2d(st + (kBM + kRtChunk) * kRtBK, &p.g, kb * kRtBK, 0, &full[s], pol);
                    }
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            const uint32_t id_e = idesc_bf16_f32(kBM, p.nbox);
            const uint32_t id_g = idesc_bf16_f32(kBM, 16);
            int it = 0, acc_it = 0;
            for (int tile = blockIdx.x; tile < n_tiles && !s_abort; tile += gridDim.x) {
                for (int ps = 0; ps < npass && !s_abort; ++ps, ++acc_it) {
                    if (acc_it >= 1 && !mbar_wait(&acc_empty, (acc_it - 1) & 1, kWaitLimitNs)) {
                        set_status(p.counters, MOE_ETIMEOUT);
                        s_abort = 1;
                        break;
                    }
                    tc_fence_after();
                    for (int kb = 0; kb < nkb; ++kb, ++it) {
                        const int s = it % kRtStages;
                        if (!mbar_wait(&full[s], (it / kRtStages) & 1, kWaitLimitNs)) {
                            set_status(p.counters, MOE_ETIMEOUT);
                            s_abort = 1;
                            break;
                        }
                        tc_fence_after();
                        const uint32_t st = smem_u32(smem + s * kRtStageBytes);
                        const uint32_t bw = st + kBM * kRtBK, bg = st + (kBM + kRtChunk) * kRtBK;
#pragma unroll
                        for (int k4 = 0; k4 < kRtBK / 32; ++k4) {
                            const uint64_t ad = umma_desc_sw128(st + k4 * 32);
                            const uint32_t acc = (kb | k4) ? 1u : 0u;
                            umma_bf16(tmem_base, ad, umma_desc_sw128(bw + k4 * 32), id_e, acc);
                            if (ps == 0) umma_bf16(tmem_base + kRtChunk, ad, umma_desc_sw128(bg + k4 * 32), id_g, acc);
                        }
                        umma_commit(&empty[s]);
                    }
                    if (s_abort) break;
                    umma_commit(&acc_full);
                }
            }
        }
    } else {
        const int q = warp & 3;
        const int r = q * 32 + lane;
        int acc_it = 0;
        for (int tile = blockIdx.x; tile < n_tiles; tile += gridDim.x) {
            const int t = tile * kBM + r;
            uint32_t keys[KM];
            int ids[KM];
#pragma unroll
            for (int j = 0; j < KM; ++j) {
                keys[j] = 0u;
                ids[j] = 0;
            }
            float z = 0.f;
            bool ok = true;
            for (int ps = 0; ps < npass; ++ps, ++acc_it) {
                if (!mbar_wait(&acc_full, acc_it & 1, kWaitLimitNs)) {
                    set_status(p.counters, MOE_ETIMEOUT);
                    s_abort = 1;
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t tb = tmem_base + ((uint32_t)(q * 32) << 16);
                const int ncol = min(kRtChunk, p.E - ps * kRtChunk);
                for (int c0 = 0; c0 < ncol; c0 += 32) {
                    float v[32];
                    tmem_ld_32x32(tb + (uint32_t)c0, v);
                    tmem_wait_ld();
                    uint32_t kk[32];
#pragma unroll
                    for (int i = 0; i < 32; ++i) {  // keys first (independent), then the inserts
                        const int e = ps * kRtChunk + c0 + i;
                        kk[i] = (c0 + i < ncol) ? topk_key(v[i] + s_bias[min(e, p.E - 1)]) : 0u;
                    }
#pragma unroll
                    for (int i = 0; i < 32; ++i)
                        if (kk[i] > keys[KM - 1]) topk_insert<KM>(keys, ids, kk[i], ps * kRtChunk + c0 + i);
                }
                if (ps == 0) {
                    float v[32];
                    tmem_ld_32x32(tb + (uint32_t)kRtChunk, v);
                    tmem_wait_ld();
                    z = v[0];
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&acc_empty);
            }
            if (!ok) break;
            if (t < p.T) {
                const float top = (keys[0] == 1u) ? __int_as_float(0x7FC00000) : key_value(keys[0]);
                float ev[KM], sum = 0.f;
#pragma unroll
                for (int j = 0; j < KM; ++j) {
                    const float vj = (keys[j] == 1u) ? __int_as_float(0x7FC00000) : key_value(keys[j]);
                    ev[j] = (j < p.K) ? expf(vj - top) : 0.f;
                    sum += ev[j];
                }
#pragma unroll
                for (int j = 0; j < KM; ++j) {
                    if (j < p.K) {
                        p.topk_idx[(size_t)t * p.K + j] = ids[j];
                        p.topk_w[(size_t)t * p.K + j] = ev[j] / sum;
                    }
                }
                p.gsig[t] = sigmoidf_(z);
            }
            // each pair's rank within its expert: one atomic per group of lanes
            // that picked the same expert at the same rank position
            const unsigned live = __ballot_sync(0xFFFFFFFFu, t < p.T);
#pragma unroll
            for (int j = 0; j < KM; ++j) {
                if (j < p.K && t < p.T) {
                    const unsigned grp = __match_any_sync(live, ids[j]);
                    const int leader = __ffs(grp) - 1;
                    int base = 0;
                    if (lane == leader) base = atomicAdd(&p.counts[ids[j]], __popc(grp));
                    base = __shfl_sync(grp, base, leader);
                    p.rank[(size_t)t * p.K + j] = base + __popc(grp & ((1u << lane) - 1));
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, 512);
    }
}

// ------------------------------------------------------------ grouped GEMM

struct GemmParams {
    CUtensorMap a_routed;  // A rows of the routed groups (GEMM1: permuted x; GEMM2: h)
    CUtensorMap a_shared;  // A rows of the shared group (GEMM1: x in token order; GEMM2: h)
    CUtensorMap b_routed;  // 3D: (K bytes, rows, expert)
    CUtensorMap b_shared;  // 3D with one expert
    int H, E, I, Is;
    int imax;
    const int4 *mtiles;
    const float *a_scales_routed;  // [rows][K/128]
    const float *a_scales_shared;
    int a_scales_ld;               // floats per row of the A scales
    const float *w_scales;         // routed experts' scale slabs
    const float *w_scales_shared;
    uint8_t *hq;                   // GEMM1 out: [rows][2*imax] (hi | lo)
    float *hs;                     // GEMM1 out: [rows][imax/128]
    const float *slot_w;           // GEMM2: blend weight per row
    float *yslot;                  // GEMM2 out: [rows][H]
    int32_t *counters;
    int max_ntiles;
};

// Per tile facts every role needs.
struct TileInfo {
    int group, row0, rows, a_row0, nt, kdim, ntiles;
    bool shared_grp;
};

template <int MODE>
__device__ __forceinline__ bool tile_info(const GemmParams &p, int n_mtiles, int t, TileInfo &ti)
{
    const int mt = t / p.max_ntiles;
    ti.nt = t - mt * p.max_ntiles;
    if (mt >= n_mtiles) return false;
    const int4 m = __ldcg(p.mtiles + 1 + mt);
    ti.group = m.x;
    ti.row0 = m.y;
    ti.rows = m.z;
    ti.a_row0 = m.w;
    ti.shared_grp = (m.x == p.E);
    const int inter = ti.shared_grp ? p.Is : p.I;
    if (MODE == 1) {
        ti.kdim = p.H;
        ti.ntiles = inter / 128;  // one 128-column block of h per tile
    } else {
        ti.kdim = inter;
        ti.ntiles = (p.H + kBN - 1) / kBN;  // the last tile is half empty when H is an odd multiple of 128
    }
    return true;
}

// MODE 1 (GEMM1): B tile = gate rows [128 nt, +128) and up rows [inter + 128 nt, +128) of W13.
// MODE 2 (GEMM2): B tile = rows [256 nt, +256) of W2.
template <int MODE>
__global__ void __launch_bounds__(kGemmThreads, 1) gemm_kernel(const __grid_constant__ GemmParams p)
{
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    __shared__ __align__(8) uint64_t full[kGemmStages], empty[kGemmStages], acc_full[2], acc_empty[2];
    __shared__ uint32_t tmem_base_s;
    __shared__ volatile int s_abort;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    unsigned char *smem = reinterpret_cast<unsigned char *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    float *epi_scratch = reinterpret_cast<float *>(smem + kGemmStages * kStageBytes);  // [4][128] amax exchange

    if (threadIdx.x == 0) {
        s_abort = 0;
        for (int s = 0; s < kGemmStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&acc_full[b], 1);
            mbar_init(&acc_empty[b], kEpiThreads / 32);
        }
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(&tmem_base_s, kTmemCols);
        tmem_relinquish();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&p.a_routed);
        tma_prefetch_desc(&p.a_shared);
        tma_prefetch_desc(&p.b_routed);
        tma_prefetch_desc(&p.b_shared);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = tmem_base_s;

    pdl_wait();
    pdl_trigger();
    const int n_mtiles = __ldcg(p.mtiles).x;
    const int n_tiles = n_mtiles * p.max_ntiles;

    if (warp == 0) {
        // --------------------------------------------------- TMA producer
        if (lane == 0) {
            const uint64_t pol_w = policy_evict_first();  // weights stream once per M tile
            const uint64_t pol_a = policy_evict_last();   // activations are re-read for every N tile
            int it = 0;
            for (int t = blockIdx.x; t < n_tiles && !s_abort; t += gridDim.x) {
                TileInfo ti;
                if (!tile_info<MODE>(p, n_mtiles, t, ti) || ti.nt >= ti.ntiles) continue;
                const int nkb = ti.kdim / kBK;
                const CUtensorMap *amap = ti.shared_grp ? &p.a_shared : &p.a_routed;
                const CUtensorMap *bmap = ti.shared_grp ? &p.b_shared : &p.b_routed;
                const int ez = ti.shared_grp ? 0 : ti.group;
                const int inter = ti.shared_grp ? p.Is : p.I;
                // A rows: GEMM1 reads x rows (permuted rows, or token rows for the
                // shared group); GEMM2 reads h at the tile's rows of the row space.
                const int arow = MODE == 1 ? ti.a_row0 : ti.row0;
                const int lo_x = MODE == 1 ? p.H : p.imax;  // where the lo half of a row starts
                for (int kb = 0; kb < nkb; ++kb, ++it) {
                    const int s = it % kGemmStages;
                    if (it >= kGemmStages && !mbar_wait(&empty[s], ((it / kGemmStages) - 1) & 1, kWaitLimitNs)) {
                        set_status(p.counters, MOE_ETIMEOUT);
                        s_abort = 1;
                        break;
                    }
                    unsigned char *st = smem + s * kStageBytes;
                    mbar_arrive_expect_tx(&full[s], (uint32_t)kStageBytes);
                    // A: hi at x = kb*128, lo at x = kdim + kb*128 of the row
                    tma_load_2d(st, amap, kb * kBK, arow, &full[s], pol_a);
                    tma_load_2d(st + kBM * kBK, amap, lo_x + kb * kBK, arow, &full[s], pol_a);
                    unsigned char *bt = st + 2 * kBM * kBK;
                    if (MODE == 1) {
                        tma_load_3d(bt, bmap, kb * kBK, ti.nt * 128, ez, &full[s], pol_w);
                        tma_load_3d(bt + 128 * kBK, bmap, kb * kBK, inter + ti.nt * 128, ez, &full[s], pol_w);
                    } else {
                        tma_load_3d(bt, bmap, kb * kBK, ti.nt * kBN, ez, &full[s], pol_w);
                    }
                }
            }
        }
    } else if (warp == 1) {
        // --------------------------------------------------- MMA issuer
        if (lane == 0) {
            const uint32_t idesc = idesc_e4m3_f32(kBM, kBN);
            int it = 0, acc_it = 0;
            for (int t = blockIdx.x; t < n_tiles && !s_abort; t += gridDim.x) {
                TileInfo ti;
                if (!tile_info<MODE>(p, n_mtiles, t, ti) || ti.nt >= ti.ntiles) continue;
                const int nkb = ti.kdim / kBK;
                for (int kb = 0; kb < nkb; ++kb, ++it, ++acc_it) {
                    const int s = it % kGemmStages;
                    const int b = acc_it & 1;
                    if (!mbar_wait(&full[s], (it / kGemmStages) & 1, kWaitLimitNs) ||
                        (acc_it >= 2 && !mbar_wait(&acc_empty[b], ((acc_it >> 1) - 1) & 1, kWaitLimitNs))) {
                        set_status(p.counters, MOE_ETIMEOUT);
                        s_abort = 1;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t st = smem_u32(smem + s * kStageBytes);
                    const uint32_t d = tmem_base + (uint32_t)(b * kBN);
                    const uint32_t bsm = st + 2 * kBM * kBK;
#pragma unroll
                    for (int part = 0; part < 2; ++part) {  // hi, then lo
                        const uint32_t asm_ = st + part * kBM * kBK;
#pragma unroll
                        for (int k4 = 0; k4 < kBK / 32; ++k4)
                            umma_f8f6f4(d, umma_desc_sw128(asm_ + k4 * 32), umma_desc_sw128(bsm + k4 * 32), idesc,
                                        (part | k4) ? 1u : 0u);
                    }
                    umma_commit(&empty[s]);   // the stage may be refilled once these MMAs have read it
                    umma_commit(&acc_full[b]);  // the K block's partial sum is ready
                }
            }
        }
    } else {
        // --------------------------------------------------- epilogue (warps 2..17)
        // Warp w reads TMEM lanes 32 (w mod 4) .. +32 (its rows); the four warps
        // of a lane quadrant split the columns in quarters.  GEMM1: quarter j
        // holds gate columns [32 j, +32) and the matching up columns, so
        // silu(gate) * up stays in the thread; GEMM2: columns [64 j, +64).
        const int ew = warp - 2;
        const int q = warp & 3;                    // TMEM lane quadrant of this warp
        const int quarter = ew >> 2;               // column quarter
        const int r = q * 32 + lane;               // row within the tile
        unsigned char *stg = smem + kGemmStages * kStageBytes + 4096 + (size_t)ew * kStgBytes;
        int acc_it = 0;
        for (int t = blockIdx.x; t < n_tiles; t += gridDim.x) {
            TileInfo ti;
            if (!tile_info<MODE>(p, n_mtiles, t, ti) || ti.nt >= ti.ntiles) continue;
            const int nkb = ti.kdim / kBK;
            const bool valid = r < ti.rows;
            const int arow = (MODE == 1 ? ti.a_row0 : ti.row0) + r;  // row in the A tensor (and its scales)
            const float *asc = (ti.shared_grp ? p.a_scales_shared : p.a_scales_routed) + (size_t)arow * p.a_scales_ld;
            const int inter = ti.shared_grp ? p.Is : p.I;
            const float *wsc;
            int wld, wn0, wn1;  // the block-scale rows of this thread's columns (gate and up; or one)
            if (MODE == 1) {
                wsc = ti.shared_grp ? p.w_scales_shared
                                    : p.w_scales + (size_t)ti.group * ((2 * p.I / 128) * (p.H / 128) + (p.H / 128) * (p.I / 128));
                wld = p.H / 128;
                wn0 = ti.nt;                 // gate block row
                wn1 = inter / 128 + ti.nt;   // up block row
            } else {
                wsc = (ti.shared_grp ? p.w_scales_shared
                                     : p.w_scales + (size_t)ti.group * ((2 * p.I / 128) * (p.H / 128) + (p.H / 128) * (p.I / 128))) +
                      (2 * inter / 128) * (p.H / 128);
                wld = inter / 128;
                // a column quarter past H (the empty half of a last tile) keeps a
                // valid scale row; its results are not stored
                wn0 = wn1 = min(ti.nt * 2 + (quarter >> 1), p.H / 128 - 1);
            }
            float tot[64];
#pragma unroll
            for (int i = 0; i < 64; ++i) tot[i] = 0.f;
            bool ok = true;
            // the row's blend weight (GEMM2) is needed only at the tile's end: load it now
            const float w_row = (MODE == 2 && valid) ? __ldg(p.slot_w + (size_t)ti.row0 + r) : 0.f;
            // scales one K block ahead, so their loads overlap the wait for the accumulator
            float sa_n = valid ? __ldg(asc) : 0.f;
            float s0_n = __ldg(wsc + (size_t)wn0 * wld), s1_n = __ldg(wsc + (size_t)wn1 * wld);
            for (int kb = 0; kb < nkb; ++kb, ++acc_it) {
                const int b = acc_it & 1;
                const float sa = sa_n, s0 = s0_n, s1 = s1_n;
                if (kb + 1 < nkb) {
                    sa_n = valid ? __ldg(asc + kb + 1) : 0.f;
                    s0_n = __ldg(wsc + (size_t)wn0 * wld + kb + 1);
                    s1_n = __ldg(wsc + (size_t)wn1 * wld + kb + 1);
                }
                if (ok) {
                    // warp-uniform outcome: the TMEM loads below are warp-collective
                    const bool w = mbar_wait(&acc_full[b], (acc_it >> 1) & 1, kWaitLimitNs);
                    if (!__all_sync(0xFFFFFFFFu, w)) {
                        set_status(p.counters, MOE_ETIMEOUT);
                        s_abort = 1;
                        ok = false;
                    }
                }
                if (!ok) continue;
                tc_fence_after();
                const uint32_t tbase = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(b * kBN);
#pragma unroll
                for (int c = 0; c < 4; ++c) {  // 16 columns at a time
                    const int col = MODE == 1 ? ((c < 2) ? 32 * quarter + 16 * c : 128 + 32 * quarter + 16 * (c - 2))
                                              : 64 * quarter + 16 * c;
                    const float sc = sa * ((MODE == 1 && c >= 2) ? s1 : s0);
                    float v[16];
                    tmem_ld_32x16(tbase + (uint32_t)col, v);
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 16; ++i) tot[16 * c + i] = fmaf(sc, v[i], tot[16 * c + i]);
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&acc_empty[b]);
            }
            if (MODE == 1) {
                // h = silu(gate) * up for this thread's 32 columns of the block
                float amax = 0.f;
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    const float g = tot[i], u = tot[32 + i];
                    const float hv = g * __frcp_rn(1.f + __expf(-g)) * u;
                    tot[i] = hv;
                    amax = fmaxf(amax, fabsf(hv));
                }
                // the four quarters of the row's 128-column block share one scale
                named_barrier(2, kEpiThreads);
                epi_scratch[quarter * 128 + r] = amax;
                named_barrier(2, kEpiThreads);
                amax = fmaxf(fmaxf(epi_scratch[r], epi_scratch[128 + r]), fmaxf(epi_scratch[256 + r], epi_scratch[384 + r]));
                const float sc = amax > 0.f ? amax / 448.f : 1.f;
                const float inv = 1.f / sc;
                if (ok) {
                    // quantise once: hi words to the staging buffer, lo words in
                    // registers; each part leaves as 32-byte row segments, 16 bytes
                    // per lane
                    uint4 *srow = reinterpret_cast<uint4 *>(stg + lane * 48);
                    uint32_t low[8];
#pragma unroll
                    for (int i = 0; i < 2; ++i) {
                        uint32_t w4[4];
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            const int c = 16 * i + 4 * j;
                            quant4_hilo(make_float4(tot[c], tot[c + 1], tot[c + 2], tot[c + 3]), inv, w4[j], low[4 * i + j]);
                        }
                        srow[i] = make_uint4(w4[0], w4[1], w4[2], w4[3]);
                    }
                    for (int part = 0; part < 2; ++part) {
                        if (part == 1) {
                            srow[0] = make_uint4(low[0], low[1], low[2], low[3]);
                            srow[1] = make_uint4(low[4], low[5], low[6], low[7]);
                        }
                        __syncwarp();
#pragma unroll
                        for (int i = 0; i < 2; ++i) {
                            const int rr = 16 * i + (lane >> 1), ch = lane & 1;
                            const uint4 v = *reinterpret_cast<const uint4 *>(stg + rr * 48 + ch * 16);
                            if (q * 32 + rr < ti.rows) {
                                const size_t grow = (size_t)ti.row0 + q * 32 + rr;
                                *reinterpret_cast<uint4 *>(p.hq + grow * 2 * p.imax + (part ? p.imax : 0) + ti.nt * 128 +
                                                           32 * quarter + ch * 16) = v;
                            }
                        }
                        __syncwarp();
                    }
                    if (valid && quarter == 0) p.hs[((size_t)ti.row0 + r) * (p.imax / 128) + ti.nt] = sc;
                }
            } else {
                if (ok && ti.nt * kBN + 64 * quarter < p.H) {
                    // 8 columns at a time through the staging buffer (rows of 9
                    // floats), then out as 32-byte row segments, 16 bytes per lane
                    float *sf = reinterpret_cast<float *>(stg);
#pragma unroll
                    for (int c = 0; c < 8; ++c) {
#pragma unroll
                        for (int j = 0; j < 8; ++j) sf[lane * 9 + j] = w_row * tot[8 * c + j];
                        __syncwarp();
#pragma unroll
                        for (int i = 0; i < 2; ++i) {
                            const int rr = 16 * i + (lane >> 1), ch = lane & 1;
                            const float *src = sf + rr * 9 + ch * 4;
                            const float4 v = make_float4(src[0], src[1], src[2], src[3]);
                            if (q * 32 + rr < ti.rows) {
                                const size_t grow = (size_t)ti.row0 + q * 32 + rr;
                                *reinterpret_cast<float4 *>(p.yslot + grow * p.H + ti.nt * kBN + 64 * quarter + 8 * c +
                                                            4 * ch) = v;
                            }
                        }
                        __syncwarp();
                    }
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, kTmemCols);
    }
}

// ------------------------------------------------------------ narrow grouped GEMM
//
// For a few rows per expert the 128-row token tiles above are mostly padding.
// Here the roles swap: the MMA's M is 128 weight rows (one 128-row scale
// block of W13 or W2) and its N covers up to 32 rows of one group, so an item
// streams one weight block once, whatever the group's row count.  The hi and
// lo codes of the tile's rows are stacked as one 64-row B operand: one MMA
// (M = 128, N = 64, K = 32) computes both terms into neighbouring accumulator
// columns, and the weight tile is read from shared memory once per K step.
// D[weight row][token] lands in TMEM with one lane per weight row; an
// epilogue thread owns a weight row (an h column in GEMM1, an output column
// in GEMM2) for all 32 tokens and, per 128-wide K block, adds
// (activation scale x weight scale) x (hi + lo) in K-block order.  Two
// epilogue warpgroups take the items in turn, so that one group's item tail
// (GEMM1: silu, the per-row scale, quantisation and the h stores) overlaps
// the other group's accumulation.

constexpr int kNtEpiWarps = 4;                      // per group: one per TMEM lane quadrant
constexpr int kNtEpiGroups = 2;
constexpr int kNtThreads = 64 + 32 * kNtEpiWarps * kNtEpiGroups;  // warp 0: TMA, warp 1: MMA + TMEM, 2..9: epilogue
constexpr int kNtN = 2 * kNT;                       // MMA N: the tile's hi rows, then its lo rows
constexpr uint32_t kNtTmemCols = 512;
constexpr int kWB = 128;                            // weight rows per item (one scale block)
constexpr int kNtPre = kNtMaxKb * kNT / (32 * kNtEpiWarps);  // activation scales per epilogue thread and item

// An item reads two 128-row weight blocks (GEMM1: the gate block and its up
// block; GEMM2: two neighbouring W2 blocks, the second absent past H), each
// into its own accumulator: TMEM columns per buffer, and buffers.
template <int MODE>
__host__ __device__ constexpr int nt_acc_stride()
{
    return 2 * kNtN;
}
template <int MODE>
__host__ __device__ constexpr int nt_acc_bufs()
{
    return (int)kNtTmemCols / nt_acc_stride<MODE>();
}
template <int MODE>
__host__ __device__ constexpr size_t nt_stage_bytes()
{
    return 2 * (size_t)kWB * kBK + 2 * (size_t)kNT * kBK;  // two weight blocks, then the rows' hi and lo codes
}
template <int MODE>
__host__ __device__ constexpr int nt_stages()
{
    return 5;
}
template <int MODE>
__host__ __device__ constexpr size_t nt_smem()
{
    return nt_stages<MODE>() * nt_stage_bytes<MODE>() + 1024;
}

struct NtItem {
    int group, row0, rows, a_row0, nb, kdim, inter;
    bool shared_grp;
};

// Item t = (group tile t / max_ntiles, weight block t % max_ntiles).
template <int MODE>
__device__ __forceinline__ bool nt_item(const GemmParams &p, int n_mtiles, int t, NtItem &ti)
{
    const int mt = t / p.max_ntiles;
    ti.nb = t - mt * p.max_ntiles;
    if (mt >= n_mtiles) return false;
    const int4 m = __ldcg(p.mtiles + 1 + mt);
    ti.group = m.x;
    ti.row0 = m.y;
    ti.rows = m.z;
    ti.a_row0 = m.w;
    ti.shared_grp = (m.x == p.E);
    ti.inter = ti.shared_grp ? p.Is : p.I;
    if (MODE == 1) {
        ti.kdim = p.H;
        return ti.nb < ti.inter / kWB;  // 128-column blocks of h
    }
    ti.kdim = ti.inter;
    return true;                        // max_ntiles = (H / 128 + 1) / 2 pairs of output blocks
}

// Weight blocks of an item: GEMM1 two (gate, up); GEMM2 two, or one for the
// last pair when H / 128 is odd.
template <int MODE>
__device__ __forceinline__ int nt_blocks(const GemmParams &p, const NtItem &ti)
{
    return MODE == 1 ? 2 : min(2, p.H / kWB - 2 * ti.nb);
}

// The first valid item at or after t, in steps of the grid (n_items if none).
template <int MODE>
__device__ __forceinline__ int nt_next(const GemmParams &p, int n_mtiles, int n_items, int t, NtItem &ti)
{
    while (t < n_items && !nt_item<MODE>(p, n_mtiles, t, ti)) t += gridDim.x;
    return t;
}

// One epilogue thread's share of an item's scale tables (activation scales
// [K block][row], the two weight-scale rows, GEMM2's blend weights), loaded
// into registers while the previous item is computed.
struct NtPre {
    float sx[kNtPre];
    float sw, wr;
};

template <int MODE>
__device__ __forceinline__ void nt_prefetch(const GemmParams &p, const NtItem &ti, int et, NtPre &pr)
{
    const int nkb = ti.kdim / kBK;
    const int arow0 = MODE == 1 ? ti.a_row0 : ti.row0;
    const float *asc = (ti.shared_grp ? p.a_scales_shared : p.a_scales_routed) + (size_t)arow0 * p.a_scales_ld;
    const float *wsc = ti.shared_grp
                           ? p.w_scales_shared
                           : p.w_scales + (size_t)ti.group * ((2 * p.I / 128) * (p.H / 128) + (p.H / 128) * (p.I / 128));
    int wld, wn0, wn1;
    if (MODE == 1) {
        wld = p.H / 128;
        wn0 = ti.nb;                    // gate block row
        wn1 = ti.inter / 128 + ti.nb;   // up block row
    } else {
        wsc += (size_t)(2 * ti.inter / 128) * (p.H / 128);
        wld = ti.inter / 128;
        wn0 = 2 * ti.nb;                              // the pair's output blocks
        wn1 = min(2 * ti.nb + 1, p.H / 128 - 1);      // (a valid row when the second is absent)
    }
    const int j = et % kNT;  // this thread's row of the table
#pragma unroll
    for (int m = 0; m < kNtPre; ++m) {
        const int kb = (et + 32 * kNtEpiWarps * m) / kNT;
        pr.sx[m] = (kb < nkb && j < ti.rows) ? __ldg(asc + (size_t)j * p.a_scales_ld + kb) : 0.f;
    }
    pr.sw = et < nkb ? __ldg(wsc + (size_t)wn0 * wld + et)
                     : (et < 2 * nkb ? __ldg(wsc + (size_t)wn1 * wld + et - nkb) : 0.f);
    pr.wr = (MODE == 2 && et < ti.rows) ? __ldg(p.slot_w + (size_t)ti.row0 + et) : 0.f;
}

// MODE 1: item = h columns [128 nb, +128) of up to 32 rows: W13 gate rows
// [128 nb, +128) and up rows [inter + 128 nb, +128) against x; epilogue
// h = silu(gate) * up, quantised to hi/lo e4m3 with one scale per (row, 128
// block), in the layout gemm_kernel<1> writes.  MODE 2: item = output
// columns [256 nb, +256): W2 rows against h; epilogue x the row's blend
// weight into its partial row.
template <int MODE>
__global__ void __launch_bounds__(kNtThreads, 1) gemm_nt_kernel(const __grid_constant__ GemmParams p)
{
    constexpr int kStages = nt_stages<MODE>();
    constexpr uint32_t kSt = (uint32_t)nt_stage_bytes<MODE>();
    constexpr uint32_t kAB = 2 * kWB * kBK;  // weight bytes of a stage (two blocks)
    constexpr int kAccStride = nt_acc_stride<MODE>(), kAccBufs = nt_acc_bufs<MODE>();
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    __shared__ __align__(8) uint64_t full[kStages], empty[kStages], acc_full[kAccBufs], acc_empty[kAccBufs];
    // phase s completes once the group owning item s has received all of
    // its accumulators; the owner of item s + 1 waits for it before its
    // first accumulator wait, so no waiter on acc_full runs more than one
    // phase ahead of the barrier (a parity wait two phases ahead would pass
    // at once)
    __shared__ __align__(8) uint64_t handoff;
    __shared__ uint32_t tmem_base_s;
    __shared__ volatile int s_abort;
    // per epilogue group: the item's tables and staging
    __shared__ __align__(16) float s_sx[kNtEpiGroups][kNtMaxKb * kNT];  // [kb][row]: activation scales
    __shared__ float s_sw[kNtEpiGroups][2 * kNtMaxKb];                  // weight scales: gate row, up row
    __shared__ float s_wrow[kNtEpiGroups][MODE == 2 ? kNT : 1];         // GEMM2: blend weight per row
    __shared__ float s_inv[kNtEpiGroups][kNT], s_scl[kNtEpiGroups][kNT];
    // GEMM1: h codes (hi, lo) staged for row stores; its first 512 bytes
    // also carry the per-warp |h| maxima, which are read before the codes
    // are written
    __shared__ __align__(16) uint8_t s_hq[kNtEpiGroups][2][kNT][kWB];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    unsigned char *smem = reinterpret_cast<unsigned char *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);

    if (threadIdx.x == 0) {
        s_abort = 0;
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < kAccBufs; ++b) {
            mbar_init(&acc_full[b], 1);
            mbar_init(&acc_empty[b], kNtEpiWarps);  // the four warps of the group that owns the item
        }
        mbar_init(&handoff, kNtEpiWarps);
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(&tmem_base_s, kNtTmemCols);
        tmem_relinquish();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&p.a_routed);
        tma_prefetch_desc(&p.a_shared);
        tma_prefetch_desc(&p.b_routed);
        tma_prefetch_desc(&p.b_shared);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = tmem_base_s;

    pdl_wait();
    pdl_trigger();
    const int n_mtiles = __ldcg(p.mtiles).x;
    const int n_items = n_mtiles * p.max_ntiles;

    if (warp == 0) {
        // --------------------------------------------------- TMA producer
        if (lane == 0) {
            const uint64_t pol_w = policy_evict_first();  // each weight block streams once per group tile
            const uint64_t pol_a = policy_evict_last();   // a tile's rows are read for every weight block
            int it = 0;
            for (int t = blockIdx.x; t < n_items && !s_abort; t += gridDim.x) {
                NtItem ti;
                if (!nt_item<MODE>(p, n_mtiles, t, ti)) continue;
                const int nkb = ti.kdim / kBK;
                const CUtensorMap *amap = ti.shared_grp ? &p.a_shared : &p.a_routed;
                const CUtensorMap *wmap = ti.shared_grp ? &p.b_shared : &p.b_routed;
                const int ez = ti.shared_grp ? 0 : ti.group;
                const int arow = MODE == 1 ? ti.a_row0 : ti.row0;
                const int lo_x = MODE == 1 ? p.H : p.imax;  // where the lo half of an activation row starts
                const int nblk = nt_blocks<MODE>(p, ti);
                // weight rows of the two blocks: gate and up (GEMM1), or a pair of W2 blocks
                const int y0 = MODE == 1 ? ti.nb * kWB : 2 * ti.nb * kWB;
                const int y1 = MODE == 1 ? ti.inter + ti.nb * kWB : y0 + kWB;
                for (int kb = 0; kb < nkb; ++kb, ++it) {
                    const int s = it % kStages;
                    if (it >= kStages && !mbar_wait(&empty[s], ((it / kStages) - 1) & 1, kWaitLimitNs)) {
                        set_status(p.counters, MOE_ETIMEOUT);
                        s_abort = 1;
                        break;
                    }
                    unsigned char *st = smem + (size_t)s * kSt;
                    mbar_arrive_expect_tx(&full[s], kSt - (2 - nblk) * kWB * kBK);
                    tma_load_3d(st, wmap, kb * kBK, y0, ez, &full[s], pol_w);
                    if (nblk == 2) tma_load_3d(st + kWB * kBK, wmap, kb * kBK, y1, ez, &full[s], pol_w);
                    // hi rows, then lo rows: together the 64-row B operand
                    tma_load_2d(st + kAB, amap, kb * kBK, arow, &full[s], pol_a);
                    tma_load_2d(st + kAB + kNT * kBK, amap, lo_x + kb * kBK, arow, &full[s], pol_a);
                }
            }
        }
    } else if (warp == 1) {
        // --------------------------------------------------- MMA issuer
        if (lane == 0) {
            const uint32_t idesc = idesc_e4m3_f32(kWB, kNtN);
            int it = 0, acc_it = 0;
            for (int t = blockIdx.x; t < n_items && !s_abort; t += gridDim.x) {
                NtItem ti;
                if (!nt_item<MODE>(p, n_mtiles, t, ti)) continue;
                const int nkb = ti.kdim / kBK;
                const int nblk = nt_blocks<MODE>(p, ti);
                for (int kb = 0; kb < nkb; ++kb, ++it, ++acc_it) {
                    const int s = it % kStages;
                    const int b = acc_it % kAccBufs;
                    if (!mbar_wait(&full[s], (it / kStages) & 1, kWaitLimitNs) ||
                        (acc_it >= kAccBufs && !mbar_wait(&acc_empty[b], ((acc_it / kAccBufs) - 1) & 1, kWaitLimitNs))) {
                        set_status(p.counters, MOE_ETIMEOUT);
                        s_abort = 1;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t st = smem_u32(smem + (size_t)s * kSt);
                    const uint32_t bsm = st + kAB;
                    const uint32_t d = tmem_base + (uint32_t)(b * kAccStride);
#pragma unroll
                    for (int k4 = 0; k4 < kBK / 32; ++k4) {
                        const uint32_t acc = k4 ? 1u : 0u;
                        umma_f8f6f4(d, umma_desc_sw128(st + k4 * 32), umma_desc_sw128(bsm + k4 * 32), idesc, acc);
                        if (nblk == 2)
                            umma_f8f6f4(d + kNtN, umma_desc_sw128(st + kWB * kBK + k4 * 32), umma_desc_sw128(bsm + k4 * 32),
                                        idesc, acc);
                    }
                    umma_commit(&empty[s]);
                    umma_commit(&acc_full[b]);
                }
            }
        }
    } else {
        // --------------------------------------------------- epilogue (warps 2..9)
        // Group eg takes the items at even (eg = 0) or odd (eg = 1) places of
        // this CTA's sequence and skips the other group's K blocks.
        const int eg = (warp - 2) / kNtEpiWarps;
        const int q = warp & 3;        // TMEM lane quadrant
        const int r = q * 32 + lane;   // weight row within the block
        const int et = (warp - 2 - eg * kNtEpiWarps) * 32 + lane;
        const int bar = 1 + eg;        // the group's named barrier
        constexpr int kGT = 32 * kNtEpiWarps;
        float *sx_tab = s_sx[eg];
        float *sw_tab = s_sw[eg];
        float(*amax_tab)[kNT] = reinterpret_cast<float(*)[kNT]>(&s_hq[eg][0][0][0]);
        int acc_it = 0;
        int seq = eg;  // place of `cur` in this CTA's item sequence
        bool ok = true;
        NtItem cur;
        int t = nt_next<MODE>(p, n_mtiles, n_items, blockIdx.x, cur);
        if (eg == 1 && t < n_items) {
            acc_it += cur.kdim / kBK;
            t = nt_next<MODE>(p, n_mtiles, n_items, t + gridDim.x, cur);
        }
        NtPre pre;
        if (t < n_items) nt_prefetch<MODE>(p, cur, et, pre);
        while (t < n_items) {
            // the other group's item, then this group's next one
            NtItem mid, nxt;
            const int tm = nt_next<MODE>(p, n_mtiles, n_items, t + gridDim.x, mid);
            const int tn = tm < n_items ? nt_next<MODE>(p, n_mtiles, n_items, tm + gridDim.x, nxt) : n_items;
            const int nkb = cur.kdim / kBK;
            // the item's scale tables into shared memory, then the next item's loads
            named_barrier(bar, kGT);
#pragma unroll
            for (int m = 0; m < kNtPre; ++m) {
                const int i = et + kGT * m;
                if (i < nkb * kNT) sx_tab[i] = pre.sx[m];
            }
            if (et < 2 * nkb) sw_tab[et] = pre.sw;
            if (MODE == 2 && et < kNT) s_wrow[eg][et] = pre.wr;
            named_barrier(bar, kGT);
            if (tn < n_items) nt_prefetch<MODE>(p, nxt, et, pre);

            float g[kNT], u[kNT];  // the two blocks' sums
#pragma unroll
            for (int j = 0; j < kNT; ++j) g[j] = u[j] = 0.f;
            if (ok && seq > 0) {
                const bool w = mbar_wait(&handoff, (seq - 1) & 1, kWaitLimitNs);
                if (!__all_sync(0xFFFFFFFFu, w)) {
                    set_status(p.counters, MOE_ETIMEOUT);
                    s_abort = 1;
                    ok = false;
                }
            }
            for (int kb = 0; kb < nkb; ++kb, ++acc_it) {
                const int b = acc_it % kAccBufs;
                if (ok) {
                    const bool w = mbar_wait(&acc_full[b], (acc_it / kAccBufs) & 1, kWaitLimitNs);
                    if (!__all_sync(0xFFFFFFFFu, w)) {
                        set_status(p.counters, MOE_ETIMEOUT);
                        s_abort = 1;
                        ok = false;
                    }
                }
                if (!ok) continue;
                tc_fence_after();
                const uint32_t tb = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(b * kAccStride);
                const float sw0 = sw_tab[kb], sw1 = sw_tab[nkb + kb];
                const float4 *sx4 = reinterpret_cast<const float4 *>(sx_tab + kb * kNT);
                // the two blocks' accumulators (GEMM1 gate and up; GEMM2 the pair
                // of output blocks), 8 rows at a time
#pragma unroll
                for (int h = 0; h < kNT / 8; ++h) {  // rows [8 h, +8)
                    float gh[8], gl[8], uh[8], ul[8];
                    tmem_ld_32x8(tb + 8 * h, gh);
                    tmem_ld_32x8(tb + kNT + 8 * h, gl);
                    tmem_ld_32x8(tb + kNtN + 8 * h, uh);
                    tmem_ld_32x8(tb + kNtN + kNT + 8 * h, ul);
                    tmem_wait_ld();
#pragma unroll
                    for (int j4 = 0; j4 < 2; ++j4) {
                        const float4 sx = sx4[2 * h + j4];
                        const float sxa[4] = {sx.x, sx.y, sx.z, sx.w};
#pragma unroll
                        for (int c = 0; c < 4; ++c) {
                            const int i = 4 * j4 + c, j = 8 * h + i;
                            g[j] = fmaf(sxa[c] * sw0, gh[i] + gl[i], g[j]);
                            u[j] = fmaf(sxa[c] * sw1, uh[i] + ul[i], u[j]);
                        }
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&acc_empty[b]);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&handoff);  // this item's accumulators are all received
            if (MODE == 1) {
                // h = silu(gate) * up; the 128 columns of the block share one
                // scale per row: max |h| over the warp by recursive halving
                // (lane j ends with row j's maximum), then over the 4 warps
                float m[kNT];
#pragma unroll
                for (int j = 0; j < kNT; ++j) {
                    const float hv = g[j] * __frcp_rn(1.f + __expf(-g[j])) * u[j];
                    g[j] = hv;
                    m[j] = fabsf(hv);
                }
#pragma unroll
                for (int w = kNT / 2; w >= 1; w >>= 1) {
                    const bool upper = (lane & w) != 0;
#pragma unroll
                    for (int i = 0; i < w; ++i) {
                        const float send = upper ? m[i] : m[i + w];
                        const float keep = upper ? m[i + w] : m[i];
                        m[i] = fmaxf(keep, __shfl_xor_sync(0xFFFFFFFFu, send, w));
                    }
                }
                amax_tab[q][lane] = m[0];
                named_barrier(bar, kGT);
                if (q == 0) {
                    const float a = fmaxf(fmaxf(amax_tab[0][lane], amax_tab[1][lane]),
                                          fmaxf(amax_tab[2][lane], amax_tab[3][lane]));
                    const float sc = a > 0.f ? a / 448.f : 1.f;
                    s_scl[eg][lane] = sc;
                    s_inv[eg][lane] = 1.f / sc;
                }
                named_barrier(bar, kGT);
#pragma unroll
                for (int j = 0; j < kNT; j += 2) {
                    const float a = g[j] * s_inv[eg][j], c = g[j + 1] * s_inv[eg][j + 1];
                    const uint16_t hh = f32x2_to_e4m3x2(a, c);
                    const float2 f = e4m3x2_to_f32x2(hh);
                    const uint16_t ll = f32x2_to_e4m3x2(a - f.x, c - f.y);
                    s_hq[eg][0][j][r] = (uint8_t)(hh & 0xFF);
                    s_hq[eg][0][j + 1][r] = (uint8_t)(hh >> 8);
                    s_hq[eg][1][j][r] = (uint8_t)(ll & 0xFF);
                    s_hq[eg][1][j + 1][r] = (uint8_t)(ll >> 8);
                }
                named_barrier(bar, kGT);
                // rows of 128 codes out as 16-byte pieces
                for (int i = et; i < 2 * kNT * (kWB / 16); i += kGT) {
                    const int part = i / (kNT * (kWB / 16));
                    const int j = (i / (kWB / 16)) % kNT, ch = i % (kWB / 16);
                    if (j < cur.rows)
                        *reinterpret_cast<uint4 *>(p.hq + ((size_t)cur.row0 + j) * 2 * p.imax + (part ? p.imax : 0) +
                                                   cur.nb * kWB + ch * 16) =
                            *reinterpret_cast<const uint4 *>(&s_hq[eg][part][j][ch * 16]);
                }
                if (q == 0 && lane < cur.rows) p.hs[((size_t)cur.row0 + lane) * (p.imax / 128) + cur.nb] = s_scl[eg][lane];
            } else if (ok) {
                // a warp stores 32 consecutive floats of each row's partial row, per block
                const bool two = nt_blocks<MODE>(p, cur) == 2;
                float *dst = p.yslot + (size_t)cur.row0 * p.H + 2 * cur.nb * kWB + r;
#pragma unroll
                for (int j = 0; j < kNT; ++j) {
                    if (j < cur.rows) {
                        dst[(size_t)j * p.H] = s_wrow[eg][j] * g[j];
                        if (two) dst[(size_t)j * p.H + kWB] = s_wrow[eg][j] * u[j];
                    }
                }
            }
            if (tm < n_items) acc_it += mid.kdim / kBK;  // the other group's K blocks
            seq += 2;
            t = tn;
            cur = nxt;
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, kNtTmemCols);
    }
}

// ------------------------------------------------------------ blend

struct BlendParams {
    int T, K, H;
    const int32_t *pos;
    const float *yslot;
    const uint16_t *residual;
    uint16_t *out;
};

// out[t] = sum_r yslot[pos(t, r)] (rank order) + yslot[T*K + t] (+ residual)
__global__ void __launch_bounds__(256) blend_kernel(BlendParams p)
{
    pdl_wait();
    pdl_trigger();
    const int nv = p.H / 4;
    const size_t total = (size_t)p.T * nv;
    for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < total; i += (size_t)gridDim.x * blockDim.x) {
        const int t = (int)(i / nv), c = (int)(i - (size_t)t * nv);
        float4 a = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int r = 0; r < p.K; ++r) {
            const float4 v = __ldcg(reinterpret_cast<const float4 *>(p.yslot + (size_t)p.pos[t * p.K + r] * p.H) + c);
            a.x += v.x; a.y += v.y; a.z += v.z; a.w += v.w;
        }
        const float4 s = __ldcg(reinterpret_cast<const float4 *>(p.yslot + ((size_t)p.T * p.K + t) * p.H) + c);
        a.x += s.x; a.y += s.y; a.z += s.z; a.w += s.w;
        if (p.residual) {
            const uint2 rv = reinterpret_cast<const uint2 *>(p.residual + (size_t)t * p.H)[c];
            a.x += bf16_lo(rv.x); a.y += bf16_hi(rv.x); a.z += bf16_lo(rv.y); a.w += bf16_hi(rv.y);
        }
        uint2 o;
        o.x = (uint32_t)f32_to_bf16_bits(a.x) | ((uint32_t)f32_to_bf16_bits(a.y) << 16);
        o.y = (uint32_t)f32_to_bf16_bits(a.z) | ((uint32_t)f32_to_bf16_bits(a.w) << 16);
        reinterpret_cast<uint2 *>(p.out + (size_t)t * p.H)[c] = o;
    }
}

// ------------------------------------------------------------ host side

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn()
{
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(f);
    });
    return fn;
}

// A byte tensor [outer][rows][inner] (inner contiguous) as a TMA map with
// 128-byte-swizzled boxes of [128 bytes, box_rows, 1].
bool make_map(CUtensorMap *m, const void *base, uint64_t inner, uint64_t rows, uint64_t outer, uint64_t row_stride,
              uint64_t outer_stride, uint32_t box_rows)
{
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[3] = {inner, rows, outer};
    const cuuint64_t strides[2] = {row_stride, outer_stride};
    const cuuint32_t box[3] = {128, box_rows, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    const cuuint32_t rank = outer > 1 || outer_stride ? 3 : 2;
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, rank, const_cast<void *>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

namespace {

template <typename P>
int gemm_occupancy_once(void (*kernel)(P), size_t smem = kGemmSmem)
{
    static std::mutex mu;
    static std::vector<std::pair<const void *, int>> done;
    int dev = 0;
    cudaGetDevice(&dev);
    std::lock_guard<std::mutex> lk(mu);
    for (auto &d : done)
        if (d.first == (const void *)kernel && d.second == dev) return 1;
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
        return 0;
    done.push_back({(const void *)kernel, dev});
    return 1;
}

template <int KM>
cudaError_t launch_router_tc(unsigned grid, const RouterTcParams &rp, cudaStream_t s)
{
    if (!gemm_occupancy_once(router_tc_kernel<KM>, kRtSmem)) return cudaErrorInvalidValue;
    return launch_kernel(router_tc_kernel<KM>, dim3(grid), dim3(kRtThreads), kRtSmem, s, rp);
}

}  // namespace

int prefill_forward(const moe_dims &d, const uint16_t *x, int32_t rows, const uint16_t *router_w,
                    const uint8_t *expert_w8, const float *expert_scales, const uint8_t *shared_w8,
                    const float *shared_scales, const uint16_t *shared_gate, uint16_t *out,
                    const uint16_t *residual, const float *router_bias, void *ws, cudaStream_t s,
                    int32_t *topk_idx_out, float *topk_w_out, float *gsig_out, bool narrow)
{
    const int T = rows, E = d.n_experts, K = d.top_k, H = d.hidden, I = d.inter, Is = d.shared_inter;
    const int imax = std::max(I, Is);
    if (H % kBK) return MOE_EUNSUPPORTED;
    if (narrow && !narrow_supported(d)) return MOE_EUNSUPPORTED;
    const PrefillLayout L = prefill_layout(d, T);
    char *base = static_cast<char *>(ws);
    int32_t *counters = reinterpret_cast<int32_t *>(base + L.counters);
    int32_t *tidx = topk_idx_out ? topk_idx_out : reinterpret_cast<int32_t *>(base + L.topk_idx);
    float *tw = topk_w_out ? topk_w_out : reinterpret_cast<float *>(base + L.topk_w);
    float *gs = gsig_out ? gsig_out : reinterpret_cast<float *>(base + L.gsig);
    const DeviceInfo &di = device_info();
    const int P = T * K;

    // few rows: the decode router over many CTAs; else the tcgen05 router,
    // which also counts each expert's rows
    const bool small_router = T <= kSmallRouterRows;
    cudaError_t e = cudaSuccess;
    if (!small_router && (e = cudaMemsetAsync(base + L.counts, 0, sizeof(int32_t) * (E + 1), s)) != cudaSuccess)
        return MOE_ECUDA;

    PlanParams pp;
    pp.T = T;
    pp.E = E;
    pp.K = K;
    pp.H = H;
    pp.I = I;
    pp.Is = Is;
    pp.topk_idx = tidx;
    pp.topk_w = tw;
    pp.gsig = gs;
    pp.counts = reinterpret_cast<int32_t *>(base + L.counts);
    pp.offsets = reinterpret_cast<int32_t *>(base + L.offsets);
    pp.rank = reinterpret_cast<int32_t *>(base + L.rank);
    pp.pos = reinterpret_cast<int32_t *>(base + L.pos);
    pp.mtiles = reinterpret_cast<int4 *>(base + L.mtiles);
    pp.tile_rows = narrow ? kNT : kBM;
    pp.count_in_scan = small_router ? 1 : 0;
    pp.x = x;
    pp.xp_shared0 = std::max(P, kBM);
    pp.xp = reinterpret_cast<uint8_t *>(base + L.xp);
    pp.xps = reinterpret_cast<float *>(base + L.xps);
    pp.slot_w = reinterpret_cast<float *>(base + L.slot_w);
    pp.counters = counters;

    // 1. router + top-k (+ per-expert ranks)
    if (small_router) {
        RouterLaunch ra{};
        ra.d = &d;
        ra.x = x;
        ra.rows = T;
        ra.router_w = router_w;
        ra.router_bias = router_bias;
        ra.shared_gate = shared_gate;
        ra.topk_idx = tidx;
        ra.topk_w = tw;
        ra.gsig = gs;
        ra.logits = reinterpret_cast<float *>(base + L.logits);
        ra.counters = counters;
        if (launch_router_topk(ra, s) != cudaSuccess) return MOE_ECUDA;
    } else {
        RouterTcParams rp{};
        rp.T = T;
        rp.E = E;
        rp.K = K;
        rp.H = H;
        rp.nbox = std::min(kRtChunk, (E + 15) / 16 * 16);
        rp.bias = router_bias;
        rp.topk_idx = tidx;
        rp.topk_w = tw;
        rp.gsig = gs;
        rp.counts = pp.counts;
        rp.rank = pp.rank;
        rp.counters = counters;
        if (!make_map(&rp.x, x, 2 * (uint64_t)H, (uint64_t)T, 1, 2 * (uint64_t)H, 0, kBM) ||
            !make_map(&rp.wr, router_w, 2 * (uint64_t)H, (uint64_t)E, 1, 2 * (uint64_t)H, 0, (uint32_t)rp.nbox) ||
            !make_map(&rp.g, shared_gate, 2 * (uint64_t)H, 1, 1, 2 * (uint64_t)H, 0, 16))
            return MOE_ECUDA;
        const unsigned rt_grid = (unsigned)std::min<int64_t>(di.sm_count, (T + kBM - 1) / kBM);
        if (K <= 2) e = launch_router_tc<2>(rt_grid, rp, s);
        else if (K <= 4) e = launch_router_tc<4>(rt_grid, rp, s);
        else if (K <= 8) e = launch_router_tc<8>(rt_grid, rp, s);
        else if (K <= 16) e = launch_router_tc<16>(rt_grid, rp, s);
        else e = launch_router_tc<32>(rt_grid, rp, s);
        if (e != cudaSuccess) return MOE_ECUDA;
    }

    // 2, 3
    if ((e = launch_kernel(scan_kernel, dim3(1), dim3(1024), 0, s, pp)) != cudaSuccess) return MOE_ECUDA;
    // few tokens: a warp per destination row, so that ~32 warps per SM write
    pp.perm_split = T >= 1024 ? 1 : std::min(K + 1, std::max(1, (32 * di.sm_count + T - 1) / T));
    const int perm_warps = T * pp.perm_split;
    if ((e = launch_kernel(permute_kernel, dim3(std::max(1, std::min(8 * di.sm_count, (perm_warps + 7) / 8))),
                           dim3(256), 0, s, pp)) != cudaSuccess)
        return MOE_ECUDA;

    // 4. GEMM1
    GemmParams g{};
    g.H = H;
    g.E = E;
    g.I = I;
    g.Is = Is;
    g.imax = imax;
    g.mtiles = pp.mtiles;
    g.w_scales = expert_scales;
    g.w_scales_shared = shared_scales;
    g.hq = reinterpret_cast<uint8_t *>(base + L.hq);
    g.hs = reinterpret_cast<float *>(base + L.hs);
    g.slot_w = pp.slot_w;
    g.yslot = reinterpret_cast<float *>(base + L.yslot);
    g.counters = counters;
    const int64_t R = L.rows_total;
    // A tensors are declared with at least 128 rows (their buffers are that
    // large); rows past the valid ones are read but never stored.  The narrow
    // GEMMs read activation boxes of kNT rows.
    const uint32_t abox = narrow ? kNT : kBM;
    bool ok = make_map(&g.a_routed, pp.xp, 2 * (uint64_t)H, (uint64_t)std::max<int64_t>(L.routed, kBM), 1,
                       2 * (uint64_t)H, 0, abox) &&
              make_map(&g.a_shared, pp.xp + (size_t)pp.xp_shared0 * 2 * H, 2 * (uint64_t)H,
                       (uint64_t)std::max(T, kBM), 1, 2 * (uint64_t)H, 0, abox) &&
              make_map(&g.b_routed, expert_w8, (uint64_t)H, 2 * (uint64_t)I, (uint64_t)E, (uint64_t)H,
                       3 * (uint64_t)I * H, 128) &&
              make_map(&g.b_shared, shared_w8, (uint64_t)H, 2 * (uint64_t)Is, 1, (uint64_t)H, 3 * (uint64_t)Is * H, 128);
    if (!ok) return MOE_ECUDA;
    g.a_scales_routed = pp.xps;
    g.a_scales_shared = pp.xps + (size_t)P * (H / 128);
    g.a_scales_ld = H / 128;
    g.max_ntiles = imax / 128;
    if (narrow) {
        if (!gemm_occupancy_once(gemm_nt_kernel<1>, nt_smem<1>()) ||
            !gemm_occupancy_once(gemm_nt_kernel<2>, nt_smem<2>()))
            return MOE_ECUDA;
        e = launch_kernel(gemm_nt_kernel<1>, dim3(di.sm_count), dim3(kNtThreads), nt_smem<1>(), s, g);
    } else {
        if (!gemm_occupancy_once(gemm_kernel<1>) || !gemm_occupancy_once(gemm_kernel<2>)) return MOE_ECUDA;
        e = launch_kernel(gemm_kernel<1>, dim3(di.sm_count), dim3(kGemmThreads), kGemmSmem, s, g);
    }
    if (e != cudaSuccess) return MOE_ECUDA;

    // 5. GEMM2
    GemmParams g2 = g;
    const uint64_t Rp = (uint64_t)std::max<int64_t>(R, kBM);
    const uint32_t wbox = narrow ? kWB : kBN;  // W2 rows per box: one 128-row block, or a 256-column tile
    ok = make_map(&g2.a_routed, g.hq, 2 * (uint64_t)imax, Rp, 1, 2 * (uint64_t)imax, 0, abox) &&
         make_map(&g2.a_shared, g.hq, 2 * (uint64_t)imax, Rp, 1, 2 * (uint64_t)imax, 0, abox) &&
         make_map(&g2.b_routed, expert_w8 + (size_t)2 * I * H, (uint64_t)I, (uint64_t)H, (uint64_t)E, (uint64_t)I,
                  3 * (uint64_t)I * H, wbox) &&
         make_map(&g2.b_shared, shared_w8 + (size_t)2 * Is * H, (uint64_t)Is, (uint64_t)H, 1, (uint64_t)Is,
                  3 * (uint64_t)Is * H, wbox);
    if (!ok) return MOE_ECUDA;
    g2.a_scales_routed = g.hs;
    g2.a_scales_shared = g.hs;
    g2.a_scales_ld = imax / 128;
    if (narrow) {
        g2.max_ntiles = (H / kWB + 1) / 2;  // pairs of 128-row W2 blocks
        e = launch_kernel(gemm_nt_kernel<2>, dim3(di.sm_count), dim3(kNtThreads), nt_smem<2>(), s, g2);
    } else {
        g2.max_ntiles = (H + kBN - 1) / kBN;
        e = launch_kernel(gemm_kernel<2>, dim3(di.sm_count), dim3(kGemmThreads), kGemmSmem, s, g2);
    }
    if (e != cudaSuccess) return MOE_ECUDA;

    // 6. blend
    BlendParams bp;
    bp.T = T;
    bp.K = K;
    bp.H = H;
    bp.pos = pp.pos;
    bp.yslot = g.yslot;
    bp.residual = residual;
    bp.out = out;
    const size_t work = (size_t)T * (H / 4);
    if ((e = launch_kernel(blend_kernel, dim3((unsigned)std::min<size_t>(8 * di.sm_count, (work + 255) / 256)),
                           dim3(256), 0, s, bp)) != cudaSuccess)
        return MOE_ECUDA;
    return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ECUDA;
}

}  // namespace moe
