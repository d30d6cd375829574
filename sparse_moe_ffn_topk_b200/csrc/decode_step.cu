// decode_step.cu -- the decode step (up to kStepMaxRows rows) as one
// persistent kernel, at the arithmetic the pages give for this path.
//
// The pages' decode chain ("Qwen3.6-35B-A3B-FP8 on NVIDIA GB10" blueprint
// page, Kernels table) is a router GEMV, a top-k softmax, the FP8 gate/up
// product with the shared expert fused, SiLU and the down product, and a
// weighted blend; its Precision table reads the fp8 block128x128 weights
// against bf16 activations for gate/up and against f32 activations for down.
// The "colibri #1992" PR page gives the decode GEMV's shape: a warp per
// output row, 16 bytes a lane, the activation in shared memory.
//
// Here one CTA per SM (eight consumer warps and a producer warp that keeps a
// ring of 16 KB shared-memory slots filled by TMA) runs the whole step with
// no grid-wide barrier: CTAs wait only for the data they read (tagged
// logits, per-expert unit counts):
//
//   P0  (before the programmatic-dependent-launch wait: weights only)
//       the producer starts the copies of this CTA's router rows and of its
//       shared-expert gate/up rows;
//   P1  x -> shared memory (bf16, and as three e5m2 terms per value with one
//       power-of-two scale per (row, 128 block): the gate/up MMAs' B
//       operand); the CTA's router rows (and the gate vector) against bf16 x
//       in fp32 -> logits in the workspace, each with the call's tag in the
//       same 8-byte word;
//   P2  every CTA takes the top-k of every row from the logits as their
//       tagged words arrive (two stages over all warps; no CTA waits for a
//       designated one, nor for the others beyond their logits), builds the same
//       list of distinct experts, and runs its share of gate/up units (32
//       gate + 32 up rows of one expert) on tcgen05: A = the e4m3 weight rows
//       from the ring, B = the x terms, fp32 accumulators in tensor memory;
//       the epilogue writes h = silu(gate) * up to the workspace as eight
//       e5m2 terms per value (one power of two per 32 values, laid out as
//       the down MMAs' B registers) and counts the unit for its expert;
//   P3  no grid barrier: each down item (one expert, this CTA's one
//       or two 8-row output tiles, the full K) waits until its expert's
//       units are all counted, bulk-copies the expert's h terms, and runs
//       mma.sync m16n8k32 (A = the weight rows through ldmatrix, B = the h
//       terms); then the blend in rank order (+ shared expert * sigmoid
//       gate, + residual), one rounding to bf16.
//
// The pages' arithmetic without narrowing the activations: a bf16 value
// times a power of two that brings its block maximum into [2^14, 2^15) is
// exactly the sum of three e5m2 terms unless it lies more than 2^23 below
// that maximum; an fp32 h is exactly the sum of eight e5m2 terms within 2^7
// of its block maximum and within 2^-31 of that maximum below.  Products of
// e4m3 and e5m2 values are exact, the tensor cores accumulate in fp32, and
// each block's sum is scaled by its weight block scale and the activation's
// power of two: bf16 x times fp8 weights and f32 h times fp8 weights,
// accumulated in fp32.
//
// Weight tiles arrive by 5-D TMA boxes with the 128-byte swizzle (gate/up:
// [K window][32 gate, 32 up rows][128 bytes]; down: [K window][tile][8
// rows][128 bytes]); the same layout is the tcgen05 operand and the ldmatrix
// source (16-byte chunk c of row r at c xor (r % 8)).
//
// Every wait is bounded (kWaitLimitNs): a wait that runs out records
// MOE_ETIMEOUT in the workspace status word; the CTA waits (bounded) for its
// copies in flight and leaves.
#include <math.h>

#include <algorithm>
#include <mutex>

#include "common.cuh"
#include "internal.h"
#include "launch.h"
#include "tcgen05.cuh"
#include "topk.cuh"

namespace moe {

namespace {

constexpr int kSlot = 16384;           // ring slot bytes
constexpr int kMaxNt = 8;              // output 8-row tiles per CTA
constexpr int kGuRows = 32;            // gate (and up) rows of one gate/up unit: M = 64 of the MMA
constexpr uint32_t kGuWindow = 8192;   // one 128-byte K window of a unit's 64 rows
// The gate/up MMAs are issued by lane 0 of warps kIssuer0 .. kIssuer0 +
// kIssuers - 1 (an issuing thread is the bottleneck of MMAs this small, so
// several take the items in turn; not the epilogue warps, which the
// issuers wait for when the accumulator buffers run out).
constexpr int kIssuer0 = 4;
constexpr int kIssuers = 4;
constexpr int kEpiWaiter = 32;         // the epilogue's waiting thread (warp 1, lane 0)
constexpr uint32_t kSmemCap = 232448;  // dynamic shared memory per block (B200 opt-in)

// ------------------------------------------------------------ device helpers

// Two fp32 -> two e5m2 (round to nearest even, saturating), lo in the low byte.
__device__ __forceinline__ uint32_t f32x2_to_e5m2x2(float lo, float hi)
{
    uint16_t r;
    asm("cvt.rn.satfinite.e5m2x2.f32 %0, %2, %1;" : "=h"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ float2 e5m2x2_to_f32x2(uint32_t two)
{
    uint32_t h;
    asm("{ .reg .b16 l, u; mov.b32 {l, u}, %1; cvt.rn.f16x2.e5m2x2 %0, l; }" : "=r"(h) : "r"(two));
    return __half22float2(*reinterpret_cast<__half2 *>(&h));
}

__device__ __forceinline__ void tma_load_5d(uint32_t dst, const CUtensorMap *map, int c0, int c1, int c2, int c3,
                                            int c4, uint64_t *bar, uint64_t policy)
{
    asm volatile(
        "cp.async.bulk.tensor.5d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%3, %4, %5, %6, %7}], [%2], %8;" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(c4),
        "l"(policy)
        : "memory");
}

// The power of two that brings a block's largest magnitude into [2^14, 2^15),
// as its exponent, clamped so that 2^s and 2^-s are normal floats.
__device__ __forceinline__ int block_shift(float amax)
{
    if (!(amax > 0.f) || !isfinite(amax)) return 0;
    const int be = (int)((__float_as_uint(amax) >> 23) & 0xFFu);  // 0 for a subnormal
    return max(-100, min(100, 141 - be));
}
__device__ __forceinline__ float pow2f(int s) { return __uint_as_float((uint32_t)(s + 127) << 23); }

__device__ __forceinline__ int atomic_add_relaxed_gpu(int32_t *p, int v)
{
    int old;
    asm volatile("atom.relaxed.gpu.global.add.s32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
    return old;
}
__device__ __forceinline__ void red_release_gpu(int32_t *p, int v)
{
    asm volatile("red.release.gpu.global.add.s32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ int ld_acquire_cta_shared(const int32_t *p)
{
    int v;
    asm volatile("ld.acquire.cta.shared.b32 %0, [%1];" : "=r"(v) : "r"(smem_u32(p)) : "memory");
    return v;
}
__device__ __forceinline__ void st_release_cta_shared(int32_t *p, int v)
{
    asm volatile("st.release.cta.shared.b32 [%0], %1;" ::"r"(smem_u32(p)), "r"(v) : "memory");
}
__device__ __forceinline__ int ld_acquire_gpu(const int32_t *p)
{
    int v;
    asm volatile("ld.acquire.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ uint32_t ld_relaxed_gpu_u32(const int32_t *p)
{
    uint32_t v;
    asm volatile("ld.relaxed.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// Router logits travel between CTAs as 8-byte words: the fp32 value in the
// low half and the call's tag in the high half, stored and loaded whole (an
// aligned 8-byte access is single-copy atomic), so a reader that sees the
// tag sees the value, with no barrier between writer and reader.  The tag is
// the call's epoch + 1; words of earlier calls carry smaller tags and a
// fresh workspace holds zeros.
__device__ __forceinline__ void st_logit(uint64_t *w, float v, uint32_t tag)
{
    const uint64_t x = ((uint64_t)tag << 32) | (uint64_t)__float_as_uint(v);
    asm volatile("st.relaxed.gpu.global.b64 [%0], %1;" ::"l"(w), "l"(x) : "memory");
}
// The value of a logit word once it carries `tag`; false when the wait runs
// out (t0: the caller's start of waiting).
__device__ __forceinline__ bool ld_logit(const uint64_t *w, uint32_t tag, uint64_t t0, float &v)
{
    uint64_t x;
    asm volatile("ld.relaxed.gpu.global.b64 %0, [%1];" : "=l"(x) : "l"(w) : "memory");
    while ((uint32_t)(x >> 32) != tag) {
        if (globaltimer_ns() - t0 > kWaitLimitNs) return false;
        asm volatile("ld.relaxed.gpu.global.b64 %0, [%1];" : "=l"(x) : "l"(w) : "memory");
    }
    v = __uint_as_float((uint32_t)x);
    return true;
}

// Top-k of one row of tagged logits (one warp; the layout of topk_select);
// false in every lane when a wait ran out.
template <int EPL>
__device__ bool topk_select_tagged(const uint64_t *lrow, int E, int K, uint32_t tag, uint64_t t0, int32_t *out_idx,
                                   float *out_w, float *out_gsig)
{
    const int lane = threadIdx.x & 31;
    uint32_t v[EPL];
    int id[EPL];
    bool ok = true;
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
        const int e = lane * EPL + i;
        float l = 0.f;
        if (e < E && ok) ok = ld_logit(lrow + e, tag, t0, l);
        v[i] = (e < E) ? topk_key(l) : 0u;
        id[i] = e;
    }
    float z = 0.f;
    if (ok) ok = ld_logit(lrow + E, tag, t0, z);
    if (!__all_sync(0xFFFFFFFFu, ok)) return false;
    topk_select_keys<EPL>(v, id, z, K, out_idx, out_w, out_gsig);
    return true;
}

// A bounded wait, taken by lane 0 for the whole warp, for item q in ring
// slot s: the result is the same in every lane and the warp is converged
// again afterwards, as the mma.sync.aligned instructions that follow require.
//
// A warp's items are not consecutive in the ring (each warp takes its own
// units), so a warp can reach item q while its slot still holds an older
// item; a parity wait alone would then see the phase two back (same parity)
// completed.  The producer writes q into the slot's tag after arming the
// slot's barrier for q, which it does only once the slot's previous item was
// consumed: once the tag reads q, phase q / ns is the barrier's current (or
// just completed) phase and the parity wait is exact.
__device__ __forceinline__ bool wait_item(const volatile int32_t *tag, uint64_t *full, int s, int q, int ns)
{
    bool ok = true;
    if ((threadIdx.x & 31) == 0) {
        if (tag[s] != q) {
            const uint64_t t0 = globaltimer_ns();
            while (tag[s] != q) {
                if (globaltimer_ns() - t0 > kWaitLimitNs) {
                    ok = false;
                    break;
                }
            }
        }
        if (ok) ok = mbar_wait(&full[s], (uint32_t)((q / ns) & 1), kWaitLimitNs);
    }
    ok = __shfl_sync(0xFFFFFFFFu, ok ? 1 : 0, 0) != 0;
    __syncwarp();
    return ok;
}

// wait_item for one thread (the gate/up MMA issuer).
__device__ __forceinline__ bool wait_item_lane(const volatile int32_t *tag, uint64_t *full, int s, int q, int ns)
{
    if (tag[s] != q) {
        const uint64_t t0 = globaltimer_ns();
        while (tag[s] != q)
            if (globaltimer_ns() - t0 > kWaitLimitNs) return false;
    }
    return mbar_wait_spin(&full[s], (uint32_t)((q / ns) & 1), kWaitLimitNs);
}

// The router items' wait (their slots' first use): lane 0 for the warp.
__device__ __forceinline__ bool warp_wait(uint64_t *bar, uint32_t parity)
{
    bool ok = true;
    if ((threadIdx.x & 31) == 0) ok = mbar_wait(bar, parity, kWaitLimitNs);
    ok = __shfl_sync(0xFFFFFFFFu, ok ? 1 : 0, 0) != 0;
    __syncwarp();
    return ok;
}

// A wait that ran out: MOE_ETIMEOUT in the status word, and where this CTA
// gave up (the first time) in its diagnostic word: kind << 24 | item.
//   kind 1 router rows, 2 gate/up item (consumer), 3 down item (consumer),
//   4 producer, 6 a router logit (top-k), 8-10 gate/up MMAs and epilogue.
__device__ __forceinline__ void gave_up(int32_t *counters, int kind, int item)
{
    set_status(counters, MOE_ETIMEOUT);
    atomicCAS(&counters[kCtrStepDiag + blockIdx.x], 0, (kind << 24) | (item & 0xFFFFFF));
}

// Progress markers of a development build (-DMOE_STEP_TRACE): per (CTA,
// warp) the last point reached, stage << 24 | item.  Nothing in the library
// build.
#ifdef MOE_STEP_TRACE
#define STEP_MARK(stage, item)                                                                              \
    do {                                                                                                    \
        if ((threadIdx.x & 31) == 0)                                                                        \
            ((volatile int32_t *)p.counters)[kCtrStepDiag + 256 + blockIdx.x * 16 + (threadIdx.x >> 5)] =   \
                ((stage) << 24) | ((item) & 0xFFFFFF);                                                      \
    } while (0)
// the words of a slot's full and empty barriers when a wait ran out
#define STEP_SNAP(slot)                                                                                     \
    do {                                                                                                    \
        unsigned long long f_, e_;                                                                          \
        asm volatile("ld.shared.b64 %0, [%1];" : "=l"(f_) : "r"(smem_u32(&full[slot])));                   \
        asm volatile("ld.shared.b64 %0, [%1];" : "=l"(e_) : "r"(smem_u32(&empty[slot])));                  \
        int32_t *d_ = p.counters + kCtrStepDiag + 1024 + blockIdx.x * 4;                                    \
        if (atomicCAS(d_, 0, (int)(f_ & 0xFFFFFFFF)) == 0) {                                                \
            d_[1] = (int)(f_ >> 32);                                                                        \
            d_[2] = (int)(e_ & 0xFFFFFFFF);                                                                 \
            d_[3] = (int)(e_ >> 32);                                                                        \
        }                                                                                                   \
    } while (0)
#define STEP_CONSUMED(item)                                                                                 \
    do {                                                                                                    \
        if ((threadIdx.x & 31) == 0 && (item) < 64)                                                         \
            atomicOr((unsigned *)&p.counters[kCtrStepDiag + 256 + blockIdx.x * 16 + 10 + ((item) >> 5)],     \
                     1u << ((item) & 31));                                                                  \
    } while (0)
#else
#define STEP_MARK(stage, item) \
    do {                       \
    } while (0)
#define STEP_SNAP(slot) \
    do {                \
    } while (0)
#define STEP_CONSUMED(item) \
    do {                    \
    } while (0)
#endif

// Phase timestamps of a development build (-DMOE_STEP_TRACE): thread 0 of
// each CTA (lane 0 of warp 0 for the per-warp points) records %globaltimer
// at numbered points of the step.
#ifdef MOE_STEP_TRACE
__device__ unsigned long long g_step_trace[256 * 16];
__device__ unsigned long long g_item_trace[256 * 64 * 6];  // per CTA, item: landed, done, issued, [issue start, after expect_tx, after 1st TMA]
#define ITEM_T(q, which)                                                                        \
    do {                                                                                        \
        if ((threadIdx.x & 31) == 0 && (q) < 64)                                                \
            g_item_trace[(blockIdx.x * 64 + (q)) * 6 + (which)] = globaltimer_ns();             \
    } while (0)
#define ITEM_TL(q, which)                                                                       \
    do {                                                                                        \
        if ((q) < 64) g_item_trace[(blockIdx.x * 64 + (q)) * 6 + (which)] = globaltimer_ns();   \
    } while (0)
#define STEP_T(i)                                                                          \
    do {                                                                                   \
        if (threadIdx.x == 0) g_step_trace[blockIdx.x * 16 + (i)] = globaltimer_ns();      \
    } while (0)
#define STEP_TL(i)                                                  \
    do {                                                            \
        g_step_trace[blockIdx.x * 16 + (i)] = globaltimer_ns();     \
    } while (0)
#else
#define STEP_TL(i) \
    do {           \
    } while (0)
#define STEP_T(i) \
    do {          \
    } while (0)
#define ITEM_T(q, which) \
    do {                 \
    } while (0)
#define ITEM_TL(q, which) \
    do {                  \
    } while (0)
#endif

// One gate/up unit row's sums (this lane's tensor-memory lane of buffer
// tb): per row t of x, the K windows in order, each window's three term
// columns added first, times the window's weight block scale and the row's
// x scale.  NB = the accumulator columns of a window.
template <int NB>
__device__ __forceinline__ void gu_row_sums(uint32_t tb, int hb, int rows, const float *srow, const float *xfac,
                                            float (&acc)[kStepMaxRows])
{
    constexpr int kWpl = 32 / NB;                             // K windows per 32-column load
    constexpr int kTmax = NB == 8 ? 2 : kStepMaxRows;         // rows whose terms fit in NB columns
#pragma unroll
    for (int t = 0; t < kStepMaxRows; ++t) acc[t] = 0.f;
    for (int W0 = 0; W0 < hb; W0 += kWpl) {
        float v[32];
        tmem_ld_32x32(tb + (uint32_t)(W0 * NB), v);
        tmem_wait_ld();
#pragma unroll
        for (int wi = 0; wi < kWpl; ++wi) {
            const int W = W0 + wi;
            if (W >= hb) break;
            const float sw = srow[W];
#pragma unroll
            for (int t = 0; t < kTmax; ++t) {
                if (t >= rows) break;
                const float g = (v[wi * NB + 3 * t] + v[wi * NB + 3 * t + 1]) + v[wi * NB + 3 * t + 2];
                acc[t] = fmaf(sw * xfac[t * hb + W], g, acc[t]);
            }
        }
    }
}

// ------------------------------------------------------------ parameters

struct StepParams {
    CUtensorMap w13;   // routed W13: (128 B, I rows, gate|up, H/128 windows, E), boxes {128, 32, 2, gu_wp, 1}
    CUtensorMap w13s;  // shared W13: (128 B, Is rows, gate|up, H/128 windows, 1), the same boxes
    CUtensorMap w2;    // routed W2: (128 B, H rows, I/128 windows, E), boxes {128, 8, I/128, 1}
    CUtensorMap w2s;   // shared W2: (128 B, H rows, Is/128 windows, 1), boxes {128, 8, Is/128, 1}
    const uint16_t *x;
    const uint16_t *router_w;
    const uint16_t *shared_gate;
    const uint16_t *residual;
    const float *router_bias;
    const float *scales;   // routed experts' block scales, E slabs
    const float *sscales;  // the shared expert's
    const uint16_t *norm_w;  // RMSNorm weight [H], or null: x is the layer input as given
    double eps;
    uint16_t *out;
    int32_t *topk_idx;  // routing outputs [rows][K], [rows][K], [rows] (written by CTA 0)
    float *topk_w;
    float *gsig;
    uint64_t *lw;       // counters + kCtrStepLogits, [rows][ld]: the router logits as tagged words (column E: the gate)
    unsigned char *hterm;  // workspace [rows * (K + 1)][imax / 32][256]: h as e5m2 terms in the down MMAs' B layout
    float *hsc;            // workspace [rows * (K + 1)][imax / 32]: the power of two of each chunk of terms
    int32_t *counters;  // workspace counters (epoch, exit count, status, unit counts)
    int rows, H, E, K, I, Is, ld, imax;
    int ns;              // ring slots
    int gu_wp, gu_pieces;               // gate/up: K windows per piece, pieces
    int dn_tpi, dn_tpi_s, dn_epi;  // down: output tiles per item (routed, shared), routed experts per item
    int nt_max;          // output 8-row tiles per CTA, at most
    int rr_per_item;     // router rows per ring item
    // shared-memory offsets (from the 1024-aligned base)
    uint32_t o_uni, o_xb, o_xfac, o_y, o_sm, o_bar, o_gsc, o_dsc, o_cand;
    int rdy;             // ints between two experts' unit counters (each on its own 128-byte line when it fits)
    uint32_t o_xB;       // x as e5m2 terms: per K window a [nb rows][128 B] operand tile (128-byte swizzle)
    int nb;              // gate/up MMA N: 3 terms per row, 8 or 16
    int nbuf, tbuf;      // gate/up accumulator buffers in tensor memory, columns of each (H/128 * nb)
    int tcols;           // tensor-memory columns allocated
    int cand2;           // two-stage top-k: chunk candidates [rows][chunks][K] keys, then experts, at o_cand
    int max_units;       // gate/up units per CTA, at most (rows of the scale table)
    int x_stride;        // halves per x row in shared memory (f16 and bf16 copies)
};

// Small shared-memory block: routing and plan.
struct StepSmall {
    int32_t idx[kStepMaxRows * kMaxTopK];
    float w[kStepMaxRows * kMaxTopK];
    int32_t loc[kStepMaxRows * kMaxTopK];  // index of idx in the list of distinct experts
    float gs[kStepMaxRows];
    uint32_t mask[kMaxExperts / 32];
    int32_t list[kStepMaxRows * kMaxTopK];  // distinct routed experts, ascending
    int32_t tag[16];                        // ring slot -> the item last issued into it (-1: none)
    float xch[32 * kStepMaxRows];           // gate/up epilogue: the up rows' sums per row of x
    float hmx[2 * kStepMaxRows];            // gate/up epilogue: each gate warp's largest |h| per row of x
    uint32_t tmem;                          // tensor-memory base of this CTA's accumulators
    int32_t gu_stop;                        // gate/up epilogue: leave the unit loop (written by its waiter)
    int32_t dn_next;                        // down phase: the next item to claim
    int32_t dsc_ready;                      // the down block scales are staged (warps 0-3 -> 4-7)
    double red[kStepWarps * kStepMaxRows];  // RMSNorm: per-warp sums of squares
    double inv[kStepMaxRows];               // RMSNorm: 1 / sqrt(mean square + eps) per row
    int32_t n_list;
    int32_t abort;
    uint32_t epoch;                         // this call's epoch (the logits' tag is epoch + 1)
    int32_t pad;
};

__host__ __device__ inline int n_router_rows(int E, int G, int c)
{
    return (int)(((int64_t)(c + 1) * (E + 1)) / G - ((int64_t)c * (E + 1)) / G);
}
__host__ __device__ inline int first_router_row(int E, int G, int c) { return (int)(((int64_t)c * (E + 1)) / G); }
__host__ __device__ inline int first_tile(int n8, int G, int c) { return (int)(((int64_t)c * n8) / G); }

// ------------------------------------------------------------ item sequence
//
// Every thread of a CTA enumerates the same item sequence:
//   router items  (rr_per_item router rows each; the gate vector is row E)
//   gate/up items (local unit l = 0.., unit u = c + l*G; pieces p)
//   down items    (groups of dn_epi experts of the down list [shared,
//                  routed ascending]; the shared expert alone; pieces p)
// Item q lives in ring slot q % ns.

struct Item {
    int kind;    // 0 router, 1 gate/up, 2 down
    int a, b, p; // router: first local row, row count; gate/up: unit, local unit index; down: group, -
};

struct Seq {
    int n_router, n_units_local, n_gu, n_tc_s, n_tc_r, n_groups_r, n_dn, total;
};

// Down items: per group of experts (the shared expert alone, then groups of
// dn_epi routed experts of the list), per chunk of dn_tpi output tiles of
// this CTA, the full K of the down rows (one TMA box per expert and tile).
// The parts of make_seq that do not depend on the routing (computed before
// the plan): router items, down tile chunks, units of the shared expert and
// of one routed expert.
struct SeqConst {
    int n_router, n_tc_s, n_tc_r, us, per;
};
__device__ __forceinline__ SeqConst seq_const(const StepParams &p, int nt, int nr)
{
    SeqConst k;
    k.n_router = (nr + p.rr_per_item - 1) / p.rr_per_item;
    k.n_tc_s = nt > 0 ? (nt + p.dn_tpi_s - 1) / p.dn_tpi_s : 0;
    k.n_tc_r = nt > 0 ? (nt + p.dn_tpi - 1) / p.dn_tpi : 0;
    k.us = p.Is / kGuRows;
    k.per = p.I / kGuRows;
    return k;
}
// make_seq from those (the same sequence): one division after the plan.
__device__ __forceinline__ Seq make_seq_k(const StepParams &p, const SeqConst &k, int U)
{
    const int G = gridDim.x, c = blockIdx.x;
    Seq s;
    s.n_router = k.n_router;
    const int units = k.us + U * k.per;
    s.n_units_local = units > c ? (units - 1 - c) / G + 1 : 0;
    s.n_gu = s.n_units_local * p.gu_pieces;
    s.n_tc_s = k.n_tc_s;
    s.n_tc_r = k.n_tc_r;
    s.n_groups_r = p.dn_epi == 1 ? U : (U + p.dn_epi - 1) / p.dn_epi;
    s.n_dn = s.n_tc_s + s.n_groups_r * s.n_tc_r;
    s.total = s.n_router + s.n_gu + s.n_dn;
    return s;
}

__device__ __forceinline__ Seq make_seq(const StepParams &p, int U, int nt, int nr)
{
    const int G = gridDim.x, c = blockIdx.x;
    Seq s;
    s.n_router = (nr + p.rr_per_item - 1) / p.rr_per_item;
    const int units = p.Is / kGuRows + U * (p.I / kGuRows);
    s.n_units_local = units > c ? (units - 1 - c) / G + 1 : 0;
    s.n_gu = s.n_units_local * p.gu_pieces;
    s.n_tc_s = nt > 0 ? (nt + p.dn_tpi_s - 1) / p.dn_tpi_s : 0;
    s.n_tc_r = nt > 0 ? (nt + p.dn_tpi - 1) / p.dn_tpi : 0;
    s.n_groups_r = (U + p.dn_epi - 1) / p.dn_epi;
    s.n_dn = s.n_tc_s + s.n_groups_r * s.n_tc_r;
    s.total = s.n_router + s.n_gu + s.n_dn;
    return s;
}

// kind 0 router: a = first local router row; kind 1 gate/up: a = unit, b =
// local unit, p = piece; kind 2 down: a = group (0 shared), p = tile chunk,
// b = the down item's index (its warp is b % kStepWarps).
__device__ __forceinline__ Item item_at(const StepParams &p, const Seq &s, int q)
{
    Item it;
    if (q < s.n_router) {
        it.kind = 0;
        it.a = q * p.rr_per_item;
        it.b = 0;
        it.p = 0;
        return it;
    }
    q -= s.n_router;
    if (q < s.n_gu) {
        it.kind = 1;
        const int l = q / p.gu_pieces;
        it.b = l;
        it.a = blockIdx.x + l * gridDim.x;
        it.p = q - l * p.gu_pieces;
        return it;
    }
    q -= s.n_gu;
    it.kind = 2;
    it.b = q;
    if (q < s.n_tc_s) {
        it.a = 0;
        it.p = q;
    } else {
        q -= s.n_tc_s;
        const int g = q / s.n_tc_r;
        it.a = 1 + g;
        it.p = q - g * s.n_tc_r;
    }
    return it;
}

// Gate/up unit u -> (shared?, expert, first gate row j).
__device__ __forceinline__ void unit_of(const StepParams &p, const StepSmall &sm, int u, bool &shared, int &e, int &j)
{
    const int us = p.Is / kGuRows;
    if (u < us) {
        shared = true;
        e = 0;
        j = u * kGuRows;
    } else {
        shared = false;
        const int per = p.I / kGuRows;
        const int ue = (u - us) / per;
        e = sm.list[ue];
        j = (u - us - ue * per) * kGuRows;
    }
}

// ------------------------------------------------------------ producer

__device__ __forceinline__ uint32_t item_bytes(const StepParams &p, const Item &it, int nr_total, int nt, int U)
{
    if (it.kind == 0) return (uint32_t)min(p.rr_per_item, nr_total - it.a) * (uint32_t)p.H * 2u;
    if (it.kind == 1) return (uint32_t)p.gu_wp * kGuWindow;  // a whole box, also past the last window (zeros)
    const int tpi = it.a == 0 ? p.dn_tpi_s : p.dn_tpi;
    return (uint32_t)tpi * 8u * (uint32_t)(it.a == 0 ? p.Is : p.I);  // a whole box (tiles past H: zeros)
}

// Issue item `it` into ring slot `slot`.  With go == false the same code
// runs without arming the barrier or copying anything (it brings the
// instructions into the cache ahead of their first real use).
__device__ __noinline__ void issue_item(const StepParams &p, const StepSmall &sm, const Item &it, uint32_t slot,
                                        uint64_t *full, int r0, int nr_total, int tile0, int nt, int U, uint64_t pol,
                                        int qdbg = 0, bool go = true)
{
    ITEM_TL(qdbg, 3);
    const uint32_t bytes = item_bytes(p, it, nr_total, nt, U);
    if (go) mbar_arrive_expect_tx(full, bytes);
    ITEM_TL(qdbg, 4);
    if (it.kind == 0) {
        // router rows r0 + it.a ..; row E (the gate vector) comes from shared_gate
        const int n = min(p.rr_per_item, nr_total - it.a);
        const int first = r0 + it.a;
        const int nw = max(0, min(n, p.E - first));  // rows of router_w
        const uint32_t rowb = (uint32_t)p.H * 2u;
        if (go && nw > 0) {
            asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                             slot),
                         "l"(p.router_w + (size_t)first * p.H), "r"(nw * rowb), "r"(smem_u32(full))
                         : "memory");
        }
        if (go && nw < n) {
            asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                             slot + nw * rowb),
                         "l"(p.shared_gate), "r"(rowb), "r"(smem_u32(full))
                         : "memory");
        }
        return;
    }
    if (it.kind == 1) {
        // one box: per K window, the unit's 32 gate rows then its 32 up
        // rows, a 64-row operand tile of the 128-byte swizzle layout
        bool shared;
        int e, j;
        unit_of(p, sm, it.a, shared, e, j);
        if (go) tma_load_5d(slot, shared ? &p.w13s : &p.w13, 0, j, 0, it.p * p.gu_wp, e, full, pol);
        ITEM_TL(qdbg, 5);
        return;
    }
    // one box: per K window, the item's output tiles (8 rows each) of its
    // expert's W2, [window][tile][8 rows][128 B]
    const int tpi = it.a == 0 ? p.dn_tpi_s : p.dn_tpi;
    const int e = it.a == 0 ? 0 : sm.list[(it.a - 1) * p.dn_epi];
    if (go) tma_load_5d(slot, it.a == 0 ? &p.w2s : &p.w2, 0, 0, tile0 + it.p * tpi, 0, e, full, pol);
}

// The gate/up item of local unit l, K piece pc into `slot` (one 5-D box);
// with go == false nothing is armed or copied (instruction-cache warm-up).
__device__ __noinline__ void issue_gu(const StepParams &p, const StepSmall &sm, int l, int pc, uint32_t slot,
                                      uint64_t *full, uint64_t pol, bool go)
{
    bool shared;
    int e, j;
    unit_of(p, sm, blockIdx.x + l * gridDim.x, shared, e, j);
    if (go) {
        mbar_arrive_expect_tx(full, (uint32_t)p.gu_wp * kGuWindow);
        tma_load_5d(slot, shared ? &p.w13s : &p.w13, 0, j, 0, pc * p.gu_wp, e, full, pol);
    }
}

// A down item's expert: wait until all of its gate/up units (in whichever
// CTAs) are counted (lane 0 polls with acquire semantics, bounded; the warp
// barrier then orders the lanes' reads of h after the counted writes).
// sl[t] = the slot of h of row t of x routed to the expert (-1: not routed),
// bit t of *routed set for those rows.  False if the wait ran out.
__device__ __forceinline__ bool wait_expert(const StepParams &p, const StepSmall &sm, const Item &it,
                                            int (&sl)[kStepMaxRows], uint32_t *routed)
{
    const int lane = threadIdx.x & 31;
    const int rows = p.rows, K = p.K;
    const bool shared = it.a == 0;
    const int li = shared ? -1 : (it.a - 1) * p.dn_epi;  // one expert a down item
    const int e = shared ? 0 : sm.list[li];
    const int de = shared ? 0 : 1 + li;
    const int need = (shared ? p.Is : p.I) / kGuRows;
    const int32_t *ready = p.counters + kCtrStepReady + (int)(sm.epoch & 1u) * kStepReadyHalf + de * p.rdy;
    int ok = 1;
    if (lane == 0 && ld_acquire_gpu(ready) < need) {
        const uint64_t t0 = globaltimer_ns();
        while (ld_acquire_gpu(ready) < need) {
            if (globaltimer_ns() - t0 > kWaitLimitNs) {
                ok = 0;
                break;
            }
        }
    }
    if (!__shfl_sync(0xFFFFFFFFu, ok, 0)) return false;
    uint32_t m = 0;
#pragma unroll
    for (int t = 0; t < kStepMaxRows; ++t) {
        sl[t] = -1;
        if (t < rows) {
            if (shared) {
                sl[t] = rows * K + t;
            } else {
                for (int r = 0; r < K; ++r)
                    if (sm.idx[t * K + r] == e) sl[t] = t * K + r;
            }
            if (sl[t] >= 0) m |= 1u << t;
        }
    }
    *routed = m;
    return true;
}

__device__ __forceinline__ void ldmatrix_x4(uint32_t addr, uint32_t (&a)[4])
{
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(a[0]), "=r"(a[1]), "=r"(a[2]), "=r"(a[3])
                 : "r"(addr));
}

// D = A * B for one K chunk of 32: A 16 x 32 e4m3 (row major), B 32 x 8 e5m2
// (column major), fp32 accumulation from zero.
__device__ __forceinline__ void mma_e4m3_e5m2_16832(float (&d)[4], const uint32_t (&a)[4], uint2 b)
{
    asm volatile(
        "mma.sync.aligned.m16n8k32.row.col.f32.e4m3.e5m2.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%10, %10, %10, %10};"
        : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b.x), "r"(b.y), "f"(0.f));
}

// One down item, by one warp, on the tensor cores (mma.sync): per K chunk of
// 32, A = the item's weight rows (its two 8-row output tiles as MMA rows 0-7
// and 8-15; with one tile a copy of it) straight from the TMA slot through
// ldmatrix (the 128-byte swizzle: 16-byte chunk c of row r sits at c xor
// (r % 8)), B = the eight e5m2 terms of h of a row of x routed to the expert
// (column j = term j), as the gate/up epilogue laid them out (lane l's eight
// bytes of a chunk are its two B registers), brought into the warp's buffer
// bbuf (16 chunks) by one bulk copy a round.  Each chunk's D, its eight term
// columns added, times the window's weight block scale and the chunk's power
// of two of h, into a running sum per row; the four lanes of a row then add
// their sums.  Products are exact (e4m3 x e5m2); sums fp32.  *bphase: the
// parity of bbar's next phase.  False if a copy's wait ran out.
template <int R>
__device__ __forceinline__ bool down_item_mma(const StepParams &p, uint32_t slot_u32, int tpi, int ibu, int tl0,
                                              int nt, int tile0, int rb0, const float *s2e, int ibm, float *yb,
                                              int yrow, const int (&sl)[kStepMaxRows], uint32_t routed,
                                              unsigned char *bbuf, uint64_t *bbar, uint32_t *bphase)
{
    const int lane = threadIdx.x & 31, g = lane >> 2;
    const int nch = ibu * 4;         // K chunks of 32
    const int ntc = p.imax / 32;     // chunks of a slot of h terms
    // this lane's ldmatrix row: matrix lane / 8 (0: rows 0-7, K 0-15; 1: rows
    // 8-15; 2, 3: K 16-31), row lane % 8 of it
    const int mi = lane >> 3, rr = lane & 7;
    const uint32_t abase = slot_u32 + (uint32_t)((tpi == 2 ? (mi & 1) : 0) * 1024 + rr * 128);
    const int tlB = min(tl0 + 1, nt - 1);
    const float *s2a = s2e + min(1, ((tile0 + tl0) * 8) / 128 - rb0) * ibm;
    const float *s2b = s2e + min(1, ((tile0 + tlB) * 8) / 128 - rb0) * ibm;
    const uint32_t bb = smem_u32(bbuf) + (uint32_t)lane * 8;
#pragma unroll
    for (int t = 0; t < R; ++t) {
        if (!((routed >> t) & 1u)) continue;  // the same in every lane
        // four independent sums per tile row (chunk i into sums i % 4), added
        // in a fixed order at the end
        float acc0[4] = {0.f, 0.f, 0.f, 0.f}, acc1[4] = {0.f, 0.f, 0.f, 0.f};
        for (int c0 = 0; c0 < nch; c0 += 16) {
            const int n = min(16, nch - c0);
            if (lane == 0) {
                fence_proxy_async_smem();  // the lanes' reads of the last round (ordered by the warp barrier)
                mbar_arrive_expect_tx(bbar, (uint32_t)n * 256);
                bulk_g2s(bbuf, p.hterm + ((size_t)sl[t] * ntc + c0) * 256, (uint32_t)n * 256, bbar);
            }
            const float hs = lane < n ? __ldcg(p.hsc + (size_t)sl[t] * ntc + c0 + lane) : 0.f;
            int ok = 1;
            if (lane == 0) ok = mbar_wait_spin(bbar, *bphase, kWaitLimitNs) ? 1 : 0;
            *bphase ^= 1u;
            if (!__shfl_sync(0xFFFFFFFFu, ok, 0)) return false;
            // a window (four chunks) at a time: n is a multiple of 4
            for (int i0 = 0; i0 < n; i0 += 4) {
                const int w = (c0 + i0) >> 2;
                uint32_t a[4][4];
                uint2 b[4];
#pragma unroll
                for (int kc = 0; kc < 4; ++kc) {
                    ldmatrix_x4(abase + (uint32_t)(w * tpi * 1024) + ((uint32_t)((2 * kc + (mi >> 1)) ^ rr) << 4),
                                a[kc]);
                    asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];"
                                 : "=r"(b[kc].x), "=r"(b[kc].y)
                                 : "r"(bb + (uint32_t)(i0 + kc) * 256));
                }
                float d[4][4];
#pragma unroll
                for (int kc = 0; kc < 4; ++kc) mma_e4m3_e5m2_16832(d[kc], a[kc], b[kc]);
                const float sa = s2a[w], sb = s2b[w];
#pragma unroll
                for (int kc = 0; kc < 4; ++kc) {
                    const float f = __shfl_sync(0xFFFFFFFFu, hs, i0 + kc);
                    acc0[kc] = fmaf(sa * f, d[kc][0] + d[kc][1], acc0[kc]);
                    acc1[kc] = fmaf(sb * f, d[kc][2] + d[kc][3], acc1[kc]);
                }
            }
            __syncwarp();  // the buffer is free for the next round
        }
        float v0 = (acc0[0] + acc0[1]) + (acc0[2] + acc0[3]);
        float v1 = (acc1[0] + acc1[1]) + (acc1[2] + acc1[3]);
        v0 += __shfl_xor_sync(0xFFFFFFFFu, v0, 1);
        v0 += __shfl_xor_sync(0xFFFFFFFFu, v0, 2);
        v1 += __shfl_xor_sync(0xFFFFFFFFu, v1, 1);
        v1 += __shfl_xor_sync(0xFFFFFFFFu, v1, 2);
        if ((lane & 3) == 0) {
            if (tl0 < nt) yb[(size_t)t * yrow + tl0 * 8 + g] = v0;
            if (tpi == 2 && tl0 + 1 < nt) yb[(size_t)t * yrow + (tl0 + 1) * 8 + g] = v1;
        }
    }
    return true;
}

// P3, by each consumer warp: down items claimed one at a time in item order
// (warps arrive as they finish gate/up); each waits until its
// expert's gate/up units (in whichever CTAs) are all counted and for its
// weight rows, then multiplies them by the expert's h terms on the tensor
// cores (mma.sync, one warp an item) into the down buffer.
__device__ __forceinline__ void down_phase(const StepParams &p, StepSmall &sm, unsigned char *sbase, uint32_t base,
                                           uint64_t *full, uint64_t *empty, uint64_t *tdone, uint64_t *bbars,
                                           const Seq &seq, int nt, int tile0, int rb0, int ibm, const float *dsc,
                                           float *ybuf, volatile int32_t *abort)
{
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int rows = p.rows;
    {
        const int yrow = p.nt_max * 8;
        // the warp's buffer of h terms (in the x-term region: first every
        // gate/up MMA, which reads the x terms, must be done)
        unsigned char *bbuf = sbase + p.o_uni + (size_t)warp * 16 * 256;
        uint64_t *bbar = &bbars[warp];
        uint32_t bphase = 0;
        {
            int okd = 1;
            if (lane == 0) okd = mbar_wait(tdone, 0, kWaitLimitNs) ? 1 : 0;
            // the down block scales staged by warps 0-3 (long done by now)
            if (lane == 0 && okd && ld_acquire_cta_shared(&sm.dsc_ready) == 0) {
                const uint64_t t0 = globaltimer_ns();
                while (ld_acquire_cta_shared(&sm.dsc_ready) == 0)
                    if (globaltimer_ns() - t0 > kWaitLimitNs) {
                        okd = 0;
                        break;
                    }
            }
            if (!__shfl_sync(0xFFFFFFFFu, okd, 0)) {
                if (lane == 0) {
                    gave_up(p.counters, 10, 2);
                    *abort = 1;
                }
            }
        }
        for (;;) {
            // the next unclaimed item (warps arrive as they finish gate/up)
            int b = 0;
            if (lane == 0) b = atomicAdd(&sm.dn_next, 1);
            b = __shfl_sync(0xFFFFFFFFu, b, 0);
            if (b >= seq.n_dn || *abort) break;
            const int q = seq.n_router + seq.n_gu + b;
            const Item it = item_at(p, seq, q);
            const int s = q % p.ns;
            int sl[kStepMaxRows];
            uint32_t routed = 0;
            if (!wait_expert(p, sm, it, sl, &routed)) {
                if (lane == 0) {
                    gave_up(p.counters, 11, q);
                    *abort = 1;
                }
                break;
            }
            ITEM_T(48 + b, 0);  // (trace rows 48-63: down items in claim order) expert seen counted
            if (!wait_item(sm.tag, full, s, q, p.ns)) {
                if (lane == 0) {
                    gave_up(p.counters, 3, q);
                    *abort = 1;
                }
                break;
            }
            ITEM_T(48 + b, 1);  // weight rows seen
            const bool shared = it.a == 0;
            const int de = shared ? 0 : 1 + (it.a - 1) * p.dn_epi;
            const int tpi = shared ? p.dn_tpi_s : p.dn_tpi;
            const int ibu = (shared ? p.Is : p.I) / 128;
            const uint32_t su = base + (uint32_t)s * kSlot;
            const float *s2e = dsc + (size_t)de * 2 * ibm;
            float *yb = ybuf + (size_t)de * rows * yrow;
            const int tl0 = it.p * tpi;
            bool ok;
            switch (rows) {
            case 1: ok = down_item_mma<1>(p, su, tpi, ibu, tl0, nt, tile0, rb0, s2e, ibm, yb, yrow, sl, routed, bbuf, bbar, &bphase); break;
            case 2: ok = down_item_mma<2>(p, su, tpi, ibu, tl0, nt, tile0, rb0, s2e, ibm, yb, yrow, sl, routed, bbuf, bbar, &bphase); break;
            case 3: ok = down_item_mma<3>(p, su, tpi, ibu, tl0, nt, tile0, rb0, s2e, ibm, yb, yrow, sl, routed, bbuf, bbar, &bphase); break;
            case 4: ok = down_item_mma<4>(p, su, tpi, ibu, tl0, nt, tile0, rb0, s2e, ibm, yb, yrow, sl, routed, bbuf, bbar, &bphase); break;
            default: ok = down_item_mma<kStepMaxRows>(p, su, tpi, ibu, tl0, nt, tile0, rb0, s2e, ibm, yb, yrow, sl, routed, bbuf, bbar, &bphase); break;
            }
            if (!ok) {
                if (lane == 0) {
                    gave_up(p.counters, 12, q);
                    *abort = 1;
                }
                break;
            }
            ITEM_T(48 + b, 2);  // done
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[s]);
        }
    }
}

// ------------------------------------------------------------ the kernel

__global__ void __launch_bounds__(kStepThreads, 1) decode_step_kernel(const __grid_constant__ StepParams p)
{
    extern __shared__ unsigned char smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    unsigned char *sbase = smem_raw + (base - raw);
    StepSmall &sm = *reinterpret_cast<StepSmall *>(sbase + p.o_sm);
    uint64_t *full = reinterpret_cast<uint64_t *>(sbase + p.o_bar);
    uint64_t *empty = full + p.ns;
    uint64_t *tfull = empty + p.ns;  // [2] a unit's gate/up MMAs done (tcgen05.commit)
    uint64_t *tfree = tfull + 2;     // [2] its accumulators read (the 4 epilogue warps)
    uint64_t *tdone = tfree + 2;     // every gate/up MMA of this CTA done
    uint64_t *bbars = tdone + 1;     // [kStepWarps] each consumer warp's bulk copies of h terms
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int G = gridDim.x, c = blockIdx.x;
    const int rows = p.rows, H = p.H, E = p.E, K = p.K;
    const int hb = H / 128;
    const int nr_total = n_router_rows(E, G, c);
    const int r0 = first_router_row(E, G, c);
    const int n8 = H / 8;
    const int tile0 = first_tile(n8, G, c);
    const int nt = first_tile(n8, G, c + 1) - tile0;
    const bool producer = warp == kStepWarps;
    int exit_old = -1;  // (thread 0) the count of CTAs that had read the epoch before this one
    volatile int32_t *abort = &sm.abort;

    if (threadIdx.x == 0) {
        for (int s = 0; s < p.ns; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
            sm.tag[s] = -1;
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&tfull[b], kIssuers);
            mbar_init(&tfree[b], 4);
        }
        mbar_init(tdone, kIssuers);
        for (int w = 0; w < kStepWarps; ++w) mbar_init(&bbars[w], 1);
        sm.abort = 0;
        sm.dn_next = 0;
        sm.dsc_ready = 0;
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(&sm.tmem, (uint32_t)p.tcols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem;

    STEP_T(0);
    // ---------------------------------------------------------------- P0
    // The producer issues the items that depend only on weights: router
    // rows, then the shared expert's gate/up units (the first local units).
    const uint64_t pol = policy_evict_first();
    const Seq s0 = make_seq(p, 0, 0, nr_total);  // U = 0: router and shared-expert items only (a prefix of the full sequence)
    const SeqConst sk = seq_const(p, nt, nr_total);
    const int p0_count = min(s0.total, p.ns);
    // This CTA's first gate/up unit is the shared expert's and all of its
    // copies are issued in P0: its MMAs go out while the CTA waits at the
    // other CTAs' logits (they need only x's terms), not after the plan.
    const bool gu_early = s0.n_units_local > 0 && s0.n_router + p.gu_pieces <= p0_count;
    if (producer) {
        if (lane == 0) {
            tma_prefetch_desc(&p.w13);
            tma_prefetch_desc(&p.w13s);
            tma_prefetch_desc(&p.w2);
            tma_prefetch_desc(&p.w2s);
        }
        // the lanes issue in parallel: lane l takes items l, l + 32, ...
        for (int q = lane; q < p0_count; q += kWarp) {
            issue_item(p, sm, item_at(p, s0, q), base + (uint32_t)q * kSlot, &full[q], r0, nr_total, tile0, nt, 0,
                       pol, q);
            ((volatile int32_t *)sm.tag)[q] = q;
            ITEM_T(q, 2);
        }
    }

    // Each producer lane's first item after the plan, if a gate/up item in
    // a fresh slot (its unit and piece do not depend on the routing), and
    // the issue paths run once without issuing, so that the first wave after
    // the plan neither divides nor waits for instruction fetches (the
    // distinct-expert list is not built yet: no coordinate is used).
    int fq = lane;
    while (fq < p0_count) fq += kWarp;
    const int fg = fq - s0.n_router;
    const int fl = fg >= 0 ? fg / p.gu_pieces : 0, fpc = fg >= 0 ? fg - fl * p.gu_pieces : 0;
    if (producer && lane == 0) {
        const int Uw = min(rows * K, E);
        const Seq sw = make_seq(p, Uw, nt, nr_total);
        if (sw.n_gu > 0) issue_gu(p, sm, 0, 0, base, &full[0], pol, false);
        if (sw.n_dn > 0)
            issue_item(p, sm, item_at(p, sw, sw.n_router + sw.n_gu), base, &full[0], r0, nr_total, tile0, nt, Uw,
                       pol, 0, false);
    }
    pdl_wait();  // x and the workspace may be written by the previous kernel
    STEP_T(1);
    // this call's epoch, written by the previous call's last CTA (its grid has
    // finished: the PDL wait); the load is not waited on before x's loads
    const uint32_t ep = threadIdx.x == 0 ? ld_relaxed_gpu_u32(p.counters + kCtrStepEpoch) : 0u;

    // ---------------------------------------------------------------- P1
    if (!producer) {
        // x (bf16) -> shared memory: the rows as given, or the RMSNorm of the
        // residual rows (in double, rounded once to bf16, as the norm's
        // definition reads)
        uint16_t *xb = reinterpret_cast<uint16_t *>(sbase + p.o_xb);
        const int ct = threadIdx.x;  // 0 .. kStepWarps*32 - 1
        if (p.norm_w) {
            for (int t = 0; t < rows; ++t) {
                double ss = 0.0;
                for (int h = ct; h < H; h += kStepWarps * kWarp) {
                    const double v = (double)bf16_bits_to_f32(p.x[(size_t)t * H + h]);
                    ss = fma(v, v, ss);
                }
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xFFFFFFFFu, ss, o);
                if (lane == 0) sm.red[warp * kStepMaxRows + t] = ss;
            }
            named_barrier(1, kStepWarps * kWarp);
            if (ct < rows) {
                double tot = 0.0;
                for (int w = 0; w < kStepWarps; ++w) tot += sm.red[w * kStepMaxRows + ct];
                sm.inv[ct] = 1.0 / sqrt(tot / (double)H + p.eps);
            }
            named_barrier(1, kStepWarps * kWarp);
            for (int i = ct; i < rows * H; i += kStepWarps * kWarp) {
                const int t = i / H, h = i - t * H;
                const double v = ((double)bf16_bits_to_f32(p.x[(size_t)t * H + h]) * sm.inv[t]) *
                                 (double)bf16_bits_to_f32(p.norm_w[h]);
                xb[(size_t)t * p.x_stride + h] = f64_to_bf16_rn(v);
            }
        } else {
            for (int i = ct; i < rows * (H / 8); i += kStepWarps * kWarp) {
                const int t = i / (H / 8), ch = i - t * (H / 8);
                *reinterpret_cast<uint4 *>(xb + (size_t)t * p.x_stride + ch * 8) =
                    __ldg(reinterpret_cast<const uint4 *>(p.x + (size_t)t * H) + ch);
            }
        }
        if (ct == 0) sm.epoch = ep;
        named_barrier(1, kStepWarps * kWarp);
        // (thread 0) this CTA has read the epoch: the count's answer is needed
        // only after P3 (the last CTA to be counted advances the epoch then)
        if (ct == 0) exit_old = atomic_add_relaxed_gpu(p.counters + kCtrStepExit, 1);
        // x -> three e5m2 terms per value, the B operand of the gate/up
        // products: per (row, 128 block) a power of two puts the block's
        // largest magnitude in [2^14, 2^15), and t1 = e5m2(x'),
        // t2 = e5m2(x' - t1), t3 = e5m2(x' - t1 - t2) (differences exact in
        // fp32) sum exactly to x' for every value within 2^23 of that
        // maximum.  Term j of row t is operand row 3t + j; K window W is a
        // [nb rows][128 B] tile with the 128-byte swizzle (16-byte chunk c of
        // row n at chunk c ^ (n % 8) of the row).
        unsigned char *xB = sbase + p.o_xB;
        float *xfac = reinterpret_cast<float *>(sbase + p.o_xfac);
        for (int u = warp; u < rows * hb; u += kStepWarps) {
            const int t = u / hb, kb = u - t * hb;
            const uint2 raw2 = *reinterpret_cast<const uint2 *>(xb + (size_t)t * p.x_stride + kb * 128 + lane * 4);
            const float v[4] = {bf16_lo(raw2.x), bf16_hi(raw2.x), bf16_lo(raw2.y), bf16_hi(raw2.y)};
            const float amax = warp_max(fmaxf(fmaxf(fabsf(v[0]), fabsf(v[1])), fmaxf(fabsf(v[2]), fabsf(v[3]))));
            const int sh = block_shift(amax);
            const float f = pow2f(sh);
            uint32_t tw[3] = {0u, 0u, 0u};
#pragma unroll
            for (int i = 0; i < 2; ++i) {
                const float x0 = v[2 * i] * f, x1 = v[2 * i + 1] * f;
                const uint32_t c1 = f32x2_to_e5m2x2(x0, x1);
                const float2 d1 = e5m2x2_to_f32x2(c1);
                const float y0 = x0 - d1.x, y1 = x1 - d1.y;
                const uint32_t c2 = f32x2_to_e5m2x2(y0, y1);
                const float2 d2 = e5m2x2_to_f32x2(c2);
                const uint32_t c3 = f32x2_to_e5m2x2(y0 - d2.x, y1 - d2.y);
                tw[0] |= c1 << (16 * i);
                tw[1] |= c2 << (16 * i);
                tw[2] |= c3 << (16 * i);
            }
#pragma unroll
            for (int jt = 0; jt < 3; ++jt) {
                const int n = 3 * t + jt;
                const uint32_t off = (uint32_t)(kb * p.nb * 128 + (n >> 3) * 1024 + (n & 7) * 128) +
                                     (uint32_t)((((lane >> 2) ^ (n & 7)) * 16) + (lane & 3) * 4);
                *reinterpret_cast<uint32_t *>(xB + off) = tw[jt];
            }
            if (lane == 0) xfac[t * hb + kb] = pow2f(-sh);
        }
        fence_proxy_async_smem();  // the tensor cores read the terms through the async proxy
        STEP_T(2);  // x staged
        // router rows (router items 0 .. n_router-1 in slots 0 ..), each
        // logit published with this call's tag
        const uint32_t tag = sm.epoch + 1;
        for (int ri = 0; ri < s0.n_router; ++ri) {
            if (!warp_wait(&full[ri], 0)) {
                if (lane == 0) {
                    gave_up(p.counters, 1, ri);
                    *abort = 1;
                }
                break;
            }
            const int first = ri * p.rr_per_item;
            const int n = min(p.rr_per_item, nr_total - first);
            for (int rr = warp; rr < n; rr += kStepWarps) {
                const int e = r0 + first + rr;
                const uint4 *wrow = reinterpret_cast<const uint4 *>(sbase + (size_t)ri * kSlot + (size_t)rr * H * 2);
                float acc[kStepMaxRows];
#pragma unroll
                for (int t = 0; t < kStepMaxRows; ++t) acc[t] = 0.f;
                for (int ch = lane; ch < H / 8; ch += kWarp) {
                    const uint4 w8 = wrow[ch];
#pragma unroll
                    for (int t = 0; t < kStepMaxRows; ++t) {
                        if (t < rows) {
                            const uint4 xv = *reinterpret_cast<const uint4 *>(xb + (size_t)t * p.x_stride + ch * 8);
                            float a = bf16_lo(w8.x) * bf16_lo(xv.x);
                            float b = bf16_hi(w8.x) * bf16_hi(xv.x);
                            a = fmaf(bf16_lo(w8.y), bf16_lo(xv.y), a);
                            b = fmaf(bf16_hi(w8.y), bf16_hi(xv.y), b);
                            a = fmaf(bf16_lo(w8.z), bf16_lo(xv.z), a);
                            b = fmaf(bf16_hi(w8.z), bf16_hi(xv.z), b);
                            a = fmaf(bf16_lo(w8.w), bf16_lo(xv.w), a);
                            b = fmaf(bf16_hi(w8.w), bf16_hi(xv.w), b);
                            acc[t] += a + b;
                        }
                    }
                }
#pragma unroll
                for (int t = 0; t < kStepMaxRows; ++t) {
                    if (t < rows) {
                        const float v = warp_sum(acc[t]);
                        if (lane == 0)
                            st_logit(p.lw + (size_t)t * p.ld + e, v + ((e < E && p.router_bias) ? p.router_bias[e] : 0.f),
                                     tag);
                    }
                }
            }
        }
        // the unit counts of the next call start at zero: calls alternate
        // between two sets by epoch, and the call before this one (the
        // other set's last user) has finished
        if (c == 0) {
            int32_t *nxt = p.counters + kCtrStepReady + (int)((sm.epoch + 1u) & 1u) * kStepReadyHalf;
            for (int i = threadIdx.x; i < kStepReadyHalf; i += kStepWarps * kWarp) nxt[i] = 0;
        }
        named_barrier(1, kStepWarps * kWarp);  // every warp is done with the router rows
        STEP_T(3);  // router rows done
        if (threadIdx.x == 0)
            for (int ri = 0; ri < s0.n_router; ++ri) mbar_arrive(&empty[ri]);  // the router slots are free again
        if (gu_early && warp >= kIssuer0 && warp < kIssuer0 + kIssuers && lane == 0) {
            // the shared unit's MMAs (buffer 0), as the issuing loop below
            // would issue them; x's terms were fenced for the async proxy and
            // ordered by the CTA barrier above
            const int me = warp - kIssuer0;
            const uint32_t idesc = idesc_e4m3_e5m2_f32(2 * kGuRows, p.nb);
            const uint32_t xb_u32 = base + p.o_xB;
            bool ok = true;
            for (int pc = me; pc < p.gu_pieces && ok; pc += kIssuers) {
                const int q = s0.n_router + pc;
                const int s = q % p.ns;
                if (!wait_item_lane(sm.tag, full, s, q, p.ns)) {
                    gave_up(p.counters, 2, q);
                    *abort = 1;
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t sl = base + (uint32_t)s * kSlot;
                for (int wl = 0; wl < p.gu_wp; ++wl) {
                    const int W = pc * p.gu_wp + wl;
                    if (W >= hb) break;
                    const uint32_t a0 = sl + (uint32_t)wl * kGuWindow;
                    const uint32_t b0 = xb_u32 + (uint32_t)(W * p.nb * 128);
                    const uint32_t d = tmem + (uint32_t)(W * p.nb);
#pragma unroll
                    for (int k4 = 0; k4 < 4; ++k4)
                        umma_f8f6f4(d, umma_desc_sw128(a0 + 32 * k4), umma_desc_sw128(b0 + 32 * k4), idesc,
                                    k4 > 0 ? 1u : 0u);
                }
                umma_commit(&empty[s]);
            }
            if (ok) umma_commit(&tfull[0]);
        }
        // ------------------------------------------------------------ P2
        // top-k of every row, in every CTA: in two stages over all warps
        // (the k best of each chunk of 32 experts, then of the chunks'
        // candidates), or one warp per row
        if (warp == 0) STEP_T(12);
        const int nch = (E + kWarp - 1) / kWarp;
        // Each logit is read once its word carries this call's tag: no CTA
        // waits for the others beyond the logits it reads.
        const uint64_t t0 = globaltimer_ns();
        if (!*abort && p.cand2) {
            uint32_t *ckey = reinterpret_cast<uint32_t *>(sbase + p.o_cand);
            int32_t *cid = reinterpret_cast<int32_t *>(ckey + rows * nch * K);
            for (int task = warp; task < rows * nch; task += kStepWarps) {
                const int t = task / nch, ch = task - t * nch;
                const int e = ch * kWarp + lane;
                float l = 0.f;
                const bool ok = e >= E || ld_logit(p.lw + (size_t)t * p.ld + e, tag, t0, l);
                if (!__all_sync(0xFFFFFFFFu, ok)) {
                    if (lane == 0) {
                        gave_up(p.counters, 6, task);
                        *abort = 1;
                    }
                    break;
                }
                topk_chunk(e < E ? topk_key(l) : 0u, e, K, ckey + task * K, cid + task * K);
            }
            named_barrier(1, kStepWarps * kWarp);
            if (!*abort && warp < rows) {
                // the shared-gate logit (column E), by lane 0 for the warp
                float z = 0.f;
                int okz = 1;
                if (lane == 0) okz = ld_logit(p.lw + (size_t)warp * p.ld + E, tag, t0, z) ? 1 : 0;
                okz = __shfl_sync(0xFFFFFFFFu, okz, 0);
                z = __shfl_sync(0xFFFFFFFFu, z, 0);
                const int n = nch * K;
                const uint32_t *rk = ckey + warp * n;
                const int32_t *ri = cid + warp * n;
                int32_t *oi = sm.idx + warp * K;
                float *ow = sm.w + warp * K;
                float *og = sm.gs + warp;
                if (!okz) {
                    if (lane == 0) {
                        gave_up(p.counters, 6, rows * nch + warp);
                        *abort = 1;
                    }
                } else if (n <= kWarp) topk_merge<1>(rk, ri, n, z, K, oi, ow, og);
                else if (n <= 2 * kWarp) topk_merge<2>(rk, ri, n, z, K, oi, ow, og);
                else if (n <= 4 * kWarp) topk_merge<4>(rk, ri, n, z, K, oi, ow, og);
                else if (n <= 8 * kWarp) topk_merge<8>(rk, ri, n, z, K, oi, ow, og);
                else topk_merge<16>(rk, ri, n, z, K, oi, ow, og);
            }
            if (warp == 0) STEP_T(13);
        } else if (!*abort && warp < rows) {
            const uint64_t *lrow = p.lw + (size_t)warp * p.ld;
            int32_t *oi = sm.idx + warp * K;
            float *ow = sm.w + warp * K;
            float *og = sm.gs + warp;
            bool ok;
            if (E <= 32) ok = topk_select_tagged<1>(lrow, E, K, tag, t0, oi, ow, og);
            else if (E <= 64) ok = topk_select_tagged<2>(lrow, E, K, tag, t0, oi, ow, og);
            else if (E <= 128) ok = topk_select_tagged<4>(lrow, E, K, tag, t0, oi, ow, og);
            else if (E <= 256) ok = topk_select_tagged<8>(lrow, E, K, tag, t0, oi, ow, og);
            else if (E <= 512) ok = topk_select_tagged<16>(lrow, E, K, tag, t0, oi, ow, og);
            else ok = topk_select_tagged<32>(lrow, E, K, tag, t0, oi, ow, og);
            if (!ok && lane == 0) {
                gave_up(p.counters, 6, warp);
                *abort = 1;
            }
            if (warp == 0) STEP_T(13);
        }
        named_barrier(1, kStepWarps * kWarp);
        if (!*abort && warp == 0 && rows * K <= kWarp) {
            // distinct routed experts, ascending, and each pair's place in the
            // list: lane i holds pair i as (expert << 5 | i); a bitonic sort
            // across the warp orders the pairs by expert, the first pair of
            // each expert marks a list entry
            const int n = rows * K;
            uint32_t key = lane < n ? ((uint32_t)sm.idx[lane] << 5) | (uint32_t)lane : 0xFFFFFFFFu;
#pragma unroll
            for (int k2 = 2; k2 <= kWarp; k2 <<= 1) {
#pragma unroll
                for (int j = k2 >> 1; j > 0; j >>= 1) {
                    const uint32_t o = __shfl_xor_sync(0xFFFFFFFFu, key, j);
                    key = (((lane & j) == 0) == ((lane & k2) == 0)) ? min(key, o) : max(key, o);
                }
            }
            const uint32_t prev = __shfl_up_sync(0xFFFFFFFFu, key, 1);
            const bool valid = lane < n;
            const bool first = valid && (lane == 0 || (prev >> 5) != (key >> 5));
            const uint32_t firsts = __ballot_sync(0xFFFFFFFFu, first);
            const int pos = __popc(firsts & (0xFFFFFFFFu >> (31 - lane))) - 1;
            if (first) sm.list[pos] = (int32_t)(key >> 5);
            if (valid) sm.loc[key & 31u] = pos;
            if (lane == 0) sm.n_list = __popc(firsts);
            __syncwarp();
            STEP_T(14);
            if (c == 0) {
                for (int i = lane; i < rows * K; i += kWarp) {
                    p.topk_idx[i] = sm.idx[i];
                    p.topk_w[i] = sm.w[i];
                }
                if (lane < rows) p.gsig[lane] = sm.gs[lane];
            }
        } else if (!*abort && warp == 0) {
            // the same for more pairs than lanes, through a bitmask of experts
            for (int i = lane; i < kMaxExperts / 32; i += kWarp) sm.mask[i] = 0u;
            __syncwarp();
            for (int i = lane; i < rows * K; i += kWarp) atomicOr(&sm.mask[sm.idx[i] >> 5], 1u << (sm.idx[i] & 31));
            __syncwarp();
            const int nwords = (E + 31) / 32;
            int before = 0;
            for (int w0 = 0; w0 < nwords; w0 += kWarp) {
                const int wi = w0 + lane;
                const uint32_t m = wi < nwords ? sm.mask[wi] : 0u;
                const int cnt = __popc(m);
                int incl = cnt;
#pragma unroll
                for (int o = 1; o < kWarp; o <<= 1) {
                    const int y = __shfl_up_sync(0xFFFFFFFFu, incl, o);
                    if (lane >= o) incl += y;
                }
                int pos = before + incl - cnt;
                uint32_t mm = m;
                while (mm) {
                    const int b = __ffs(mm) - 1;
                    sm.list[pos++] = wi * 32 + b;
                    mm &= mm - 1;
                }
                before += __shfl_sync(0xFFFFFFFFu, incl, kWarp - 1);
            }
            if (lane == 0) sm.n_list = before;
            __syncwarp();
            STEP_T(14);
            for (int i = lane; i < rows * K; i += kWarp) {
                const int e = sm.idx[i];
                int pos = 0;
                for (int wi = 0; wi < (e >> 5); ++wi) pos += __popc(sm.mask[wi]);
                pos += __popc(sm.mask[e >> 5] & ((1u << (e & 31)) - 1u));
                sm.loc[i] = pos;
            }
            if (c == 0) {
                for (int i = lane; i < rows * K; i += kWarp) {
                    p.topk_idx[i] = sm.idx[i];
                    p.topk_w[i] = sm.w[i];
                }
                if (lane < rows) p.gsig[lane] = sm.gs[lane];
            }
        }
    }
    __syncthreads();  // the plan is ready (all 288 threads)
    STEP_T(5);
    const int U = *abort ? 0 : sm.n_list;
    const Seq seq = make_seq_k(p, sk, U);

    if (producer) {
        // ---------------------------------------------------------- producer
        // The lanes issue in parallel, lane l the items l, l + 32, ... in
        // order; item q reuses ring slot q % ns once the slot's previous item
        // (q - ns) was consumed.
        int q = fq;  // items before it were issued in P0
        // first the items that take a slot for the first time: no lane waits,
        // so none holds up the others' issue (lanes of a warp that spin in
        // different places are scheduled one path at a time); a lane's first
        // one, when a gate/up item, straight from what P0 worked out
        if (q < min(p.ns, seq.total) && fg >= 0 && fg < seq.n_gu && !*abort) {
            issue_gu(p, sm, fl, fpc, base + (uint32_t)q * kSlot, &full[q], pol, true);
            ((volatile int32_t *)sm.tag)[q] = q;
            ITEM_TL(q, 2);
            q += kWarp;
        }
        for (; q < min(p.ns, seq.total) && !*abort; q += kWarp) {
            issue_item(p, sm, item_at(p, seq, q), base + (uint32_t)q * kSlot, &full[q], r0, nr_total, tile0, nt, U,
                       pol, q);
            ((volatile int32_t *)sm.tag)[q] = q;
            ITEM_TL(q, 2);
        }
        __syncwarp();
        for (; q < seq.total && !*abort; q += kWarp) {
            const int s = q % p.ns;
            if (q >= p.ns) {
                // The slot's previous item (q - ns) belongs to another lane:
                // wait until it is issued (its tag), which proves that the
                // item before it in the slot was consumed; the parity wait
                // for its consumption is then exact (a lane running ahead
                // would otherwise see the phase two back completed).
                bool issued = ((volatile int32_t *)sm.tag)[s] == q - p.ns;
                if (!issued) {
                    const uint64_t t0 = globaltimer_ns();
                    while (!(issued = ((volatile int32_t *)sm.tag)[s] == q - p.ns))
                        if (globaltimer_ns() - t0 > kWaitLimitNs) break;
                }
                if (!issued || !mbar_wait(&empty[s], ((q / p.ns) - 1) & 1, kWaitLimitNs)) {
                    STEP_SNAP(s);
                    gave_up(p.counters, 4, q);
                    *abort = 1;
                    break;
                }
                fence_proxy_async_smem();
            }
            issue_item(p, sm, item_at(p, seq, q), base + (uint32_t)s * kSlot, &full[s], r0, nr_total, tile0, nt, U,
                       pol, q);
            ((volatile int32_t *)sm.tag)[s] = q;
            ITEM_TL(q, 2);
        }
        // every issued copy lands before the CTA may leave: the last item
        // issued into each slot (all of them were consumed on the normal path)
        __syncwarp();
        if (lane == 0) {
            for (int sl = 0; sl < p.ns; ++sl) {
                const int t = ((volatile int32_t *)sm.tag)[sl];
                if (t >= 0) mbar_wait(&full[sl], (t / p.ns) & 1, kWaitLimitNs);
            }
        }
        return;
    }

    // ---------------------------------------------------------------- consumers
    const float *xfac = reinterpret_cast<const float *>(sbase + p.o_xfac);

    // Block scales of this CTA's work into shared memory, one round trip for
    // all of them (the weight copies are in flight meanwhile), by the
    // epilogue warps 0-3 (the issuing warps need none and start their MMAs
    // at once): per local gate/up unit its gate and up row blocks [2][H/128];
    // per down expert (shared first, then the routed list) the row blocks of
    // this CTA's output rows [2][Iu/128].  The down items of warps 4-7 read
    // the latter after thread 0's release below.
    float *gsc = reinterpret_cast<float *>(sbase + p.o_gsc);
    float *dsc = reinterpret_cast<float *>(sbase + p.o_dsc);
    const int ibm = p.imax / 128;
    const int rb0 = (tile0 * 8) / 128;
    if (warp < 4) {
        const int ng = seq.n_units_local * 2 * hb;
        const int nd = nt > 0 ? (U + 1) * 2 * ibm : 0;
        for (int i = threadIdx.x; i < ng + nd; i += 4 * kWarp) {
            if (i < ng) {
                const int l = i / (2 * hb), rem = i - l * 2 * hb, half = rem / hb, W = rem - half * hb;
                bool shared;
                int e, j;
                unit_of(p, sm, c + l * G, shared, e, j);
                const int Iu = shared ? p.Is : p.I;
                const float *sc = shared ? p.sscales
                                         : p.scales + (size_t)e * ((size_t)(2 * Iu / 128) * hb + (size_t)hb * (Iu / 128));
                gsc[i] = __ldg(sc + (size_t)((half ? Iu + j : j) / 128) * hb + W);
            } else {
                const int k = i - ng;
                const int de = k / (2 * ibm), rem = k - de * 2 * ibm, rb = rem / ibm, W = rem - rb * ibm;
                const bool shared = de == 0;
                const int e = shared ? 0 : sm.list[de - 1];
                const int Iu = shared ? p.Is : p.I;
                const int ibu = Iu / 128;
                float v = 0.f;
                if (W < ibu && rb0 + rb < H / 128) {
                    const float *s2 = (shared ? p.sscales
                                              : p.scales + (size_t)e * ((size_t)(2 * Iu / 128) * hb + (size_t)hb * ibu)) +
                                      (size_t)(2 * Iu / 128) * hb;
                    v = __ldg(s2 + (size_t)(rb0 + rb) * ibu + W);
                }
                dsc[k] = v;
            }
        }
        named_barrier(5, 4 * kWarp);
        if (threadIdx.x == 0) st_release_cta_shared(&sm.dsc_ready, 1);  // (the barrier ordered warps 0-3's writes)
    }

    // gate/up on the tensor cores.  Four issuing threads take, per local unit, the MMAs
    // of its items as their copies land: A = the unit's 32 gate and 32 up
    // rows of one K window (e4m3), B = the x terms (e5m2), K = 32 an
    // instruction, one fp32 accumulator of nb columns per K window (each
    // window has its own block scales); it commits them to the slot's empty
    // barrier, so the producer may refill the slot once they are done, and
    // after the unit's last item to the unit's accumulator buffer.  Warps
    // 0-3 then read the buffer (unit row m sits in tensor-memory lane
    // m % 16 + 32 (m / 16)), add each row of x's three term columns, scale
    // and add the K windows in order, and write h = silu(gate) * up.  With
    // two buffers the next unit's MMAs run during an epilogue.
    {
        const uint32_t xb_u32 = base + p.o_xB;
        if (warp >= kIssuer0 && warp < kIssuer0 + kIssuers) {
            if (lane == 0) {
                const int me = warp - kIssuer0;
                const uint32_t idesc = idesc_e4m3_e5m2_f32(2 * kGuRows, p.nb);
                for (int l = gu_early ? 1 : 0; l < seq.n_units_local && !*abort; ++l) {  // (unit 0 went out early)
                    const int b = l % p.nbuf, kk = l / p.nbuf;
                    if (kk >= 1 && !mbar_wait_spin(&tfree[b], (uint32_t)((kk - 1) & 1), kWaitLimitNs)) {
                        gave_up(p.counters, 8, l);
                        *abort = 1;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t dbase = tmem + (uint32_t)(b * p.tbuf);
                    bool ok = true;
                    for (int pc = me; pc < p.gu_pieces; pc += kIssuers) {
                        const int q = seq.n_router + l * p.gu_pieces + pc;
                        const int s = q % p.ns;
                        STEP_MARK(2, q);
                        if (!wait_item_lane(sm.tag, full, s, q, p.ns)) {
                            STEP_SNAP(s);
                            gave_up(p.counters, 2, q);
                            *abort = 1;
                            ok = false;
                            break;
                        }
                        ITEM_T(q, 0);
                        if (q == seq.n_router) STEP_T(6);  // the first gate/up item landed
                        tc_fence_after();
                        const uint32_t sl = base + (uint32_t)s * kSlot;
                        for (int wl = 0; wl < p.gu_wp; ++wl) {
                            const int W = pc * p.gu_wp + wl;
                            if (W >= hb) break;
                            const uint32_t a0 = sl + (uint32_t)wl * kGuWindow;
                            const uint32_t b0 = xb_u32 + (uint32_t)(W * p.nb * 128);
                            const uint32_t d = dbase + (uint32_t)(W * p.nb);
#pragma unroll
                            for (int k4 = 0; k4 < 4; ++k4)
                                umma_f8f6f4(d, umma_desc_sw128(a0 + 32 * k4), umma_desc_sw128(b0 + 32 * k4), idesc,
                                            k4 > 0 ? 1u : 0u);
                        }
                        umma_commit(&empty[s]);
                        ITEM_T(q, 1);
                    }
                    if (!ok) break;
                    umma_commit(&tfull[b]);
                }
                umma_commit(tdone);  // also with nothing issued: the barrier then completes at once
            }
            __syncwarp();
        } else if (warp < 4) {
            const int m = lane + 16 * warp;  // the unit row of this lane (lanes 0-15)
            const bool gate = warp < 2;
            // one thread waits for each unit and tells the four warps through
            // a flag only it writes, so that they leave the loop together
            // (the loop holds named barriers)
            for (int l = 0; l < seq.n_units_local; ++l) {
                const int b = l % p.nbuf, kk = l / p.nbuf;
                // the unit and its rows' slots of h while its MMAs run
                bool shared;
                int e, j;
                unit_of(p, sm, c + l * G, shared, e, j);
                int slots[kStepMaxRows];
#pragma unroll
                for (int t = 0; t < kStepMaxRows; ++t) {
                    slots[t] = -1;
                    if (t >= rows) continue;
                    if (shared) {
                        slots[t] = rows * K + t;
                    } else {
                        for (int r = 0; r < K; ++r)
                            if (sm.idx[t * K + r] == e) slots[t] = t * K + r;
                    }
                }
                if (threadIdx.x == kEpiWaiter) {
                    const bool ok = !*abort && mbar_wait_spin(&tfull[b], (uint32_t)(kk & 1), kWaitLimitNs);
                    if (!ok) {
                        if (!*abort) gave_up(p.counters, 9, l);
                        *abort = 1;
                    }
                    sm.gu_stop = ok ? 0 : 1;
                }
                named_barrier(3, 4 * kWarp);
                if (sm.gu_stop) break;
                tc_fence_after();
                const float *srow = gsc + (size_t)l * 2 * hb + (gate ? 0 : hb);
                float acc[kStepMaxRows];
                const uint32_t tb = tmem + (uint32_t)(b * p.tbuf) + ((uint32_t)(32 * warp) << 16);
                if (p.nb == 8) gu_row_sums<8>(tb, hb, rows, srow, xfac, acc);
                else gu_row_sums<16>(tb, hb, rows, srow, xfac, acc);
                // the up rows' sums to the gate rows' lanes
                if (!gate && lane < 16) {
#pragma unroll
                    for (int t = 0; t < kStepMaxRows; ++t) sm.xch[(m - kGuRows) * kStepMaxRows + t] = acc[t];
                }
                tc_fence_before();
                named_barrier(3, 4 * kWarp);
                if (gate) {
                    // h = silu(gate) * up for the rows routed to this expert
                    // (lanes 0-15 of both warps: the unit's 32 values, one K
                    // chunk of the down MMAs), as eight e5m2 terms: a power of
                    // two puts the chunk's largest |h| in [2^14, 2^15), and
                    // t_k = e5m2(h' - t_1 - ... - t_(k-1)) (differences exact in
                    // fp32) sum to h' exactly for every value within 2^7 of that
                    // maximum and to within 2^-31 of it below.  Term k of value
                    // m goes where the down MMA's B registers want it: byte
                    // (m % 4) + 4 (m / 16) of lane 4k + (m % 16) / 4's eight.
                    float hv[kStepMaxRows];
#pragma unroll
                    for (int t = 0; t < kStepMaxRows; ++t) {
                        hv[t] = 0.f;
                        if (t >= rows) continue;
                        if (slots[t] >= 0 && lane < 16) hv[t] = siluf_(acc[t]) * sm.xch[m * kStepMaxRows + t];
                        const float mx = warp_max(fabsf(hv[t]));
                        if (lane == 0) sm.hmx[warp * kStepMaxRows + t] = mx;
                    }
                    named_barrier(2, 2 * kWarp);  // both gate warps' maxima
                    const int ntc = p.imax / 32;
#pragma unroll
                    for (int t = 0; t < kStepMaxRows; ++t) {
                        if (t >= rows || slots[t] < 0) continue;  // the same in every lane
                        const int sh = block_shift(fmaxf(sm.hmx[t], sm.hmx[kStepMaxRows + t]));
                        float x = hv[t] * pow2f(sh);
                        unsigned char *dst = p.hterm + ((size_t)slots[t] * ntc + j / 32) * 256 + (lane >> 2) * 8 +
                                             warp * 4 + (lane & 3);
#pragma unroll
                        for (int k = 0; k < 8; ++k) {
                            const uint32_t c = f32x2_to_e5m2x2(x, 0.f);
                            x -= e5m2x2_to_f32x2(c).x;
                            if (lane < 16) dst[k * 32] = (unsigned char)(c & 0xFFu);
                        }
                        if (warp == 0 && lane == 0) p.hsc[(size_t)slots[t] * ntc + j / 32] = pow2f(-sh);
                    }
                }
                named_barrier(3, 4 * kWarp);  // the exchange slots are free again
                if (lane == 0) mbar_arrive(&tfree[b]);
                if (threadIdx.x == kEpiWaiter) {
                    // this unit's h before its count for the expert: the
                    // releasing add is cumulative over both warps' h writes,
                    // which the named barrier above ordered before it; the
                    // down items of every CTA wait for their expert's full
                    // count with acquiring loads
                    const int u = c + l * G, us = p.Is / kGuRows;
                    const int de = u < us ? 0 : 1 + (u - us) / (p.I / kGuRows);
                    red_release_gpu(p.counters + kCtrStepReady + (int)(sm.epoch & 1u) * kStepReadyHalf + de * p.rdy, 1);
                    STEP_TL(15);  // (trace) this CTA's last unit counted
                }
            }
        }
        // every gate/up MMA done (before P3 reuses the x-term region and the
        // accumulator columns)
        if (warp == 0) {
            if (lane == 0 && !mbar_wait(tdone, 0, kWaitLimitNs)) {
                gave_up(p.counters, 10, 0);
                *abort = 1;
            }
            __syncwarp();
            tc_fence_after();
            tmem_dealloc(tmem, (uint32_t)p.tcols);
        }
    }
    float *ybuf = reinterpret_cast<float *>(sbase + p.o_y);  // [U + 1][rows][nt_max * 8]
    STEP_MARK(6, 0);
    STEP_T(7);  // warp 0's gate/up items done
    pdl_trigger();  // this CTA's weight reads are all issued: the next kernel may start

    // ---------------------------------------------------------------- P3
    // No grid barrier: down items claimed by the warps as they come free
    // (down_phase).
    STEP_T(8);  // P3 starts
    down_phase(p, sm, sbase, base, full, empty, tdone, bbars, seq, nt, tile0, rb0, ibm, dsc, ybuf, abort);
    named_barrier(1, kStepWarps * kWarp);  // every down item of the CTA done
    // (thread 0) the last CTA to have read the epoch advances it and resets
    // the count for the next call, which reads both only after its PDL wait,
    // that is after this grid has finished
    if (threadIdx.x == 0 && exit_old == G - 1) {
        p.counters[kCtrStepExit] = 0;
        p.counters[kCtrStepEpoch] = (int32_t)(sm.epoch + 1u);
    }
    if (*abort) return;

    STEP_T(10);  // down items done
    // blend: rank order, then the shared expert, then the residual; one rounding
    const int yrow = p.nt_max * 8;
    for (int u = threadIdx.x; u < rows * nt * 8; u += kStepWarps * kWarp) {
        const int t = u / (nt * 8), nn = u - t * (nt * 8);
        float acc = 0.f;
        for (int r = 0; r < K; ++r) acc = fmaf(sm.w[t * K + r], ybuf[((size_t)(1 + sm.loc[t * K + r]) * rows + t) * yrow + nn], acc);
        acc = fmaf(sm.gs[t], ybuf[(size_t)t * yrow + nn], acc);
        const size_t o = (size_t)t * H + (size_t)tile0 * 8 + nn;
        if (p.residual) acc += bf16_bits_to_f32(p.residual[o]);
        p.out[o] = f32_to_bf16_bits(acc);
    }
    STEP_T(11);
}

// ------------------------------------------------------------ host side

std::mutex g_mu;

bool configured_for(int dev)
{
    static bool done[64] = {};
    std::lock_guard<std::mutex> lk(g_mu);
    if (dev < 0 || dev >= 64) return false;
    if (!done[dev]) {
        if (cudaFuncSetAttribute(decode_step_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemCap) !=
            cudaSuccess)
            return false;
        done[dev] = true;
    }
    return true;
}

// W13 of one expert slab [gate rows | up rows][windows of 128 bytes] (inter
// rows each) as a 5-D TMA map over (128 bytes, rows, gate|up, windows,
// experts) with 128-byte-swizzled boxes {128, 32, 2, box_windows, 1}: a box
// lands as [window][gate 32 rows, up 32 rows][128 bytes].
bool make_map_gate_up(CUtensorMap *m, const void *base, uint64_t inter, uint64_t kbytes, uint64_t experts,
                      uint64_t expert_stride, uint32_t box_windows)
{
    using EncodeFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
    static EncodeFn fn = [] {
        void *f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return static_cast<EncodeFn>(nullptr);
        return reinterpret_cast<EncodeFn>(f);
    }();
    if (!fn) return false;
    const cuuint64_t dims[5] = {128, inter, 2, kbytes / 128, experts};
    const cuuint64_t strides[4] = {kbytes, inter * kbytes, 128, expert_stride ? expert_stride : 3 * inter * kbytes};
    const cuuint32_t box[5] = {128, (cuuint32_t)kGuRows, 2, box_windows, 1};
    const cuuint32_t estr[5] = {1, 1, 1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 5, const_cast<void *>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// W2 of the expert slabs [H rows][inter bytes] as a 5-D TMA map over (128
// bytes, 8 rows, H/8 tiles, windows, experts) with 128-byte-swizzled boxes
// {128, 8, tiles, inter/128, 1}: a box lands as [window][tile][8 rows][128 B].
bool make_map_down(CUtensorMap *m, const void *base, uint64_t hidden, uint64_t inter, uint64_t experts,
                   uint64_t expert_stride, uint32_t tiles)
{
    using EncodeFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
    static EncodeFn fn = [] {
        void *f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return static_cast<EncodeFn>(nullptr);
        return reinterpret_cast<EncodeFn>(f);
    }();
    if (!fn) return false;
    const cuuint64_t dims[5] = {128, 8, hidden / 8, inter / 128, experts};
    const cuuint64_t strides[4] = {inter, 8 * inter, 128, expert_stride ? expert_stride : 3 * inter * hidden};
    const cuuint32_t box[5] = {128, 8, tiles, (cuuint32_t)(inter / 128), 1};
    const cuuint32_t estr[5] = {1, 1, 1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 5, const_cast<void *>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

StepShape step_shape(const moe_dims &d, int rows, int sms)
{
    StepShape s{};
    const int H = d.hidden, I = d.inter, Is = d.shared_inter, K = d.top_k;
    const int imax = std::max(I, Is);
    const int G = std::max(1, sms);
    s.grid = G;
    // gate/up items: two K windows of a unit's 64 rows (16 KB)
    s.gu_wp = 2;
    s.gu_pieces = (H / 128 + s.gu_wp - 1) / s.gu_wp;
    // gate/up MMA N: three x terms per row, in 8 or 16 columns; one
    // accumulator of nb columns per K window, two buffers when they fit in
    // the 512 columns of tensor memory
    s.nb = 3 * rows <= 8 ? 8 : 16;
    s.tbuf = (H / 128) * s.nb;
    s.nbuf = 2 * s.tbuf <= 512 ? 2 : 1;
    s.tcols = 32;
    while (s.tcols < s.nbuf * s.tbuf) s.tcols *= 2;
    const int n8 = H / 8;
    s.nt_max = (n8 + G - 1) / G;
    // down items: the full K of one or two output tiles of one expert (one
    // 5-D box, [window][tile][8 rows][128 B])
    s.dn_tpi = 2 * 8 * I <= kSlot ? 2 : 1;
    s.dn_tpi_s = 2 * 8 * Is <= kSlot ? 2 : 1;
    s.dn_epi = 1;
    s.rr_per_item = std::max(1, kSlot / (2 * H));
    // shared memory, after the ring
    s.x_stride = H + 8;
    const size_t xbytes = (size_t)rows * s.x_stride * 2;
    const int umax = std::min(d.n_experts, rows * K);
    // the down experts' unit counters, one 128-byte line each where they fit
    s.rdy = 32;
    while (s.rdy > 1 && (rows * K + 1) * s.rdy > kStepReadyHalf) s.rdy /= 2;
    size_t o = 0;
    auto take = [&](size_t b) { size_t at = o; o = align_up(o + b, 16); return (uint32_t)at; };
    const size_t xBbytes = (size_t)(H / 128) * s.nb * 128;
    // x terms, then bf16 x; in P3 the consumer warps' buffers of h terms (16
    // chunks of 256 bytes each)
    const uint32_t uni = take(std::max(xBbytes + xbytes, (size_t)kStepWarps * 16 * 256));
    const uint32_t xfac = take((size_t)rows * (H / 128) * 4);
    const uint32_t y = take((size_t)(umax + 1) * rows * s.nt_max * 8 * 4);
    const int64_t units_max = Is / kGuRows + (int64_t)umax * (I / kGuRows);
    s.max_units = (int)((units_max + G - 1) / G);
    const uint32_t gsc = take((size_t)s.max_units * 2 * (H / 128) * 4);
    const uint32_t dsc = take((size_t)(umax + 1) * 2 * (imax / 128) * 4);
    // two-stage top-k: more than one chunk of 32 experts, at most 16
    // candidates a lane in the second stage
    const int nch = (d.n_experts + kWarp - 1) / kWarp;
    s.cand2 = nch > 1 && nch * K <= 16 * kWarp;
    const uint32_t cand = take(s.cand2 ? (size_t)rows * nch * K * 8 : 0);
    const uint32_t smo = take(sizeof(StepSmall));
    const size_t tail = o;
    // ring slots: whatever is left, up to 16
    const size_t avail = (size_t)kSmemCap - 1024 - tail - (16 * 2 + 16) * 8;
    s.ns = (int)std::min<size_t>(16, avail / kSlot);
    const uint32_t ring = (uint32_t)s.ns * kSlot;
    s.o_uni = ring + uni;  // 1024-aligned: the ring is a multiple of 16 KB and uni comes first
    s.o_xB = ring + uni;
    s.o_xb = ring + uni + (uint32_t)xBbytes;
    s.o_xfac = ring + xfac;
    s.o_y = ring + y;
    s.o_gsc = ring + gsc;
    s.o_dsc = ring + dsc;
    s.o_cand = ring + cand;
    s.o_sm = ring + smo;
    s.o_bar = (uint32_t)align_up(ring + tail, 8);
    s.smem = s.o_bar + (2 * s.ns + 16) * 8 + 1024;
    // the router items all sit in the ring before the first slot is reused
    const int rr_max = (d.n_experts + 1 + G - 1) / G;
    const int router_items = (rr_max + s.rr_per_item - 1) / s.rr_per_item;
    s.ok = s.ns >= 2 && s.ns > router_items && s.nt_max <= kMaxNt && s.smem <= kSmemCap && 2 * H <= kSlot &&
           8 * I <= kSlot && 8 * Is <= kSlot && 3 * rows <= 16 && s.tbuf <= 512 && I % kGuRows == 0 &&
           Is % kGuRows == 0 && (rows * K + 1) * s.rdy <= kStepReadyHalf;
    return s;
}

int step_rows_per_launch(const moe_dims &d, int sms)
{
    for (int r = kStepMaxRows; r >= 1; --r) {
        const StepShape s = step_shape(d, r, sms);
        if (s.ok && s.ns >= 4) return r;
    }
    return step_shape(d, 1, sms).ok ? 1 : 0;
}

cudaError_t launch_decode_step(const StepLaunch &a, cudaStream_t st)
{
    const moe_dims &d = *a.d;
    const DeviceInfo &di = device_info();
    int dev = 0;
    cudaGetDevice(&dev);
    if (!configured_for(dev)) return cudaErrorInvalidConfiguration;
    const StepShape sh = step_shape(d, a.rows, di.sm_count);
    if (!sh.ok || a.rows < 1 || a.rows > kStepMaxRows) return cudaErrorInvalidConfiguration;
    const int H = d.hidden, I = d.inter, Is = d.shared_inter, E = d.n_experts;
    StepParams p;
    if (!make_map_gate_up(&p.w13, a.expert_w8, (uint64_t)I, (uint64_t)H, (uint64_t)E, 3 * (uint64_t)I * H,
                          (uint32_t)sh.gu_wp) ||
        !make_map_gate_up(&p.w13s, a.shared_w8, (uint64_t)Is, (uint64_t)H, 1, 0, (uint32_t)sh.gu_wp) ||
        !make_map_down(&p.w2, a.expert_w8 + (size_t)2 * I * H, (uint64_t)H, (uint64_t)I, (uint64_t)E,
                       3 * (uint64_t)I * H, (uint32_t)sh.dn_tpi) ||
        !make_map_down(&p.w2s, a.shared_w8 + (size_t)2 * Is * H, (uint64_t)H, (uint64_t)Is, 1, 0,
                       (uint32_t)sh.dn_tpi_s))
        return cudaErrorInvalidValue;
    p.x = a.x;
    p.router_w = a.router_w;
    p.shared_gate = a.shared_gate;
    p.residual = a.residual;
    p.router_bias = a.router_bias;
    p.scales = a.expert_scales;
    p.sscales = a.shared_scales;
    p.norm_w = a.norm_w;
    p.eps = a.eps;
    p.out = a.out;
    p.topk_idx = a.topk_idx;
    p.topk_w = a.topk_w;
    p.gsig = a.gsig;
    p.lw = reinterpret_cast<uint64_t *>(a.counters + kCtrStepLogits);
    p.hterm = a.hterm;
    p.hsc = a.hsc;
    p.counters = a.counters;
    p.rows = a.rows;
    p.H = H;
    p.E = E;
    p.K = d.top_k;
    p.I = I;
    p.Is = Is;
    p.ld = a.logits_ld;
    p.imax = std::max(I, Is);
    p.ns = sh.ns;
    p.gu_wp = sh.gu_wp;
    p.gu_pieces = sh.gu_pieces;
    p.dn_tpi = sh.dn_tpi;
    p.dn_tpi_s = sh.dn_tpi_s;
    p.dn_epi = sh.dn_epi;
    p.nt_max = sh.nt_max;
    p.rr_per_item = sh.rr_per_item;
    p.o_uni = sh.o_uni;
    p.o_xb = sh.o_xb;
    p.o_xfac = sh.o_xfac;
    p.o_y = sh.o_y;
    p.rdy = sh.rdy;
    p.o_gsc = sh.o_gsc;
    p.o_dsc = sh.o_dsc;
    p.o_xB = sh.o_xB;
    p.nb = sh.nb;
    p.nbuf = sh.nbuf;
    p.tbuf = sh.tbuf;
    p.tcols = sh.tcols;
    p.o_cand = sh.o_cand;
    p.cand2 = sh.cand2 ? 1 : 0;
    p.max_units = sh.max_units;
    p.o_sm = sh.o_sm;
    p.o_bar = sh.o_bar;
    p.x_stride = sh.x_stride;
    return launch_kernel(decode_step_kernel, dim3(sh.grid), dim3(kStepThreads), sh.smem, st, p);
}

}  // namespace moe

#ifdef MOE_STEP_TRACE
extern "C" MOE_API int moe_debug_item_trace(void *host, void *stream)
{
    cudaError_t e = cudaMemcpyFromSymbolAsync(host, moe::g_item_trace, sizeof(moe::g_item_trace), 0,
                                              cudaMemcpyDeviceToHost, static_cast<cudaStream_t>(stream));
    if (e == cudaSuccess) e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? 0 : -4;
}

extern "C" MOE_API int moe_debug_step_trace(void *host, void *stream)
{
    cudaError_t e = cudaMemcpyFromSymbolAsync(host, moe::g_step_trace, sizeof(moe::g_step_trace), 0,
                                              cudaMemcpyDeviceToHost, static_cast<cudaStream_t>(stream));
    if (e == cudaSuccess) e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? 0 : -4;
}
#endif
