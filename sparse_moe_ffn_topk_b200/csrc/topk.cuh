// topk.cuh -- top-k softmax of router logits, shared by the router kernel
// and the decode step kernel.
#pragma once

#include "common.cuh"

namespace moe {

// The k largest of a warp's keys.  Lane L holds EPL (key, expert) pairs in
// the order of its candidates; keys are order-preserving (larger = larger
// logit), 0 marks an absent candidate, and candidates with equal keys are
// held in ascending expert order (within a lane, and lane by lane).  Each lane
// sorts its pairs once (a stable sort), then each round takes the best head
// across the warp (equal heads: the lower lane) and the winning lane pops it.
// Lane r < k ends with the r-th largest: my_k its key, my_e its expert.
template <int EPL>
__device__ __forceinline__ void topk_rounds(uint32_t (&v)[EPL], int (&id)[EPL], int K, int &my_e, uint32_t &my_k)
{
    const int lane = threadIdx.x & 31;
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
    my_e = 0;
    my_k = 0;
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
}

// Softmax over the k chosen (lane r < k holds the r-th largest) and the
// shared-expert gate: out_idx[r], out_w[r], *out_gsig = sigmoid(z).
__device__ __forceinline__ void topk_finish(int K, int my_e, uint32_t my_k, float z, int32_t *out_idx, float *out_w,
                                            float *out_gsig)
{
    const int lane = threadIdx.x & 31;
    const float my_v = (my_k == 1u) ? __int_as_float(0x7FC00000) : key_value(my_k);
    const float top = __shfl_sync(0xFFFFFFFFu, my_v, 0);
    const float ev = (lane < K) ? expf(my_v - top) : 0.f;
    const float sum = warp_sum(ev);
    if (lane < K) {
        out_idx[lane] = my_e;
        out_w[lane] = ev / sum;
    }
    if (lane == 0) *out_gsig = sigmoidf_(z);
}

// Top-k of one row from its keys (one warp): lane L holds the keys of the
// experts L*EPL .. L*EPL+EPL-1 in v (0 for absent ones) and their ids, z is
// the shared-gate logit.
template <int EPL>
__device__ __forceinline__ void topk_select_keys(uint32_t (&v)[EPL], int (&id)[EPL], float z, int K,
                                                 int32_t *out_idx, float *out_w, float *out_gsig)
{
    int my_e;
    uint32_t my_k;
    topk_rounds<EPL>(v, id, K, my_e, my_k);
    topk_finish(K, my_e, my_k, z, out_idx, out_w, out_gsig);
}

// Top-k of one row of logits (one warp): lane L holds the experts
// L*EPL .. L*EPL+EPL-1.  A NaN logit gets key 1, so the selection always
// returns valid experts.
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
    topk_select_keys<EPL>(v, id, z, K, out_idx, out_w, out_gsig);
}

// Two-stage top-k for a CTA's warps.  Stage 1 (one warp per chunk of 32
// experts): the chunk's k best, best first, as (key, expert) candidates.
// Stage 2 (one warp per row, topk_merge): the k best of the row's chunk
// candidates, taken in chunk order.  Equal keys keep ascending expert order
// through both stages (a chunk's candidates of equal key come out by lane,
// and lower chunks hold lower experts), so the result is the one-warp
// selection's.
//
// Stage 1 for one chunk: lane L holds the key of expert e = chunk * 32 + L
// (0 when absent).
__device__ __forceinline__ void topk_chunk(uint32_t key, int e, int K, uint32_t *ckey, int32_t *cid)
{
    const int lane = threadIdx.x & 31;
    for (int r = 0; r < K; ++r) {
        const uint32_t kmax = __reduce_max_sync(0xFFFFFFFFu, key);
        const int wl = __ffs(__ballot_sync(0xFFFFFFFFu, key == kmax)) - 1;
        if (lane == wl) {
            ckey[r] = key;
            cid[r] = e;
            key = 0u;
        }
    }
}

// Stage 2 over n = chunks * k candidates: lane L takes candidates
// L*CPL .. L*CPL+CPL-1 (n <= 32 * CPL); z is the shared-gate logit.
template <int CPL>
__device__ void topk_merge(const uint32_t *ckey, const int32_t *cid, int n, float z, int K, int32_t *out_idx,
                           float *out_w, float *out_gsig)
{
    const int lane = threadIdx.x & 31;
    uint32_t v[CPL];
    int id[CPL];
#pragma unroll
    for (int i = 0; i < CPL; ++i) {
        const int c = lane * CPL + i;
        v[i] = c < n ? ckey[c] : 0u;
        id[i] = c < n ? cid[c] : 0;
    }
    topk_select_keys<CPL>(v, id, z, K, out_idx, out_w, out_gsig);
}

}  // namespace moe
