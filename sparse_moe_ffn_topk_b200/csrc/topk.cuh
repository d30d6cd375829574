// topk.cuh -- top-k softmax of one row of router logits (one warp), shared
// by the router kernel and the decode step kernel.
#pragma once

#include "common.cuh"

namespace moe {

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

}  // namespace moe
