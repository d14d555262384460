// Warp-level top-k selection shared by the decode kernel and the batched router.
#pragma once

#include "common.cuh"
#include "internal.h"

namespace redmoe {

// ---------------------------------------------------------------- top-k
// Top-k of one token's E logits by one warp: each lane keeps order keys of experts
// lane, lane + 32, ...; k rounds of (warp max key, lowest id among the lanes holding it).
// Writes ids and renormalised weights w_j = exp(l_j - l_0) / sum_j' exp(l_j' - l_0).
__device__ __forceinline__ void warp_topk(const float* logits, int E, int k, int* ids, float* wts) {
    const int lane = threadIdx.x & 31;
    constexpr int EPL = MAX_EXPERTS / 32;
    uint32_t key[EPL];
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
        const int e = i * 32 + lane;
        key[i] = (e < E) ? order_key(__ldcg(logits + e)) : 0u;
    }
    const int nit = (E + 31) / 32;
    uint32_t best = 0u;
    int bi = 0;
#pragma unroll
    for (int i = 0; i < EPL; ++i)
        if (i < nit && key[i] > best) { best = key[i]; bi = i; }
    float mylogit = 0.0f;
    int myid = 0;
    for (int j = 0; j < k; ++j) {
        const uint32_t m = __reduce_max_sync(FULL, best);
        const uint32_t cand = (best == m) ? uint32_t(bi * 32 + lane) : 0xffffffffu;
        const uint32_t win = __reduce_min_sync(FULL, cand);
        if (lane == j) { myid = int(win); mylogit = key_to_float(m); }
        if (lane == int(win & 31u)) {
#pragma unroll
            for (int i = 0; i < EPL; ++i)
                if (i == bi) key[i] = 0u;
            best = 0u;
            bi = 0;
#pragma unroll
            for (int i = 0; i < EPL; ++i)
                if (i < nit && key[i] > best) { best = key[i]; bi = i; }
        }
    }
    const float l0 = __shfl_sync(FULL, mylogit, 0);
    const float ex = (lane < k) ? expf(mylogit - l0) : 0.0f;
    const float sum = warp_sum(ex);
    if (lane < k) {
        ids[lane] = myid;
        wts[lane] = ex / sum;
    }
}

}  // namespace redmoe
