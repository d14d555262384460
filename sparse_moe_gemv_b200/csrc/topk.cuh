// Warp-level top-k selection shared by the decode kernel and the batched router.
#pragma once

#include "common.cuh"
#include "internal.h"

namespace redmoe {

// Top-k of one token's E logits by one warp, ties to the lower expert id.
//
// The logits arrive as order-preserving integer keys (`keys`, E entries in shared
// memory); lane L holds the keys of experts L, L + 32, ... in registers. Each of the k
// rounds takes the warp-wide largest key (redux.sync max), breaks ties by the lowest
// expert id (redux.sync min over the candidates), and lets the owning lane drop that key
// and rescan its own registers.
//
// Writes ids[0..k) and the renormalised weights w_j = exp(l_j - l_0) / sum_j' exp(l_j' - l_0)
// (the softmax over all experts, restricted to the selection and renormalised, equals the
// softmax over the selected logits).
//
// warp_topk_core takes the keys in registers (key[i] of lane L is expert i * 32 + L, 0 past
// E) and leaves the j-th selection in lane j (< k): its id and its weight.
template <int EPL>
__device__ __forceinline__ void warp_topk_core(uint32_t (&key)[EPL], int k, int& out_id, float& out_w) {
    const int lane = threadIdx.x & 31;
    uint32_t best = 0u;
    int bi = 0;
#pragma unroll
    for (int i = 0; i < EPL; ++i)
        if (key[i] > best) { best = key[i]; bi = i; }
    float mylogit = 0.0f;
    int myid = 0;
#pragma unroll 1
    for (int j = 0; j < k; ++j) {
        const uint32_t m = __reduce_max_sync(FULL, best);
        const uint32_t win = __reduce_min_sync(FULL, best == m ? uint32_t(bi * 32 + lane) : 0xffffffffu);
        if (lane == j) { myid = int(win); mylogit = key_to_float(m); }
        if (lane == int(win & 31u)) {
            best = 0u;
            const int drop = bi;
            bi = 0;
#pragma unroll
            for (int i = 0; i < EPL; ++i) {
                if (i == drop) key[i] = 0u;
                if (key[i] > best) { best = key[i]; bi = i; }
            }
        }
    }
    const float l0 = __shfl_sync(FULL, mylogit, 0);
    const float ex = (lane < k) ? expf(mylogit - l0) : 0.0f;
    const float sum = warp_sum(ex);
    out_id = myid;
    out_w = ex / sum;
}

template <int EPL>
__device__ __forceinline__ void warp_topk_reg(int E, int k, const uint32_t* keys, int* ids, float* wts) {
    const int lane = threadIdx.x & 31;
    uint32_t key[EPL];
#pragma unroll
    for (int i = 0; i < EPL; ++i) key[i] = (i * 32 + lane < E) ? keys[i * 32 + lane] : 0u;
    int id;
    float wv;
    warp_topk_core<EPL>(key, k, id, wv);
    if (lane < k) {
        ids[lane] = id;
        wts[lane] = wv;
    }
}

// The keys are read once into registers (EPL per lane); `keys` is not modified.
__device__ __forceinline__ void warp_topk_keys(int E, int k, const uint32_t* keys, int* ids, float* wts) {
    if (E <= 256) warp_topk_reg<8>(E, k, keys, ids, wts);
    else if (E <= 512) warp_topk_reg<16>(E, k, keys, ids, wts);
    else warp_topk_reg<MAX_EXPERTS / 32>(E, k, keys, ids, wts);
}

// Same, loading the logits (global memory written earlier) into the key buffer first.
__device__ __forceinline__ void warp_topk(const float* logits, int E, int k, uint32_t* keys, int* ids, float* wts) {
    const int lane = threadIdx.x & 31;
#pragma unroll 8
    for (int e = lane; e < E; e += 32) keys[e] = order_key(__ldcg(logits + e));
    __syncwarp();
    warp_topk_keys(E, k, keys, ids, wts);
}

}  // namespace redmoe
