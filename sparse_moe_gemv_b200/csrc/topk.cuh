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

// Top-k of one token's E logits (global memory written earlier in the launch) by one warp,
// optionally with the opt-in cache-aware routing bias ("Research notes, October 2026",
// section 4: z + lambda * Delta * cached, opt-in because it changes outputs). With
// cached != nullptr the selection ranks z[e] + lambda * Delta * cached[e], Delta the
// token's logit range (max - min over the E logits), ties to the lower id; the weights are
// the softmax of the unbiased logits over the selected experts (the bias changes which
// experts run, not how their outputs are mixed). Lane j < k ends with (id_j, w_j).
// The same from logits already in registers: z[i] of lane L is expert i * 32 + L (any
// value past E; it is not selected).
template <int EPL>
__device__ __forceinline__ void warp_route_z(const float (&z)[EPL], int E, int k, const uint8_t* cached, float lambda,
                                             int& out_id, float& out_w) {
    const int lane = threadIdx.x & 31;
    uint32_t key[EPL];
    if (cached == nullptr) {
#pragma unroll
        for (int i = 0; i < EPL; ++i) key[i] = (i * 32 + lane < E) ? order_key(z[i]) : 0u;
        warp_topk_core<EPL>(key, k, out_id, out_w);
        return;
    }
    float zmax = -INFINITY, zmin = INFINITY;
#pragma unroll
    for (int i = 0; i < EPL; ++i)
        if (i * 32 + lane < E) { zmax = fmaxf(zmax, z[i]); zmin = fminf(zmin, z[i]); }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        zmax = fmaxf(zmax, __shfl_xor_sync(FULL, zmax, o));
        zmin = fminf(zmin, __shfl_xor_sync(FULL, zmin, o));
    }
    const float b = lambda * (zmax - zmin);
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
        const int e = i * 32 + lane;
        key[i] = e < E ? order_key(cached[e] ? z[i] + b : z[i]) : 0u;
    }
    float wb;
    warp_topk_core<EPL>(key, k, out_id, wb);
    // weights from the unbiased logits of the selection: lane j fetches z of its id from
    // the lane that holds it
    float zj = -INFINITY;
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
        const float v = __shfl_sync(FULL, z[i], out_id & 31);
        if (lane < k && (out_id >> 5) == i) zj = v;
    }
    float m = zj;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(FULL, m, o));
    const float ex = lane < k ? expf(zj - m) : 0.0f;
    out_w = ex / warp_sum(ex);
}

template <int EPL>
__device__ __forceinline__ void warp_route(const float* logits, int E, int k, const uint8_t* cached, float lambda,
                                           int& out_id, float& out_w) {
    const int lane = threadIdx.x & 31;
    float z[EPL];
#pragma unroll
    for (int i = 0; i < EPL; ++i) z[i] = (i * 32 + lane < E) ? __ldcg(logits + i * 32 + lane) : 0.0f;
    warp_route_z<EPL>(z, E, k, cached, lambda, out_id, out_w);
}

// warp_route with EPL chosen from E.
__device__ __forceinline__ void warp_route_any(const float* logits, int E, int k, const uint8_t* cached, float lambda,
                                               int& out_id, float& out_w) {
    if (E <= 256) warp_route<8>(logits, E, k, cached, lambda, out_id, out_w);
    else if (E <= 512) warp_route<16>(logits, E, k, cached, lambda, out_id, out_w);
    else warp_route<MAX_EXPERTS / 32>(logits, E, k, cached, lambda, out_id, out_w);
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
