// Router stage of redmoe_router, for any number of token rows:
//   router_logits_kernel  l[t, e] = x_t . Wr[e] (+ b[e])   (CUDA cores, rows streamed once
//                         per block of 4 tokens; the batched forward path computes the same
//                         logits with a tensor-core GEMM and its top-k in route.cu)
//   topk_kernel           per token (one warp): top-k of the logits with ties to the lower
//                         id, renormalised weights and the shared gate sigmoid(x . g).
// Router, top-k and shared gate belong to one stage of the layer ("Research notes,
// October 2026", section 1 "DwarfStar today": router, top-k and shared gate run in one
// kernel).
#include "common.cuh"
#include "gemv.cuh"
#include "internal.h"
#include "topk.cuh"

namespace redmoe {

namespace {

constexpr int RL_THREADS = 256;
constexpr int RL_WARPS = RL_THREADS / 32;
constexpr int RL_TOK = 4;  // tokens per block

template <int XT, int RT>
__global__ void __launch_bounds__(RL_THREADS) router_logits_kernel(const void* x, int T, int H, int E,
                                                                   const void* wr, const float* bias,
                                                                   float* logits) {
    extern __shared__ __align__(128) unsigned char smem[];
    uint4* xs = reinterpret_cast<uint4*>(smem);
    const int xstride = staged_bytes(H, RT, XT) / 16;
    const int t0 = blockIdx.y * RL_TOK;
    const int nt = min(RL_TOK, T - t0);
    for (int t = 0; t < RL_TOK; ++t) {
        if (t < nt) {
            stage_vec<RT, XT>(xs + t * xstride, static_cast<const char*>(x) + size_t(t0 + t) * H * vbytes(XT), H, false);
        } else {
            for (int i = threadIdx.x; i < xstride; i += blockDim.x) xs[t * xstride + i] = make_uint4(0u, 0u, 0u, 0u);
        }
    }
    __syncthreads();
    const int lane = threadIdx.x & 31;
    const int e = blockIdx.x * RL_WARPS + (threadIdx.x >> 5);
    if (e >= E) return;
    float2 acc[RL_TOK];
#pragma unroll
    for (int t = 0; t < RL_TOK; ++t) acc[t] = make_float2(0.f, 0.f);
    row_dots<RT, XT, RL_TOK>(static_cast<const char*>(wr) + size_t(e) * row_bytes(RT, H), nullptr, H / Wv<RT>::V, xs,
                             xstride, lane, acc);
    const float b = bias ? bias[e] : 0.0f;
#pragma unroll
    for (int t = 0; t < RL_TOK; ++t) {
        const float v = warp_sum(acc[t].x + acc[t].y);
        if (lane == 0 && t < nt) logits[size_t(t0 + t) * E + e] = v + b;
    }
}

template <int XT, int RT>
__global__ void __launch_bounds__(RL_THREADS) topk_kernel(const float* logits, int T, int E, int k, const void* x,
                                                          const void* g, int H, int32_t* ids, float* w,
                                                          float* sgate) {
    extern __shared__ __align__(16) uint32_t keys[];  // [RL_WARPS][E]
    const int lane = threadIdx.x & 31;
    const int t = blockIdx.x * RL_WARPS + (threadIdx.x >> 5);
    if (t >= T) return;
    warp_topk(logits + size_t(t) * E, E, k, keys + (threadIdx.x >> 5) * E, ids + size_t(t) * k, w + size_t(t) * k);
    float acc = 0.0f;
    if constexpr (XT == DT_BF16 && RT == DT_BF16) {
        // 16-byte loads, eight chunks of 8 elements per lane issued together (H % 8 == 0)
        const uint4* xr = reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(x) + size_t(t) * H);
        const uint4* gr = reinterpret_cast<const uint4*>(g);
        const int nc = H / 8;
        for (int c0 = 0; c0 < nc; c0 += 32 * 8) {
            uint4 xv[8], gv[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int c = c0 + 32 * i + lane;
                xv[i] = c < nc ? __ldg(xr + c) : make_uint4(0u, 0u, 0u, 0u);
                gv[i] = c < nc ? __ldg(gr + c) : make_uint4(0u, 0u, 0u, 0u);
            }
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const uint32_t xa[4] = {xv[i].x, xv[i].y, xv[i].z, xv[i].w};
                const uint32_t ga[4] = {gv[i].x, gv[i].y, gv[i].z, gv[i].w};
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    acc = fmaf(bf16f(uint16_t(xa[j] & 0xffffu)), bf16f(uint16_t(ga[j] & 0xffffu)), acc);
                    acc = fmaf(bf16f(uint16_t(xa[j] >> 16)), bf16f(uint16_t(ga[j] >> 16)), acc);
                }
            }
        }
    } else {
        for (int h = lane; h < H; h += 32) {
            float xv, gv;
            if constexpr (XT == DT_BF16) xv = bf16f(static_cast<const uint16_t*>(x)[size_t(t) * H + h]);
            else xv = static_cast<const float*>(x)[size_t(t) * H + h];
            if constexpr (RT == DT_BF16) gv = bf16f(static_cast<const uint16_t*>(g)[h]);
            else gv = static_cast<const float*>(g)[h];
            acc = fmaf(xv, gv, acc);
        }
    }
    acc = warp_sum(acc);
    if (lane == 0 && sgate) sgate[t] = 1.0f / (1.0f + expf(-acc));
}

template <int XT, int RT>
redmoe_status launch_router_dt(const redmoe_layer* L, const void* x, int T, float* logits, int32_t* ids,
                               float* w, float* sgate, cudaStream_t stream, int* launches) {
    const int H = L->hidden, E = L->n_experts;
    const int smem = RL_TOK * staged_bytes(H, RT, XT);
    auto kern = router_logits_kernel<XT, RT>;
    if (smem > 48 * 1024 &&
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
        return REDMOE_ERR_CUDA;
    dim3 grid((E + RL_WARPS - 1) / RL_WARPS, (T + RL_TOK - 1) / RL_TOK);
    kern<<<grid, RL_THREADS, smem, stream>>>(x, T, H, E, L->router_w, L->router_bias, logits);
    if (cudaGetLastError() != cudaSuccess) return REDMOE_ERR_CUDA;
    if (launches) *launches += 1;
    const int ksmem = RL_WARPS * E * 4;
    if (ksmem > 48 * 1024 &&
        cudaFuncSetAttribute(topk_kernel<XT, RT>, cudaFuncAttributeMaxDynamicSharedMemorySize, ksmem) != cudaSuccess)
        return REDMOE_ERR_CUDA;
    topk_kernel<XT, RT><<<(T + RL_WARPS - 1) / RL_WARPS, RL_THREADS, ksmem, stream>>>(
        logits, T, E, L->top_k, x, L->shared_gate_w, H, ids, w, sgate);
    if (cudaGetLastError() != cudaSuccess) return REDMOE_ERR_CUDA;
    if (launches) *launches += 1;
    return REDMOE_OK;
}

}  // namespace

redmoe_status launch_router(const redmoe_layer* L, const void* x, int T, float* logits, int32_t* ids, float* w,
                            float* sgate, cudaStream_t stream, int* launches) {
    if (L->x_dtype == DT_F32 && L->router_dtype == DT_F32)
        return launch_router_dt<DT_F32, DT_F32>(L, x, T, logits, ids, w, sgate, stream, launches);
    if (L->x_dtype == DT_BF16 && L->router_dtype == DT_BF16)
        return launch_router_dt<DT_BF16, DT_BF16>(L, x, T, logits, ids, w, sgate, stream, launches);
    return REDMOE_ERR_UNSUPPORTED;
}

}  // namespace redmoe
