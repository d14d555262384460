// Batched path (T > 4 token rows, bf16): the whole layer as four kernels on one stream.
//
//   1 router logits   tensor-core GEMM  x[T,H] . Wr[E,H]^T (+ b)      -> logits [T,E] fp32;
//                     its epilogue warps also zero out, which step 4 adds into
//   2 routing         one cooperative kernel (route.cu): top-k, renormalised weights,
//                     sigmoid(x . g); the stable counting sort of the
//                     T*k rows by expert (counts, offsets, perm) and the GEMM tile schedule;
//                     and xg, the x rows in grouped order (row offsets[e] + r of expert e is
//                     token perm[offsets[e] + r] / k). Loading these rows inside the GEMM
//                     with tile::gather4 TMA copies, or with cp.async from a producer warp,
//                     measured 1.6-2.7x slower on B200 than this copy plus tiled loads.
//   3 gate/up GEMM    per group: h = silu(xg . Wg^T) * (xg . Wu^T), bf16  -> h [T*k+T, I];
//                     the shared expert's group (h rows T*k .. T*k+T-1) reads x itself
//   4 down GEMM       per group: out[token] += weight * (h . Wd^T), fp32, added with
//                     bulk reductions of the copy engine
//
// The weighted combine of step 4 adds fp32 partial rows with atomic reductions: the summation
// order of the (k + 1) contributions to an output element varies from run to run, within
// the rounding of fp32 (the decode path, by contrast, is deterministic).
#include <cuda.h>

#include "common.cuh"
#include "internal.h"

#include "ggemm_params.h"

namespace redmoe {

bool make_tmap_bf16(CUtensorMap* m, const void* base, uint64_t rows, uint64_t K, uint32_t box_rows);
redmoe_status gemm_router(GemmParams& p, cudaStream_t s);
redmoe_status gemm_swiglu(GemmParams& p, cudaStream_t s);
redmoe_status gemm_scatter(GemmParams& p, cudaStream_t s);
redmoe_status launch_route(const redmoe_layer* L, const void* x, int T, const float* logits, int32_t* ids, float* w,
                           float* sgate, int32_t* counts, int32_t* offsets, int32_t* perm, int tile_m,
                           int32_t* tiles, void* xg, int32_t* bhist, Control* ctl, cudaStream_t stream,
                           int* launches, CacheBias cb);

BatchLayout batch_layout(int T, int E, int k, int H, int I) {
    BatchLayout b;
    size_t o = 256;
    const size_t rows = size_t(T) * k + T;
    b.logits = o; o = align256(o + 4ull * T * E);
    b.sgate = o; o = align256(o + 4ull * T);
    b.counts = o; o = align256(o + 4ull * E);
    b.offsets = o; o = align256(o + 4ull * (E + 1));
    b.perm = o; o = align256(o + 4ull * T * k);
    b.tiles = o; o = align256(o + 4ull * (E + 2));
    b.bhist = o; o = align256(o + 4ull * ROUTE_MAX_BLOCKS * E);
    b.xg = o; o = align256(o + 2ull * T * k * H);
    b.h = o; o = align256(o + 2ull * rows * I);
    b.total = o;
    return b;
}

bool batch_shape_ok(const redmoe_layer* L) {
    return L->x_dtype == DT_BF16 && L->router_dtype == DT_BF16 && L->expert_dtype == DT_BF16 &&
           L->inter == L->shared_inter && L->hidden % 256 == 0 && L->inter % 128 == 0;
}

redmoe_status launch_batched(const redmoe_layer* L, const void* x, int T, float* out, int32_t* ids, float* w,
                             void* ws, const redmoe_route_debug* dbg, cudaStream_t s, int* launches,
                             CacheBias cb) {
    const int H = L->hidden, E = L->n_experts, k = L->top_k, I = L->inter;
    const BatchLayout B = batch_layout(T, E, k, H, I);
    char* base = static_cast<char*>(ws);
    float* logits = reinterpret_cast<float*>(base + B.logits);
    float* sgate = reinterpret_cast<float*>(base + B.sgate);
    int32_t* counts = reinterpret_cast<int32_t*>(base + B.counts);
    int32_t* offsets = reinterpret_cast<int32_t*>(base + B.offsets);
    int32_t* perm = reinterpret_cast<int32_t*>(base + B.perm);
    int32_t* tiles = reinterpret_cast<int32_t*>(base + B.tiles);
    int32_t* bhist = reinterpret_cast<int32_t*>(base + B.bhist);
    Control* ctl = reinterpret_cast<Control*>(base);
    void* xg = base + B.xg;
    uint16_t* hbuf = reinterpret_cast<uint16_t*>(base + B.h);
    const uint64_t rows = uint64_t(T) * k + T;
    redmoe_status st;

    // 1 router logits
    GemmParams gr = {};
    if (!make_tmap_bf16(&gr.tmA, x, T, H, 128) || !make_tmap_bf16(&gr.tmB0, L->router_w, E, H, 64))
        return REDMOE_ERR_CUDA;
    gr.E = E; gr.T = T; gr.k = k; gr.N = E; gr.Nb = E; gr.n_tiles = (E + 63) / 64; gr.num_kb = H / 64;
    gr.out_f32 = logits; gr.bias = L->router_bias; gr.ctl = ctl;
    gr.zero_out = out; gr.zero_f4 = uint64_t(T) * H / 4;
    if ((st = gemm_router(gr, s)) != REDMOE_OK) return st;
    if (launches) *launches += 1;
    // 2 routing: top-k, weights, shared gate, zeroed out, grouping, tile schedule, gathered x
    if ((st = launch_route(L, x, T, logits, ids, w, sgate, counts, offsets, perm, 128, tiles, xg, bhist, ctl, s,
                           launches, cb)) != REDMOE_OK)
        return st;
    if (dbg) {
        if (cudaMemcpyAsync(dbg->counts, counts, 4ull * E, cudaMemcpyDeviceToDevice, s) != cudaSuccess ||
            cudaMemcpyAsync(dbg->offsets, offsets, 4ull * (E + 1), cudaMemcpyDeviceToDevice, s) != cudaSuccess ||
            cudaMemcpyAsync(dbg->perm, perm, 4ull * T * k, cudaMemcpyDeviceToDevice, s) != cudaSuccess)
            return REDMOE_ERR_CUDA;
    }
    // 3 gate/up + SwiGLU
    GemmParams g1 = {};
    if (!make_tmap_bf16(&g1.tmA, xg, uint64_t(T) * k, H, 128) || !make_tmap_bf16(&g1.tmA2, x, T, H, 128) ||
        !make_tmap_bf16(&g1.tmB0, L->w_gate, uint64_t(E) * I, H, 128) ||
        !make_tmap_bf16(&g1.tmB1, L->w_up, uint64_t(E) * I, H, 128) ||
        !make_tmap_bf16(&g1.tmS0, L->sh_gate, I, H, 128) || !make_tmap_bf16(&g1.tmS1, L->sh_up, I, H, 128))
        return REDMOE_ERR_CUDA;
    g1.E = E; g1.T = T; g1.k = k; g1.N = I; g1.Nb = I; g1.n_tiles = I / 128; g1.num_kb = H / 64;
    g1.offsets = offsets; g1.tiles = tiles; g1.out_bf16 = hbuf; g1.ctl = ctl;
    if ((st = gemm_swiglu(g1, s)) != REDMOE_OK) return st;
    if (launches) *launches += 1;
    // 4 down + weighted scatter-add into out
    GemmParams g2 = {};
    if (!make_tmap_bf16(&g2.tmA, hbuf, rows, I, 128) ||
        !make_tmap_bf16(&g2.tmB0, L->w_down, uint64_t(E) * H, I, 256) ||
        !make_tmap_bf16(&g2.tmS0, L->sh_down, H, I, 256))
        return REDMOE_ERR_CUDA;
    g2.E = E; g2.T = T; g2.k = k; g2.N = H; g2.Nb = H; g2.n_tiles = H / 256; g2.num_kb = I / 64;
    g2.offsets = offsets; g2.tiles = tiles; g2.out_f32 = out; g2.perm = perm; g2.topk_w = w; g2.sgate = sgate;
    g2.ctl = ctl;
    if ((st = gemm_scatter(g2, s)) != REDMOE_OK) return st;
    if (launches) *launches += 1;
    return REDMOE_OK;
}

}  // namespace redmoe
