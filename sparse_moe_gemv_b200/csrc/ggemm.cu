// Grouped GEMM on the 5th-generation tensor cores (tcgen05, TMEM accumulators, TMA),
// for the batched (prefill) path: the router logits, the experts' gate/up projection with
// a fused SwiGLU epilogue, and the down projection with a fused weighted scatter-add.
//
// One persistent kernel per GEMM, one CTA per SM, warp-specialised:
//   warp 0     one lane issues the TMA tile loads (A rows and B weight rows, 64-wide K
//              slabs, 128-byte swizzled) into a ring of shared-memory stages;
//   warp 1     allocates TMEM; one lane issues tcgen05.mma (M = 128, N = BN, K = 16 per
//              instruction) into one of two TMEM accumulators and commits completion to
//              mbarriers (stage free, accumulator full);
//   warps 2-5  the epilogue: each reads its 32 TMEM lanes (= 32 rows of the tile), applies
//              the mode's epilogue and frees the accumulator, overlapping the next tile's
//              MMAs.
// Work items are (group, n-tile, m-tile) with the m-tiles of one (group, n-tile) adjacent,
// so concurrently running CTAs read the same weight tile and HBM sends it once (L2).
//
// Groups: the experts (rows of expert e: offsets[e] .. offsets[e+1] of the grouped row
// space) and, last, the shared expert with every token (the extra expert slot of the
// DwarfStar MoE kernel, "Research notes, October 2026", section 1). Batching prompt
// tokens in 2048-token chunks follows the guide "DwarfStar Red Lite", "Chat defaults".
//
// Every wait is bounded: after the timeout the thread records ERRBIT_TIMEOUT and stops
// waiting, so a fault can never hang the GPU; the host reads the error word.
#include <cuda.h>
#include <cuda_bf16.h>

#include <mutex>
#include <vector>

#include "common.cuh"
#include "internal.h"
#include "tc.cuh"
#include "ggemm_params.h"

namespace redmoe {

namespace {

constexpr int BM = 128;
constexpr int BK = 64;
constexpr int GEMM_THREADS = 192;

constexpr int RED_COLS = 64;                    // scatter epilogue: columns per bulk reduction
constexpr int RED_STRIDE = RED_COLS * 4 + 16;   // padded staging row (bytes): 4-way bank conflicts at most
constexpr int RED_WARP = 2 * 32 * RED_STRIDE;   // two staging buffers of 32 rows per epilogue warp

template <int MODE, int BN>
struct Cfg {
    static constexpr int A_BYTES = BM * BK * 2;
    static constexpr int B_BYTES = BN * BK * 2;
    static constexpr int STAGE = A_BYTES + B_BYTES;
    static constexpr int NS = (STAGE <= 24 * 1024) ? 8 : (MODE == GM_SCATTER ? 3 : 4);
    static constexpr int TMEM_COLS = (2 * BN <= 32) ? 32 : (2 * BN <= 64 ? 64 : (2 * BN <= 128 ? 128 : (2 * BN <= 256 ? 256 : 512)));
    // scatter: weighted rows for the bulk reductions; router: a 32 x 33 fp32 transpose
    // buffer per epilogue warp
    static constexpr int STAGING = (MODE == GM_SCATTER) ? 4 * RED_WARP : (MODE == GM_ROUTER ? 4 * 32 * 33 * 4 : 0);
    static constexpr int SMEM = 1024 + NS * STAGE + STAGING + 256;  // alignment slack + stages + staging + barriers
};

struct Tile {
    int g, m, n, S, C;  // group, m-tile, n-tile, group's first row, group's row count
};

template <int MODE>
__device__ __forceinline__ int total_tiles(const GemmParams& p) {
    if (MODE == GM_ROUTER) return ((p.T + BM - 1) / BM) * p.n_tiles;
    return __ldg(p.tiles + p.E + 1) * p.n_tiles;
}

template <int MODE>
__device__ __forceinline__ Tile tile_of(const GemmParams& p, int w) {
    Tile t;
    if (MODE == GM_ROUTER) {
        const int mt = (p.T + BM - 1) / BM;
        t.g = 0;
        t.n = w / mt;
        t.m = w - t.n * mt;
        t.S = 0;
        t.C = p.T;
        return t;
    }
    const int q = w / p.n_tiles;  // tiles[g] <= q < tiles[g+1]
    int lo = 0, hi = p.E + 1;     // search g in [0, E]
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (__ldg(p.tiles + mid) <= q) lo = mid; else hi = mid;
    }
    const int g = lo;
    const int t0 = __ldg(p.tiles + g);
    const int mt = __ldg(p.tiles + g + 1) - t0;
    const int local = w - t0 * p.n_tiles;
    t.g = g;
    t.n = local / mt;
    t.m = local - t.n * mt;
    if (g < p.E) {
        t.S = __ldg(p.offsets + g);
        t.C = __ldg(p.offsets + g + 1) - t.S;
    } else {
        t.S = __ldg(p.offsets + p.E);
        t.C = p.T;
    }
    return t;
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" :: "r"(smem_u32(bar)) : "memory");
}

template <int MODE, int BN>
__global__ void __launch_bounds__(GEMM_THREADS, 1) ggemm_kernel(const __grid_constant__ GemmParams p) {
    using C = Cfg<MODE, BN>;
    constexpr int NS = C::NS;
    extern __shared__ unsigned char smem_raw[];
    unsigned char* smem = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    unsigned char* staging = smem + NS * C::STAGE;
    uint64_t* full = reinterpret_cast<uint64_t*>(staging + C::STAGING);
    uint64_t* empty = full + NS;
    uint64_t* tfull = empty + NS;
    uint64_t* tempty = tfull + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tempty + 2);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    int* err = &p.ctl->err;
    const uint64_t to = p.timeout_ns;

    if (threadIdx.x == 0) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(full + s, 1);
            mbar_init(empty + s, 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(tfull + a, 1);
            mbar_init(tempty + a, 4);
        }
        fence_mbar_init();
    }
    if (warp == 1) tmem_alloc(tmem_slot, C::TMEM_COLS);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    const int total = total_tiles<MODE>(p);

    if (warp == 0) {
        // ------------------------------------------------------------ producer (lane 0)
        uint32_t it = 0;
        for (int w = blockIdx.x; w < total; w += gridDim.x) {
            const Tile t = tile_of<MODE>(p, w);
            const int rowA = t.S + t.m * BM;
            const bool shared = (MODE != GM_ROUTER) && t.g == p.E;
            for (int kb = 0; kb < p.num_kb; ++kb, ++it) {
                const int s = int(it % NS);
                unsigned char* st = smem + s * C::STAGE;
                if (lane != 0) continue;
                mbar_wait(empty + s, ((it / NS) & 1u) ^ 1u, err, to);
                mbar_arrive_expect_tx(full + s, C::STAGE);
                if (MODE == GM_SWIGLU && shared) tma_load_2d(st, &p.tmA2, kb * BK, t.m * BM, full + s);
                else tma_load_2d(st, &p.tmA, kb * BK, rowA, full + s);
                unsigned char* sb = st + C::A_BYTES;
                if (MODE == GM_SWIGLU) {
                    const int nh = t.n * (BN / 2);
                    const int rb = shared ? nh : t.g * p.Nb + nh;
                    tma_load_2d(sb, shared ? &p.tmS0 : &p.tmB0, kb * BK, rb, full + s);
                    tma_load_2d(sb + (BN / 2) * 128, shared ? &p.tmS1 : &p.tmB1, kb * BK, rb, full + s);
                } else if (MODE == GM_SCATTER) {
                    const int n0 = t.n * BN;
                    tma_load_2d(sb, shared ? &p.tmS0 : &p.tmB0, kb * BK, shared ? n0 : t.g * p.Nb + n0, full + s);
                } else {
                    tma_load_2d(sb, &p.tmB0, kb * BK, t.n * BN, full + s);
                }
            }
        }
        // drain: wait until every stage issued here has landed (consumed or not)
        const uint32_t n_issued = it;
        if (lane == 0)
            for (uint32_t j = (n_issued > uint32_t(NS) ? n_issued - NS : 0u); j < n_issued; ++j)
                mbar_wait(full + (j % NS), (j / NS) & 1u, err, to);
    } else if (warp == 1 && lane == 0) {
        // ------------------------------------------------------------ MMA issuer
        constexpr uint32_t idesc = idesc_bf16_f32(BM, BN);
        uint32_t it = 0, tc = 0;
        for (int w = blockIdx.x; w < total; w += gridDim.x, ++tc) {
            const uint32_t acc = tc & 1u;
            mbar_wait(tempty + acc, ((tc >> 1) & 1u) ^ 1u, err, to);
            tc_fence_after();
            const uint32_t d_tmem = tmem_base + acc * BN;
            for (int kb = 0; kb < p.num_kb; ++kb, ++it) {
                const int s = int(it % NS);
                mbar_wait(full + s, (it / NS) & 1u, err, to);
                tc_fence_after();
                const uint32_t a_addr = smem_u32(smem + s * C::STAGE);
                const uint32_t b_addr = a_addr + C::A_BYTES;
                const uint64_t ad = sw128_kmajor_desc(a_addr), bd = sw128_kmajor_desc(b_addr);
#pragma unroll
                for (int kk = 0; kk < BK / 16; ++kk)
                    tc_mma_bf16(d_tmem, ad + uint64_t(2 * kk), bd + uint64_t(2 * kk), idesc, (kb | kk) != 0);
                tc_commit(empty + s);
            }
            tc_commit(tfull + acc);
        }
    } else if (warp >= 2) {
        // ------------------------------------------------------------ epilogue
        const int q = warp & 3;              // TMEM lane quadrant of this warp
        const int r = q * 32 + lane;         // row within the tile
        if (MODE == GM_ROUTER && p.zero_out) {
            // the output of the down GEMM, zeroed while the first tiles load
            float4* z = reinterpret_cast<float4*>(p.zero_out);
            const uint64_t nth = uint64_t(gridDim.x) * 128;
            for (uint64_t i = uint64_t(blockIdx.x) * 128 + (threadIdx.x - 64); i < p.zero_f4; i += nth)
                z[i] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
        uint32_t tc = 0;
        uint32_t red_chunk = 0;              // scatter: staging buffer sequence
        for (int w = blockIdx.x; w < total; w += gridDim.x, ++tc) {
            const Tile t = tile_of<MODE>(p, w);
            const uint32_t acc = tc & 1u;
            mbar_wait(tfull + acc, (tc >> 1) & 1u, err, to);
            tc_fence_after();
            const uint32_t taddr = tmem_base + (uint32_t(q * 32) << 16) + acc * BN;
            const int lr = t.m * BM + r;     // row within the group
            const bool valid = lr < t.C;
            const int grow = t.S + lr;       // row in the grouped row space
            if (MODE == GM_ROUTER) {
                // this warp's 32 rows x 32 columns go through a padded shared buffer, so
                // that each store instruction writes one row's 128 contiguous bytes
                float* tb = reinterpret_cast<float*>(staging) + (warp - 2) * (32 * 33);
                const int row0 = t.m * BM + q * 32;
#pragma unroll 1
                for (int c = 0; c < BN / 32; ++c) {
                    float v[32];
                    tmem_ld32(taddr + c * 32, v);
                    const int n0 = t.n * BN + c * 32;
#pragma unroll
                    for (int j = 0; j < 32; ++j) tb[lane * 33 + j] = v[j];
                    __syncwarp();
                    const int n = n0 + lane;
                    const float b = (p.bias && n < p.N) ? __ldg(p.bias + n) : 0.0f;
#pragma unroll 4
                    for (int i = 0; i < 32; ++i) {
                        const int row = row0 + i;
                        if (row < t.C && n < p.N) p.out_f32[size_t(row) * p.N + n] = tb[i * 33 + lane] + b;
                    }
                    __syncwarp();
                }
            } else if (MODE == GM_SWIGLU) {
#pragma unroll 1
                for (int c = 0; c < BN / 64; ++c) {
                    float g[32], u[32];
                    tmem_ld32(taddr + c * 32, g);
                    tmem_ld32(taddr + BN / 2 + c * 32, u);
                    if (valid) {
                        uint32_t pk[16];
#pragma unroll
                        for (int j = 0; j < 16; ++j) {
                            const float h0 = g[2 * j] / (1.0f + expf(-g[2 * j])) * u[2 * j];
                            const float h1 = g[2 * j + 1] / (1.0f + expf(-g[2 * j + 1])) * u[2 * j + 1];
                            pk[j] = uint32_t(f2bf(h0)) | (uint32_t(f2bf(h1)) << 16);
                        }
                        uint4* dst = reinterpret_cast<uint4*>(p.out_bf16 + size_t(grow) * p.N + t.n * (BN / 2) + c * 32);
#pragma unroll
                        for (int j = 0; j < 4; ++j) dst[j] = make_uint4(pk[4 * j], pk[4 * j + 1], pk[4 * j + 2], pk[4 * j + 3]);
                    }
                }
            } else {
                // weight * y for this row, staged in shared memory (a padded row per thread,
                // two buffers per warp) and added into out[token] by 256-byte bulk reductions
                int tok = 0;
                float wgt = 0.0f;
                if (valid) {
                    if (t.g < p.E) {
                        const int e = __ldg(p.perm + grow);
                        tok = e / p.k;
                        wgt = __ldg(p.topk_w + e);
                    } else {
                        tok = lr;
                        wgt = __ldg(p.sgate + lr);
                    }
                }
                unsigned char* wbuf = staging + (warp - 2) * RED_WARP;
#pragma unroll 1
                for (int c = 0; c < BN / RED_COLS; ++c, ++red_chunk) {
                    float v[32], u[32];
                    tmem_ld32(taddr + c * RED_COLS, v);
                    tmem_ld32(taddr + c * RED_COLS + 32, u);
                    unsigned char* row = wbuf + (red_chunk & 1u) * (32 * RED_STRIDE) + lane * RED_STRIDE;
                    bulk_wait_read<1>();  // the buffer used two chunks ago has been read
                    float4* r4 = reinterpret_cast<float4*>(row);
#pragma unroll
                    for (int j = 0; j < 8; ++j) r4[j] = make_float4(wgt * v[4 * j], wgt * v[4 * j + 1], wgt * v[4 * j + 2], wgt * v[4 * j + 3]);
#pragma unroll
                    for (int j = 0; j < 8; ++j) r4[8 + j] = make_float4(wgt * u[4 * j], wgt * u[4 * j + 1], wgt * u[4 * j + 2], wgt * u[4 * j + 3]);
                    fence_proxy_async_smem();
                    if (valid) bulk_reduce_add_f32(p.out_f32 + size_t(tok) * p.N + t.n * BN + c * RED_COLS, row, RED_COLS * 4);
                    bulk_commit();
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(tempty + acc);
        }
        if (MODE == GM_SCATTER) bulk_wait<0>();  // every bulk reduction of this thread has completed
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem_base, C::TMEM_COLS);
}

// ------------------------------------------------------------------- host
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static std::mutex mu;
    static EncodeTiledFn fn = nullptr;
    std::lock_guard<std::mutex> lock(mu);
    if (!fn) {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(f);
    }
    return fn;
}

template <int MODE, int BN>
int blocks_for(const void* kern, int smem) {
    static std::mutex mu;
    static std::vector<int> done;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return -1;
    std::lock_guard<std::mutex> lock(mu);
    if (dev >= int(done.size())) done.resize(dev + 1, 0);
    if (!done[dev]) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess) return -1;
        done[dev] = 1;
    }
    return 1;
}

template <int MODE, int BN>
redmoe_status launch_gemm(GemmParams& p, cudaStream_t stream) {
    using C = Cfg<MODE, BN>;
    DevInfo di;
    if (!get_dev_info(&di)) return REDMOE_ERR_CUDA;
    if (C::SMEM > di.max_smem_optin) return REDMOE_ERR_UNSUPPORTED;
    auto kern = ggemm_kernel<MODE, BN>;
    if (blocks_for<MODE, BN>(reinterpret_cast<const void*>(kern), C::SMEM) < 0) return REDMOE_ERR_CUDA;
    p.timeout_ns = BARRIER_TIMEOUT_NS;
    kern<<<di.sm_count, GEMM_THREADS, C::SMEM, stream>>>(p);
    return cudaGetLastError() == cudaSuccess ? REDMOE_OK : REDMOE_ERR_CUDA;
}

}  // namespace

// 2-D bf16 tensor map over a row-major [rows, K] matrix, box of 64 columns x box_rows rows,
// 128-byte swizzle (the layout the MMA descriptors above describe).
bool make_tmap_bf16(CUtensorMap* m, const void* base, uint64_t rows, uint64_t K, uint32_t box_rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[2] = {K, rows};
    const cuuint64_t strides[1] = {K * 2};
    const cuuint32_t box[2] = {uint32_t(BK), box_rows};
    const cuuint32_t estr[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

redmoe_status gemm_router(GemmParams& p, cudaStream_t s) { return launch_gemm<GM_ROUTER, 64>(p, s); }
redmoe_status gemm_swiglu(GemmParams& p, cudaStream_t s) { return launch_gemm<GM_SWIGLU, 256>(p, s); }
redmoe_status gemm_scatter(GemmParams& p, cudaStream_t s) { return launch_gemm<GM_SCATTER, 256>(p, s); }

}  // namespace redmoe
