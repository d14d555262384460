// Token->expert grouping for batched execution: histogram, exclusive prefix sum and a
// stable permutation, bit-exact and independent of thread timing.
//
// The pages batch prompt tokens in 2048-token chunks ("DwarfStar Red Lite" guide, "Chat
// defaults"; batched prefill was a later step after token-by-token ingestion, "Red Lite
// dev18", "Scope boundary") and group the multiplications per expert ("Research notes,
// October 2026", section 6: ds4 "regroups the multiplications to saturate the GPU"). They
// give no algorithm; this kernel is a stable counting sort of the T*k (token, slot) rows
// by expert id:
//
//   counts[e]  = number of rows routed to e
//   offsets    = exclusive prefix sum of counts (E + 1 entries)
//   perm[offsets[e] + r] = t*k + j, for the r-th row (t, j) routed to e, in increasing t
//
// One block: its 32 warps each own a contiguous slice of the rows. Per-warp histograms
// (shared-memory atomics: counts do not depend on the order of the additions) are
// prefix-summed over the warps for each expert, so that warp w's rows for expert e start
// after those of warps 0..w-1; a warp then walks its slice in order, 32 rows at a time,
// ranking rows of equal expert inside the batch by lane (match_any + popc). Every row's
// position is fixed by (expert, warp, batch, lane): the result is deterministic.
//
// With `tile_m > 0` the kernel also writes the tile schedule of the grouped GEMM: groups
// 0..E-1 are the experts and group E is the shared expert, which takes every token in
// order; tiles[g] = prefix sum over groups of ceil(rows_g / tile_m) (E + 2 entries).
#include "common.cuh"
#include "internal.h"

namespace redmoe {

namespace {

constexpr int RB_THREADS = 1024;
constexpr int RB_WARPS = RB_THREADS / 32;
constexpr int RB_BATCH = 8;  // batches of 32 ids loaded together per warp

// Exclusive scan of v over the block (1024 threads); returns the block total in *total.
__device__ int block_exclusive_scan(int v, int* warp_sums, int* total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int inc = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int n = __shfl_up_sync(FULL, inc, o);
        if (lane >= o) inc += n;
    }
    if (lane == 31) warp_sums[warp] = inc;
    __syncthreads();
    if (warp == 0) {
        int s = warp_sums[lane];
        int si = s;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int n = __shfl_up_sync(FULL, si, o);
            if (lane >= o) si += n;
        }
        warp_sums[lane] = si - s;
        if (lane == 31) *total = si;
    }
    __syncthreads();
    const int r = warp_sums[warp] + inc - v;
    __syncthreads();
    return r;
}

__global__ void __launch_bounds__(RB_THREADS) route_build_kernel(const int32_t* ids, int n, int k, int E, int T,
                                                                 int32_t* counts, int32_t* offsets, int32_t* perm,
                                                                 int tile_m, int32_t* tiles) {
    extern __shared__ __align__(16) int sm[];
    int* hist = sm;                           // [RB_WARPS][E]
    int* offs = hist + RB_WARPS * E;          // [E + 1]
    int* wsum = offs + E + 1;                 // [32]
    int* tot = wsum + 32;                     // [2]
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int lo = int((long long)n * warp / RB_WARPS);
    const int hi = int((long long)n * (warp + 1) / RB_WARPS);

    for (int i = threadIdx.x; i < RB_WARPS * E; i += RB_THREADS) hist[i] = 0;
    __syncthreads();
    // ids are read RB_BATCH batches of 32 at a time: independent loads issued together
    for (int base = lo; base < hi; base += 32 * RB_BATCH) {
        int ev[RB_BATCH];
#pragma unroll
        for (int b = 0; b < RB_BATCH; ++b) {
            const int i = base + 32 * b + lane;
            ev[b] = i < hi ? __ldg(ids + i) : -1;
        }
#pragma unroll
        for (int b = 0; b < RB_BATCH; ++b)
            if (ev[b] >= 0 && ev[b] < E) atomicAdd(&hist[warp * E + ev[b]], 1);
    }
    __syncthreads();
    // per expert: exclusive prefix over warps, total count
    for (int e = threadIdx.x; e < E; e += RB_THREADS) {
        int run = 0;
        for (int w = 0; w < RB_WARPS; ++w) {
            const int c = hist[w * E + e];
            hist[w * E + e] = run;
            run += c;
        }
        offs[e] = run;
        counts[e] = run;
    }
    __syncthreads();
    // exclusive prefix over experts (E <= 1024: one expert per thread)
    const int cnt = (threadIdx.x < E) ? offs[threadIdx.x] : 0;
    const int ex = block_exclusive_scan(cnt, wsum, tot);
    if (threadIdx.x < E) offs[threadIdx.x] = ex;
    if (threadIdx.x == 0) offs[E] = *tot;
    __syncthreads();
    for (int e = threadIdx.x; e <= E; e += RB_THREADS) offsets[e] = offs[e];
    if (tile_m > 0) {
        // tiles per group (experts, then the shared expert with T rows), exclusive prefix
        const int ntile = (threadIdx.x < E) ? (cnt + tile_m - 1) / tile_m : 0;
        const int tex = block_exclusive_scan(ntile, wsum, tot);
        if (threadIdx.x < E) tiles[threadIdx.x] = tex;
        if (threadIdx.x == 0) {
            tiles[E] = *tot;
            tiles[E + 1] = *tot + (T + tile_m - 1) / tile_m;
        }
    }
    // stable placement
    const unsigned lt = (1u << lane) - 1u;
    for (int base0 = lo; base0 < hi; base0 += 32 * RB_BATCH) {
        int ev[RB_BATCH];
#pragma unroll
        for (int b = 0; b < RB_BATCH; ++b) {
            const int i = base0 + 32 * b + lane;
            ev[b] = i < hi ? __ldg(ids + i) : -1;
        }
#pragma unroll
        for (int b = 0; b < RB_BATCH; ++b) {
            const int i = base0 + 32 * b + lane;
            int e = ev[b];
            const bool ok = i < hi && e >= 0 && e < E;
            if (!ok) e = -1;
            const unsigned peers = __match_any_sync(FULL, e);
            const int rank = __popc(peers & lt);
            if (ok) perm[offs[e] + hist[warp * E + e] + rank] = i;
            __syncwarp();
            if (ok && lane == 31 - __clz(peers)) hist[warp * E + e] += __popc(peers);
            __syncwarp();
        }
    }
    (void)k;
}

}  // namespace

int route_build_smem_bytes(int E) { return 4 * (RB_WARPS * E + E + 1 + 32 + 2); }

redmoe_status launch_route_build(const int32_t* ids, int T, int k, int E, int32_t* counts, int32_t* offsets,
                                 int32_t* perm, int tile_m, int32_t* tiles, cudaStream_t stream, int* launches) {
    const int smem = route_build_smem_bytes(E);
    if (smem > 48 * 1024 &&
        cudaFuncSetAttribute(route_build_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
        return REDMOE_ERR_CUDA;
    route_build_kernel<<<1, RB_THREADS, smem, stream>>>(ids, T * k, k, E, T, counts, offsets, perm, tile_m, tiles);
    if (cudaGetLastError() != cudaSuccess) return REDMOE_ERR_CUDA;
    if (launches) *launches += 1;
    return REDMOE_OK;
}

}  // namespace redmoe
