// Routing of a batch of tokens (the batched path) in one cooperative launch, one block
// per SM, each block owning a contiguous range of tokens:
//
//   phase 1  one warp per token: top-k of the logits (ties to the lower id) with the
//            renormalised weights and the shared gate sigmoid(x . g); the block's
//            histogram of expert ids goes to bhist[block][e]
//   phase 2  per expert e: exclusive prefix of bhist[.][e] over the blocks, and counts[e]
//   phase 3  per block: the exclusive prefix of the counts (offsets, and block 0 writes
//            offsets and the GEMM tile schedule), then the block's rows in (t, j) order:
//            row (t, j) routed to e lands at offsets[e] + (rows of e in earlier blocks)
//            + (rows of e before it in this block) -> perm; and x[t] is copied to that
//            row of xg, the gate/up GEMM's gathered input
//
// The phases are separated by bounded grid barriers. The grouping is the stable counting
// sort that route_build.cu computes, bit for bit: a row's position depends only on
// (expert, t, j), never on timing. The pages batch prompt tokens in 2048-token chunks and
// regroup the multiplications per expert ("DwarfStar Red Lite" guide, "Chat defaults";
// "Research notes, October 2026", section 6); router, top-k and shared gate belong to one
// stage (section 1, "DwarfStar today").
#include "common.cuh"
#include "internal.h"
#include "topk.cuh"

namespace redmoe {

namespace {

constexpr int RT_THREADS = 512;
constexpr int RT_WARPS = RT_THREADS / 32;

struct RouteParams {
    const float* logits;  // [T, E] fp32 (bias included)
    const uint16_t* x;    // [T, H] bf16
    const uint16_t* g;    // [H] bf16 shared-gate row
    int T, E, k, H;
    int tpb;              // tokens per block (ceil(T / grid))
    int32_t* ids;         // [T, k]
    float* w;             // [T, k]
    float* sgate;         // [T]
    int32_t* counts;      // [E]
    int32_t* offsets;     // [E + 1]
    int32_t* perm;        // [T * k]
    int tile_m;
    int32_t* tiles;       // [E + 2]
    uint16_t* xg;         // [T * k, H] bf16 gathered rows
    int32_t* bhist;       // [grid, E]
    Control* ctl;
    uint64_t timeout_ns;
    CacheBias cb;
};

// Exclusive prefix over v[0..n) (n <= 2 * RT_THREADS) into out[0..n); returns the total.
// Thread i handles entries 2i and 2i + 1. Must be reached by the whole block.
__device__ int block_scan2(const int* v, int* out, int n, int* wsum) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int i0 = 2 * threadIdx.x, i1 = i0 + 1;
    const int a = i0 < n ? v[i0] : 0, b = i1 < n ? v[i1] : 0;
    const int s = a + b;
    int inc = s;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(FULL, inc, o);
        if (lane >= o) inc += y;
    }
    __syncthreads();  // v may alias out; wsum may be in use by a previous call
    if (lane == 31) wsum[warp] = inc;
    __syncthreads();
    if (warp == 0) {
        const int ws = lane < RT_WARPS ? wsum[lane] : 0;
        int wi = ws;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(FULL, wi, o);
            if (lane >= o) wi += y;
        }
        if (lane < RT_WARPS) wsum[lane] = wi - ws;
        if (lane == RT_WARPS - 1) wsum[RT_WARPS] = wi;
    }
    __syncthreads();
    const int ex = wsum[warp] + inc - s;
    if (i0 < n) out[i0] = ex;
    if (i1 < n) out[i1] = ex + a;
    const int total = wsum[RT_WARPS];
    __syncthreads();
    return total;
}

template <int EPL>
__global__ void __launch_bounds__(RT_THREADS, 1) route_kernel(const __grid_constant__ RouteParams p) {
    extern __shared__ __align__(16) int sm[];
    const int E = p.E, k = p.k, T = p.T;
    int* hist = sm;                  // [E] histogram; later the next free position per expert
    int* offs = hist + E;            // [E + 1]
    int* tmp = offs + E + 1;         // [E]
    int* wsum = tmp + E;             // [RT_WARPS + 1]
    int* s_ids = wsum + 32;          // [tpb * k] this block's expert ids
    int* s_pos = s_ids + p.tpb * k;  // [tpb * k] positions of this block's rows
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const unsigned nb = gridDim.x;
    const int t0 = min(T, int(blockIdx.x) * p.tpb), t1 = min(T, t0 + p.tpb);

    for (int e = threadIdx.x; e < E; e += RT_THREADS) hist[e] = 0;
    __syncthreads();
    // ------------------------------------------------------------------ phase 1
    for (int t = t0 + warp; t < t1; t += RT_WARPS) {
        // the shared gate's first 2048 elements (16-byte loads, eight per lane) and the
        // logits are loaded together, so the top-k and the dot share one memory latency
        const uint4* xr = reinterpret_cast<const uint4*>(p.x + size_t(t) * p.H);
        const uint4* gr = reinterpret_cast<const uint4*>(p.g);
        const int nc = p.H / 8;
        uint4 xv[8], gv[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int c = 32 * i + lane;
            xv[i] = c < nc ? __ldg(xr + c) : make_uint4(0u, 0u, 0u, 0u);
            gv[i] = c < nc ? __ldg(gr + c) : make_uint4(0u, 0u, 0u, 0u);
        }
        int id;
        float wv;
        warp_route<EPL>(p.logits + size_t(t) * E, E, k, p.cb.cached, p.cb.lambda, id, wv);
        if (lane < k) {
            p.ids[size_t(t) * k + lane] = id;
            p.w[size_t(t) * k + lane] = wv;
            s_ids[(t - t0) * k + lane] = id;
            atomicAdd(&hist[id], 1);
        }
        float acc = 0.0f;
        for (int c0 = 0; c0 < nc; c0 += 32 * 8) {
            if (c0 > 0) {
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const int c = c0 + 32 * i + lane;
                    xv[i] = c < nc ? __ldg(xr + c) : make_uint4(0u, 0u, 0u, 0u);
                    gv[i] = c < nc ? __ldg(gr + c) : make_uint4(0u, 0u, 0u, 0u);
                }
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
        acc = warp_sum(acc);
        if (lane == 0) p.sgate[t] = 1.0f / (1.0f + expf(-acc));
    }
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += RT_THREADS) p.bhist[size_t(blockIdx.x) * E + e] = hist[e];
    grid_barrier(p.ctl, nb, 0, p.timeout_ns);

    // ------------------------------------------------------------------ phase 2
    for (int e = int(blockIdx.x) * RT_WARPS + warp; e < E; e += int(nb) * RT_WARPS) {
        int vb[ROUTE_MAX_BLOCKS / 32];  // this expert's count in block 32 c + lane, loaded together
#pragma unroll
        for (int c = 0; c < ROUTE_MAX_BLOCKS / 32; ++c) {
            const int b = 32 * c + lane;
            vb[c] = b < int(nb) ? __ldcg(p.bhist + size_t(b) * E + e) : 0;
        }
        int carry = 0;
#pragma unroll
        for (int c = 0; c < ROUTE_MAX_BLOCKS / 32; ++c) {
            const int b = 32 * c + lane;
            const int v = vb[c];
            int inc = v;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(FULL, inc, o);
                if (lane >= o) inc += y;
            }
            if (b < int(nb)) p.bhist[size_t(b) * E + e] = carry + inc - v;
            carry += __shfl_sync(FULL, inc, 31);
        }
        if (lane == 0) p.counts[e] = carry;
    }
    grid_barrier(p.ctl, nb, 1, p.timeout_ns);
    grid_release(p.ctl, nb);  // the launch's last barrier

    // ------------------------------------------------------------------ phase 3
    for (int e = threadIdx.x; e < E; e += RT_THREADS) tmp[e] = __ldcg(p.counts + e);
    __syncthreads();
    const int total = block_scan2(tmp, offs, E, wsum);
    if (threadIdx.x == 0) offs[E] = total;
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += RT_THREADS) hist[e] = offs[e] + __ldcg(p.bhist + size_t(blockIdx.x) * E + e);
    if (blockIdx.x == 0) {
        for (int e = threadIdx.x; e <= E; e += RT_THREADS) p.offsets[e] = offs[e];
        if (p.tile_m > 0) {
            for (int e = threadIdx.x; e < E; e += RT_THREADS) tmp[e] = (__ldcg(p.counts + e) + p.tile_m - 1) / p.tile_m;
            __syncthreads();
            int* tl = tmp;  // scanned in place
            const int nt = block_scan2(tmp, tl, E, wsum);
            for (int e = threadIdx.x; e < E; e += RT_THREADS) p.tiles[e] = tl[e];
            if (threadIdx.x == 0) {
                p.tiles[E] = nt;
                p.tiles[E + 1] = nt + (T + p.tile_m - 1) / p.tile_m;
            }
        }
    }
    __syncthreads();
    if (warp == 0) {
        const unsigned lt = (1u << lane) - 1u;
        for (int base = t0 * k; base < t1 * k; base += 32) {
            const int i = base + lane;
            const bool ok = i < t1 * k;
            const int e = ok ? s_ids[i - t0 * k] : -1;
            const unsigned peers = __match_any_sync(FULL, e);
            if (ok) {
                const int pos = hist[e] + __popc(peers & lt);
                p.perm[pos] = i;
                s_pos[i - t0 * k] = pos;
            }
            __syncwarp();
            if (ok && lane == 31 - __clz(peers)) hist[e] += __popc(peers);
            __syncwarp();
        }
    }
    __syncthreads();
    // gather: x[t] -> xg[position of (t, j)]; each warp copies two rows at a time in 16-byte
    // chunks, every load of both rows issued before their stores
    const int nent = (t1 - t0) * k;
    const int row16 = p.H / 8;
    const uint4* xs = reinterpret_cast<const uint4*>(p.x);
    uint4* xd = reinterpret_cast<uint4*>(p.xg);
    const uint4 z4 = make_uint4(0u, 0u, 0u, 0u);
    for (int j0 = 2 * warp; j0 < nent; j0 += 2 * RT_WARPS) {
        const int j1 = j0 + 1;
        const bool two = j1 < nent;
        const uint4* s0 = xs + size_t(t0 + j0 / k) * row16;
        const uint4* s1 = xs + size_t(t0 + (two ? j1 : j0) / k) * row16;
        uint4* d0 = xd + size_t(s_pos[j0]) * row16;
        uint4* d1 = xd + size_t(s_pos[two ? j1 : j0]) * row16;
        for (int c0 = 0; c0 < row16; c0 += 32 * 8) {
            uint4 a[8], b[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int c = c0 + 32 * i + lane;
                a[i] = c < row16 ? __ldg(s0 + c) : z4;
                b[i] = (two && c < row16) ? __ldg(s1 + c) : z4;
            }
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int c = c0 + 32 * i + lane;
                if (c < row16) {
                    d0[c] = a[i];
                    if (two) d1[c] = b[i];
                }
            }
        }
    }
}

int route_smem_bytes(int E, int tpb, int k) { return 4 * (3 * E + 1 + 32 + 2 * tpb * k); }

}  // namespace

redmoe_status launch_route(const redmoe_layer* L, const void* x, int T, const float* logits, int32_t* ids, float* w,
                           float* sgate, int32_t* counts, int32_t* offsets, int32_t* perm, int tile_m,
                           int32_t* tiles, void* xg, int32_t* bhist, Control* ctl, cudaStream_t stream,
                           int* launches, CacheBias cb) {
    DevInfo di;
    if (!get_dev_info(&di)) return REDMOE_ERR_CUDA;
    const int E = L->n_experts, k = L->top_k;
    const int nb = di.sm_count < ROUTE_MAX_BLOCKS ? di.sm_count : ROUTE_MAX_BLOCKS;
    RouteParams p;
    p.logits = logits;
    p.x = static_cast<const uint16_t*>(x);
    p.g = static_cast<const uint16_t*>(L->shared_gate_w);
    p.T = T; p.E = E; p.k = k; p.H = L->hidden;
    p.tpb = (T + nb - 1) / nb;
    p.ids = ids; p.w = w; p.sgate = sgate;
    p.counts = counts; p.offsets = offsets; p.perm = perm; p.tile_m = tile_m; p.tiles = tiles;
    p.xg = static_cast<uint16_t*>(xg); p.bhist = bhist; p.ctl = ctl; p.timeout_ns = BARRIER_TIMEOUT_NS;
    p.cb = cb;
    const int smem = route_smem_bytes(E, p.tpb, k);
    if (smem > di.max_smem_optin) return REDMOE_ERR_UNSUPPORTED;
    void (*kern)(RouteParams) = E <= 256 ? route_kernel<8> : (E <= 512 ? route_kernel<16> : route_kernel<MAX_EXPERTS / 32>);
    if (smem > 48 * 1024 &&
        cudaFuncSetAttribute(reinterpret_cast<const void*>(kern), cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
            cudaSuccess)
        return REDMOE_ERR_CUDA;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(unsigned(nb));
    cfg.blockDim = dim3(RT_THREADS);
    cfg.dynamicSmemBytes = size_t(smem);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, kern, p) != cudaSuccess) return REDMOE_ERR_CUDA;
    if (launches) *launches += 1;
    return REDMOE_OK;
}

}  // namespace redmoe
