// Routed experts that live in host memory, served through a bounded device cache.
//
// The pages keep only the dense and shared weights resident and stream routed experts
// into a bounded expert cache: per-expert hotness halved every 16 tokens ("Research notes,
// October 2026", section 1, SSD streaming bullets), a bounded shared expert cache with
// router-driven prefetch for the next MoE layer ("Architecture", "Future native Red Metal
// path"). On B200 the slow tier is pinned host memory that the GPU reads directly over
// the host link, and the cache is a set of device slots, each holding one expert's three
// matrices. One decode call (T = 1) is four launches on the caller's stream, with no host
// round trip:
//
//   1 router      logits, top-k and weights (the router entry point's kernels)
//   2 directory   one block: hotness += 1 for each selected expert, halved when the token
//                 count crosses a multiple of 16; each selected expert that is not
//                 resident takes a free slot, else the slot of the resident expert with
//                 the lowest hotness that this call does not use (ties to the lower slot);
//                 the (expert, slot) fills are listed for step 3
//   3 fill        every SM copies the listed experts from host memory into their slots
//                 with 16-byte loads over the host link
//   4 experts     the one-row decode kernel with the routing of step 1, reading routed
//                 expert e from slot slot_of[e]
//
// The directory step is deterministic (misses are listed in expert order, victims are
// chosen by (free first, hotness, slot)), so the cache state after a sequence of calls
// depends only on the routing.
#include <string.h>

#include "common.cuh"
#include "internal.h"

namespace redmoe {

redmoe_status launch_router(const redmoe_layer* L, const void* x, int T, float* logits, int32_t* ids, float* w,
                            float* sgate, cudaStream_t stream, int* launches);

namespace {

constexpr int EC_THREADS = 1024;
constexpr int EC_MAX_FILL = DECODE_MAX_T * MAX_TOPK;
constexpr int HALVE_EVERY = 16;  // tokens between halvings of the hotness

struct DirParams {
    const int32_t* ids;  // [n] expert ids of this call (T * k routed slots, or a prefetch list)
    int n, E, S;
    int count_use;       // 1: a routed call (hotness, tokens, hits); 0: a prefetch
    int tokens;          // tokens of this call (count_use)
    int32_t* slot_of;    // [E]
    int32_t* expert_in;  // [S]
    float* hot;          // [E]
    int32_t* stats;      // [4]: tokens, hits, misses, prefetch fills
    int32_t* fill;       // [1 + 2 * EC_MAX_FILL]: count, then (expert, slot) pairs
    Control* ctl;
};

__device__ __forceinline__ int block_excl_scan(int v, int* wsum, int& total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int inc = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(FULL, inc, o);
        if (lane >= o) inc += y;
    }
    if (lane == 31) wsum[warp] = inc;
    __syncthreads();
    if (warp == 0) {
        const int ws = lane < EC_THREADS / 32 ? wsum[lane] : 0;
        int wi = ws;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(FULL, wi, o);
            if (lane >= o) wi += y;
        }
        wsum[lane] = wi - ws;
        if (lane == 31) wsum[32] = wi;
    }
    __syncthreads();
    total = wsum[32];
    const int ex = wsum[warp] + inc - v;
    __syncthreads();
    return ex;
}

__global__ void __launch_bounds__(EC_THREADS) directory_kernel(const __grid_constant__ DirParams p) {
    __shared__ int uses[MAX_EXPERTS];
    __shared__ int miss[EC_MAX_FILL];
    __shared__ int wsum[33];
    __shared__ unsigned long long best;
    const int t = threadIdx.x;
    for (int e = t; e < p.E; e += EC_THREADS) uses[e] = 0;
    __syncthreads();
    for (int i = t; i < p.n; i += EC_THREADS) {
        const int e = p.ids[i];
        if (e >= 0 && e < p.E) atomicAdd(&uses[e], 1);
        else atomicOr(&p.ctl->err, ERRBIT_STATE);
    }
    __syncthreads();
    // hotness: + uses, halved when the token count crosses a multiple of HALVE_EVERY
    const int tok0 = p.stats[0];
    const bool halve = p.count_use && (tok0 / HALVE_EVERY != (tok0 + p.tokens) / HALVE_EVERY);
    // misses in expert order (E <= EC_THREADS: one expert per thread)
    int is_miss = 0, hits = 0;
    if (t < p.E) {
        if (p.count_use) {
            float h = p.hot[t] + float(uses[t]);
            if (halve) h *= 0.5f;
            p.hot[t] = h;
        }
        if (uses[t] > 0) {
            if (p.slot_of[t] < 0) is_miss = 1;
            else hits = 1;
        }
    }
    int nmiss = 0;
    const int pos = block_excl_scan(is_miss, wsum, nmiss);
    if (is_miss && pos < EC_MAX_FILL) miss[pos] = t;
    int nhit = 0;
    block_excl_scan(hits, wsum, nhit);
    if (nmiss > EC_MAX_FILL) nmiss = EC_MAX_FILL;
    // one victim per miss: free slots first, then the lowest hotness among resident experts
    // this call does not use, ties to the lower slot
    for (int m = 0; m < nmiss; ++m) {
        if (t == 0) best = ~0ull;
        __syncthreads();
        unsigned long long mine = ~0ull;
        for (int s = t; s < p.S; s += EC_THREADS) {
            const int r = p.expert_in[s];
            unsigned long long key;
            if (r < 0) key = uint64_t(s);                                   // free
            else if (uses[r] > 0) key = ~0ull;                              // needed now
            else key = (1ull << 62) | (uint64_t(__float_as_uint(p.hot[r])) << 30) | uint64_t(s);
            mine = key < mine ? key : mine;
        }
        atomicMin(&best, mine);
        __syncthreads();
        if (t == 0) {
            const int e = miss[m];
            if (best == ~0ull) {  // no slot left (more experts than slots): report, do not fill
                atomicOr(&p.ctl->err, ERRBIT_STATE);
                p.fill[1 + 2 * m] = -1;
                p.fill[2 + 2 * m] = -1;
            } else {
                const int s = int(best & ((1ull << 30) - 1));
                const int old = p.expert_in[s];
                if (old >= 0) p.slot_of[old] = -1;
                p.expert_in[s] = e;
                p.slot_of[e] = s;
                uses[e] = uses[e] > 0 ? uses[e] : 1;  // the slot is taken for the next rounds
                p.fill[1 + 2 * m] = e;
                p.fill[2 + 2 * m] = s;
            }
            __threadfence_block();
        }
        __syncthreads();
    }
    if (t == 0) {
        p.fill[0] = nmiss;
        if (p.count_use) {
            p.stats[0] = tok0 + p.tokens;
            p.stats[1] += nhit;
            p.stats[2] += nmiss;
        } else {
            p.stats[3] += nmiss;
        }
    }
}

struct FillParams {
    const int32_t* fill;
    const uint4* src[6];  // home copies: gate, up, down codes, then their scales (or null)
    uint4* dst[6];        // slot stacks in the same order
    uint64_t n16[6];      // 16-byte chunks of one expert's tensor
};

// Copy the listed experts from their home (host memory, read over the host link) into
// their slots. Every thread walks the chunks of all fills with a grid stride, four
// 16-byte loads in flight per thread.
__global__ void __launch_bounds__(512) fill_kernel(const __grid_constant__ FillParams p) {
    const int nf = p.fill[0];
    const uint64_t stride = uint64_t(gridDim.x) * blockDim.x;
    const uint64_t gid = uint64_t(blockIdx.x) * blockDim.x + threadIdx.x;
    for (int f = 0; f < nf; ++f) {
        const int e = p.fill[1 + 2 * f], s = p.fill[2 + 2 * f];
        if (e < 0 || s < 0) continue;
        for (int q = 0; q < 6; ++q) {
            if (!p.src[q]) continue;
            const uint4* a = p.src[q] + uint64_t(e) * p.n16[q];
            uint4* b = p.dst[q] + uint64_t(s) * p.n16[q];
            const uint64_t n = p.n16[q];
            uint64_t i = gid;
            for (; i + 3 * stride < n; i += 4 * stride) {
                const uint4 v0 = ld_stream(a + i), v1 = ld_stream(a + i + stride);
                const uint4 v2 = ld_stream(a + i + 2 * stride), v3 = ld_stream(a + i + 3 * stride);
                b[i] = v0;
                b[i + stride] = v1;
                b[i + 2 * stride] = v2;
                b[i + 3 * stride] = v3;
            }
            for (; i < n; i += stride) b[i] = ld_stream(a + i);
        }
    }
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Device address through which kernels read `p` (device memory, or pinned host memory
// mapped into the device's address space); null if the GPU cannot read it.
const void* device_view(const void* p) {
    cudaPointerAttributes a;
    if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
        cudaGetLastError();
        return nullptr;
    }
    if (a.type == cudaMemoryTypeDevice || a.type == cudaMemoryTypeManaged) return p;
    if (a.type == cudaMemoryTypeHost) return a.devicePointer;
    return nullptr;
}

long elem_bytes_row(int dt, int K) { return dt == DT_INT4 ? K / 2 : (dt == DT_INT2 ? K / 4 : 2L * K); }

redmoe_status check_cache(const redmoe_layer* L, const redmoe_expert_cache* c, int T) {
    if (!c || c->n_slots < T * L->top_k || c->n_slots >= (1 << 30)) return REDMOE_ERR_INVALID_ARG;
    const void* need[] = {c->slot_gate, c->slot_up, c->slot_down, c->slot_of, c->expert_in, c->hot, c->stats, c->fill};
    for (const void* q : need)
        if (!q || !aligned16(q)) return REDMOE_ERR_INVALID_ARG;
    if (L->expert_dtype != DT_BF16) {
        const void* sc[] = {c->slot_s_gate, c->slot_s_up, c->slot_s_down};
        for (const void* q : sc)
            if (!q || !aligned16(q)) return REDMOE_ERR_INVALID_ARG;
    }
    return REDMOE_OK;
}

// Fill parameters of a layer's routed stacks (home views resolved) and a cache's slots.
bool fill_params(const redmoe_layer* L, const redmoe_expert_cache* c, FillParams* f) {
    const int H = L->hidden, I = L->inter, wt = L->expert_dtype;
    const void* home[6] = {L->w_gate, L->w_up, L->w_down, L->s_gate, L->s_up, L->s_down};
    void* slot[6] = {c->slot_gate, c->slot_up, c->slot_down, c->slot_s_gate, c->slot_s_up, c->slot_s_down};
    const uint64_t bytes[6] = {uint64_t(I) * elem_bytes_row(wt, H), uint64_t(I) * elem_bytes_row(wt, H),
                               uint64_t(H) * elem_bytes_row(wt, I), uint64_t(I) * (H / 16), uint64_t(I) * (H / 16),
                               uint64_t(H) * (I / 16)};
    for (int q = 0; q < 6; ++q) {
        const bool used = q < 3 || wt != DT_BF16;
        f->src[q] = nullptr;
        f->dst[q] = nullptr;
        f->n16[q] = 0;
        if (!used) continue;
        if (bytes[q] % 16) return false;
        const void* v = device_view(home[q]);
        if (!v || !aligned16(v)) return false;
        f->src[q] = static_cast<const uint4*>(v);
        f->dst[q] = static_cast<uint4*>(slot[q]);
        f->n16[q] = bytes[q] / 16;
    }
    return true;
}

redmoe_status run_directory_and_fill(const redmoe_layer* L, redmoe_expert_cache* c, const int32_t* ids, int n,
                                     int count_use, int tokens, Control* ctl, cudaStream_t s) {
    DirParams d;
    d.ids = ids;
    d.n = n;
    d.E = L->n_experts;
    d.S = c->n_slots;
    d.count_use = count_use;
    d.tokens = tokens;
    d.slot_of = c->slot_of;
    d.expert_in = c->expert_in;
    d.hot = c->hot;
    d.stats = c->stats;
    d.fill = c->fill;
    d.ctl = ctl;
    FillParams f;
    if (!fill_params(L, c, &f)) return REDMOE_ERR_INVALID_ARG;
    f.fill = c->fill;
    directory_kernel<<<1, EC_THREADS, 0, s>>>(d);
    if (cudaGetLastError() != cudaSuccess) return REDMOE_ERR_CUDA;
    DevInfo di;
    if (!get_dev_info(&di)) return REDMOE_ERR_CUDA;
    fill_kernel<<<2 * di.sm_count, 512, 0, s>>>(f);
    return cudaGetLastError() == cudaSuccess ? REDMOE_OK : REDMOE_ERR_CUDA;
}

}  // namespace

}  // namespace redmoe

using namespace redmoe;

extern "C" {

size_t redmoe_expert_cache_slot_bytes(const redmoe_layer* L) {
    if (check_layer(L) != REDMOE_OK) return 0;
    const int H = L->hidden, I = L->inter, wt = L->expert_dtype;
    size_t b = size_t(3) * I * elem_bytes_row(wt, H);
    if (wt != DT_BF16) b += size_t(3) * I * (H / 16);
    return b;
}

redmoe_status redmoe_expert_cache_init(const redmoe_layer* L, redmoe_expert_cache* c, void* stream) {
    redmoe_status st = check_layer(L);
    if (st != REDMOE_OK) return st;
    if ((st = check_cache(L, c, 1)) != REDMOE_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (cudaMemsetAsync(c->slot_of, 0xff, sizeof(int32_t) * L->n_experts, s) != cudaSuccess ||
        cudaMemsetAsync(c->expert_in, 0xff, sizeof(int32_t) * c->n_slots, s) != cudaSuccess ||
        cudaMemsetAsync(c->hot, 0, sizeof(float) * L->n_experts, s) != cudaSuccess ||
        cudaMemsetAsync(c->stats, 0, sizeof(int32_t) * 4, s) != cudaSuccess ||
        cudaMemsetAsync(c->fill, 0, sizeof(int32_t) * (1 + 2 * EC_MAX_FILL), s) != cudaSuccess)
        return REDMOE_ERR_CUDA;
    return REDMOE_OK;
}

redmoe_status redmoe_forward_host_experts(const redmoe_layer* L, const void* x, int32_t T, float* out,
                                          int32_t* topk_ids, float* topk_w, redmoe_expert_cache* cache,
                                          void* workspace, size_t workspace_bytes, void* stream) {
    redmoe_status st = check_layer(L);
    if (st != REDMOE_OK) return st;
    if (T < 0) return REDMOE_ERR_INVALID_ARG;
    if (T == 0) return REDMOE_OK;
    if (T != 1 || !decode1_shape_ok(L)) return REDMOE_ERR_UNSUPPORTED;
    if (!x || !out || !topk_ids || !topk_w || !aligned16(x) || !aligned16(out) ||
        reinterpret_cast<uintptr_t>(topk_ids) % 4 || reinterpret_cast<uintptr_t>(topk_w) % 4)
        return REDMOE_ERR_INVALID_ARG;
    if ((st = check_cache(L, cache, T)) != REDMOE_OK) return st;
    if (!workspace || reinterpret_cast<uintptr_t>(workspace) % 256 ||
        workspace_bytes < redmoe_workspace_bytes(L, T))
        return REDMOE_ERR_WORKSPACE;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    char* ws = static_cast<char*>(workspace);
    Control* ctl = reinterpret_cast<Control*>(ws);
    const DecodeWs dl = decode_ws_layout(T, L->n_experts, L->top_k, L->inter, L->shared_inter);
    // 1 router (its shared-gate output lands in the decode kernel's scratch, unused there)
    if ((st = launch_router(L, x, T, reinterpret_cast<float*>(ws + dl.logits), topk_ids, topk_w,
                            reinterpret_cast<float*>(ws + dl.sgate), s, nullptr)) != REDMOE_OK)
        return st;
    // 2, 3 directory and fills
    if ((st = run_directory_and_fill(L, cache, topk_ids, T * L->top_k, 1, T, ctl, s)) != REDMOE_OK) return st;
    // 4 experts from the slots, with the routing of step 1
    DecLayer d = dec_layer(L, x, out, topk_ids, topk_w);
    d.w_gate = cache->slot_gate;
    d.w_up = cache->slot_up;
    d.w_down = cache->slot_down;
    d.s_gate = static_cast<const uint16_t*>(cache->slot_s_gate);
    d.s_up = static_cast<const uint16_t*>(cache->slot_s_up);
    d.s_down = static_cast<const uint16_t*>(cache->slot_s_down);
    d.given_ids = topk_ids;
    d.given_w = topk_w;
    d.slot_of = cache->slot_of;
    return launch_decode1(L, &d, 1, workspace, s, nullptr, CacheBias{nullptr, 0.0f});
}

redmoe_status redmoe_expert_cache_prefetch(const redmoe_layer* L, redmoe_expert_cache* cache, const int32_t* ids,
                                           int32_t n, void* workspace, size_t workspace_bytes, void* stream) {
    redmoe_status st = check_layer(L);
    if (st != REDMOE_OK) return st;
    if (n < 0 || n > EC_MAX_FILL) return REDMOE_ERR_INVALID_ARG;
    if (n == 0) return REDMOE_OK;
    if (!ids || reinterpret_cast<uintptr_t>(ids) % 4) return REDMOE_ERR_INVALID_ARG;
    if ((st = check_cache(L, cache, 1)) != REDMOE_OK) return st;
    if (cache->n_slots < n) return REDMOE_ERR_INVALID_ARG;
    if (!workspace || reinterpret_cast<uintptr_t>(workspace) % 256 || workspace_bytes < 256)
        return REDMOE_ERR_WORKSPACE;
    return run_directory_and_fill(L, cache, ids, n, 0, 0, static_cast<Control*>(workspace),
                                  static_cast<cudaStream_t>(stream));
}

}  // extern "C"
