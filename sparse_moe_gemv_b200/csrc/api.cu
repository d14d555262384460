// C ABI of libredmoe: argument validation, workspace carve-up and kernel dispatch.
#include <string.h>

#include <mutex>
#include <new>
#include <vector>

#include "common.cuh"
#include "internal.h"

namespace redmoe {

redmoe_status launch_router(const redmoe_layer* L, const void* x, int T, float* logits, int32_t* ids, float* w,
                            float* sgate, cudaStream_t stream, int* launches);
redmoe_status launch_route_build(const int32_t* ids, int T, int k, int E, int32_t* counts, int32_t* offsets,
                                 int32_t* perm, int tile_m, int32_t* tiles, cudaStream_t stream, int* launches);
int route_build_smem_bytes(int E);

bool get_dev_info(DevInfo* out) {
    static std::mutex mu;
    static std::vector<DevInfo> cache;
    static std::vector<bool> have;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return false;
    std::lock_guard<std::mutex> lock(mu);
    if (dev >= int(cache.size())) {
        cache.resize(dev + 1);
        have.resize(dev + 1, false);
    }
    if (!have[dev]) {
        DevInfo d;
        if (cudaDeviceGetAttribute(&d.sm_count, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return false;
        if (cudaDeviceGetAttribute(&d.max_smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess)
            return false;
        cache[dev] = d;
        have[dev] = true;
    }
    *out = cache[dev];
    return true;
}

// Copy n16 16-byte chunks from pinned host memory (its device mapping) into device memory
// with cache-volatile loads. For small inputs a kernel reading over the link ends several
// microseconds sooner than a copy-engine transfer of the same bytes.
static __global__ void stage_from_host_kernel(const uint4* __restrict__ src, uint4* __restrict__ dst, size_t n16) {
    for (size_t i = size_t(blockIdx.x) * blockDim.x + threadIdx.x; i < n16; i += size_t(gridDim.x) * blockDim.x)
        dst[i] = __ldcv(src + i);
}

namespace {

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

int elems_per_chunk(int dt) { return dt == DT_F32 ? 4 : (dt == DT_BF16 ? 8 : (dt == DT_INT4 ? 32 : 64)); }

// Workspace carve-up of the router entry point and of the batched path.
struct BatchWs {
    size_t logits, sgate, total;
};
BatchWs batch_ws_layout(int T, int E) {
    BatchWs b;
    size_t o = 256;
    b.logits = o; o = align256(o + 4ull * T * E);
    b.sgate = o; o = align256(o + 4ull * T);
    b.total = o;
    return b;
}

size_t ws_bytes(const redmoe_layer* L, int T) {
    size_t need = 256;
    if (T <= DECODE_MAX_T) {
        const DecodeWs d = decode_ws_layout(T, L->n_experts, L->top_k, L->inter, L->shared_inter);
        need = d.total > need ? d.total : need;
    } else if (batch_shape_ok(L)) {
        const BatchLayout g = batch_layout(T, L->n_experts, L->top_k, L->hidden, L->inter);
        need = g.total > need ? g.total : need;
    }
    const BatchWs b = batch_ws_layout(T, L->n_experts);
    need = b.total > need ? b.total : need;
    return need;
}

redmoe_status check_ws(const redmoe_layer* L, int T, const void* ws, size_t bytes) {
    if (!ws || !aligned(ws, 256)) return REDMOE_ERR_WORKSPACE;
    if (bytes < ws_bytes(L, T)) return REDMOE_ERR_WORKSPACE;
    return REDMOE_OK;
}

redmoe_status cuda_ok(cudaError_t e) { return e == cudaSuccess ? REDMOE_OK : REDMOE_ERR_CUDA; }

}  // namespace

// Shape, dtype and pointer checks common to every layer entry point.
redmoe_status check_layer(const redmoe_layer* L) {
    if (!L) return REDMOE_ERR_INVALID_ARG;
    const int H = L->hidden, E = L->n_experts, k = L->top_k, I = L->inter, Is = L->shared_inter;
    if (H <= 0 || E <= 0 || k <= 0 || I <= 0 || Is <= 0) return REDMOE_ERR_INVALID_ARG;
    if (k > E || k > MAX_TOPK || E > MAX_EXPERTS) return REDMOE_ERR_INVALID_ARG;
    const int xt = L->x_dtype, rt = L->router_dtype, wt = L->expert_dtype;
    if (xt < 0 || xt > 3 || rt < 0 || rt > 3 || wt < 0 || wt > 3) return REDMOE_ERR_INVALID_ARG;
    if (xt == DT_INT4 || rt == DT_INT4 || xt == DT_INT2 || rt == DT_INT2) return REDMOE_ERR_INVALID_ARG;
    const bool combo = (xt == DT_F32 && rt == DT_F32 && wt == DT_F32) ||
                       (xt == DT_BF16 && rt == DT_BF16 && (wt == DT_BF16 || wt == DT_INT4 || wt == DT_INT2));
    if (!combo) return REDMOE_ERR_UNSUPPORTED;
    // every row is read in 16-byte chunks; int4 rows also in whole scale groups
    if (H % 32 || I % 32 || Is % 32) return REDMOE_ERR_INVALID_ARG;
    if (H % elems_per_chunk(wt) || I % elems_per_chunk(wt) || Is % elems_per_chunk(wt)) return REDMOE_ERR_INVALID_ARG;
    const void* need[] = {L->router_w, L->shared_gate_w, L->w_gate, L->w_up, L->w_down, L->sh_gate, L->sh_up, L->sh_down};
    for (const void* p : need)
        if (!p || !aligned(p, 16)) return REDMOE_ERR_INVALID_ARG;
    if (L->router_bias && !aligned(L->router_bias, 4)) return REDMOE_ERR_INVALID_ARG;
    const void* sc[] = {L->s_gate, L->s_up, L->s_down, L->sh_s_gate, L->sh_s_up, L->sh_s_down};
    for (const void* p : sc) {
        if (wt == DT_INT4 || wt == DT_INT2) {
            if (!p || !aligned(p, 16)) return REDMOE_ERR_INVALID_ARG;
        }
    }
    return REDMOE_OK;
}

DecLayer dec_layer(const redmoe_layer* L, const void* x, float* out, int32_t* ids, float* w) {
    DecLayer d;
    d.router_w = L->router_w;
    d.router_bias = L->router_bias;
    d.shared_gate_w = L->shared_gate_w;
    d.w_gate = L->w_gate;
    d.w_up = L->w_up;
    d.w_down = L->w_down;
    d.s_gate = static_cast<const uint16_t*>(L->s_gate);
    d.s_up = static_cast<const uint16_t*>(L->s_up);
    d.s_down = static_cast<const uint16_t*>(L->s_down);
    d.sh_gate = L->sh_gate;
    d.sh_up = L->sh_up;
    d.sh_down = L->sh_down;
    d.sh_s_gate = static_cast<const uint16_t*>(L->sh_s_gate);
    d.sh_s_up = static_cast<const uint16_t*>(L->sh_s_up);
    d.sh_s_down = static_cast<const uint16_t*>(L->sh_s_down);
    d.x = x;
    d.out = out;
    d.ids = ids;
    d.w = w;
    d.given_ids = nullptr;
    d.given_w = nullptr;
    d.slot_of = nullptr;
    return d;
}


}  // namespace redmoe

using namespace redmoe;

extern "C" {

int32_t redmoe_abi_version(void) { return REDMOE_ABI_VERSION; }

const char* redmoe_status_string(int32_t s) {
    switch (s) {
        case REDMOE_OK: return "ok";
        case REDMOE_ERR_INVALID_ARG: return "invalid argument";
        case REDMOE_ERR_UNSUPPORTED: return "unsupported configuration";
        case REDMOE_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
        case REDMOE_ERR_CUDA: return "CUDA error";
        case REDMOE_ERR_TIMEOUT: return "in-kernel wait timed out";
        default: return "unknown status";
    }
}

size_t redmoe_workspace_bytes(const redmoe_layer* L, int32_t T) {
    if (T < 0 || check_layer(L) == REDMOE_ERR_INVALID_ARG || !L) return 0;
    return ws_bytes(L, T);
}

redmoe_status redmoe_workspace_init(void* workspace, size_t workspace_bytes, void* stream) {
    if (!workspace) {  // the allocation-free scratch of this device
        void* scratch = noalloc_scratch_address();
        if (!scratch) return REDMOE_ERR_CUDA;
        return cuda_ok(cudaMemsetAsync(scratch, 0, 256, static_cast<cudaStream_t>(stream)));
    }
    if (!aligned(workspace, 256) || workspace_bytes < 256) return REDMOE_ERR_WORKSPACE;
    return cuda_ok(cudaMemsetAsync(workspace, 0, 256, static_cast<cudaStream_t>(stream)));
}

redmoe_status redmoe_forward(const redmoe_layer* L, const void* x, int32_t T, float* out, int32_t* topk_ids,
                             float* topk_w, void* workspace, size_t workspace_bytes, const redmoe_route_debug* dbg,
                             void* stream) {
    redmoe_status st = check_layer(L);
    if (st != REDMOE_OK) return st;
    if (T < 0) return REDMOE_ERR_INVALID_ARG;
    if (T == 0) return REDMOE_OK;
    if (!x || !out || !topk_ids || !topk_w) return REDMOE_ERR_INVALID_ARG;
    if (!aligned(x, 16) || !aligned(out, 16) || !aligned(topk_ids, 4) || !aligned(topk_w, 4))
        return REDMOE_ERR_INVALID_ARG;
    if (dbg && (!dbg->counts || !dbg->offsets || !dbg->perm)) return REDMOE_ERR_INVALID_ARG;
    if ((st = check_ws(L, T, workspace, workspace_bytes)) != REDMOE_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (T > DECODE_MAX_T) {
        if (!batch_shape_ok(L)) return REDMOE_ERR_UNSUPPORTED;
        if ((long long)T * L->top_k + T > (1ll << 30)) return REDMOE_ERR_INVALID_ARG;
        return launch_batched(L, x, T, out, topk_ids, topk_w, workspace, dbg, s, nullptr);
    }
    const DecLayer d = dec_layer(L, x, out, topk_ids, topk_w);
    st = launch_decode(L, &d, 1, T, workspace, s, nullptr);
    if (st != REDMOE_OK) return st;
    if (dbg)
        st = launch_route_build(topk_ids, T, L->top_k, L->n_experts, dbg->counts, dbg->offsets, dbg->perm, 0,
                                nullptr, s, nullptr);
    return st;
}

namespace {

// Device staging of redmoe_forward_host, after the forward's own workspace: x, then out,
// ids and w (each 256-byte aligned).
struct HostStage {
    size_t x, out, ids, w, total;
};
HostStage host_stage_layout(const redmoe_layer* L, int T) {
    HostStage h;
    const size_t xb = L->x_dtype == DT_F32 ? 4 : 2;
    size_t o = ws_bytes(L, T);
    h.x = o; o = align256(o + xb * T * L->hidden);
    h.out = o; o = align256(o + 4ull * T * L->hidden);
    h.ids = o; o = align256(o + 4ull * T * L->top_k);
    h.w = o; o = align256(o + 4ull * T * L->top_k);
    h.total = o;
    return h;
}

constexpr size_t STAGE_KERNEL_MAX = 64 * 1024;  // bytes: above this the copy engine is used

// The device mapping of pinned host memory (or the pointer itself for device memory);
// null for memory the device cannot write (pageable host memory).
void* writable_view(void* p) {
    cudaPointerAttributes a;
    if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
        cudaGetLastError();
        return nullptr;
    }
    if (a.type == cudaMemoryTypeDevice || a.type == cudaMemoryTypeManaged) return p;
    if (a.type == cudaMemoryTypeHost) return a.devicePointer;
    return nullptr;
}

// The decode launches of host-memory x (layers[l].x mapped pinned memory, T rows staged at
// xstage): T = 1 and 2 on their kernels, T = 3 and 4 as rows 0-1 plus the rest.
redmoe_status launch_decode_host_x(const redmoe_layer* L, const DecLayer* d, int n, int T, void* ws, char* xstage,
                                   cudaStream_t s) {
    if (T == 1) return launch_decode1_host_x(L, d, n, ws, xstage, s);
    if (T == 2) return launch_decodefr_host_x(L, d, n, 2, ws, xstage, s);
    redmoe_status st = launch_decodefr_host_x(L, d, n, 2, ws, xstage, s);
    if (st != REDMOE_OK) return st;
    const std::vector<DecLayer> rest = dec_rows(L, d, n, 2);
    char* xs2 = xstage + size_t(2) * L->hidden * (L->x_dtype == DT_F32 ? 4 : 2);
    return T == 3 ? launch_decode1_host_x(L, rest.data(), n, ws, xs2, s)
                  : launch_decodefr_host_x(L, rest.data(), n, 2, ws, xs2, s);
}

bool host_x_ok(const redmoe_layer* L, int T) {
    return (T == 1 && decode1_shape_ok(L)) || decodefr_shape_ok(L, T) || decode_split_ok(L, T);
}

}  // namespace

size_t redmoe_workspace_bytes_host(const redmoe_layer* L, int32_t T) {
    if (T < 0 || check_layer(L) == REDMOE_ERR_INVALID_ARG || !L) return 0;
    return host_stage_layout(L, T).total;
}

redmoe_status redmoe_forward_host(const redmoe_layer* L, const void* x_host, int32_t T, float* out_host,
                                  int32_t* ids_host, float* w_host, void* workspace, size_t workspace_bytes,
                                  void* stream) {
    redmoe_status st = check_layer(L);
    if (st != REDMOE_OK) return st;
    if (T < 0) return REDMOE_ERR_INVALID_ARG;
    if (T == 0) return REDMOE_OK;
    if (!x_host || !out_host || !ids_host || !w_host) return REDMOE_ERR_INVALID_ARG;
    if (!aligned(x_host, 16) || !aligned(out_host, 16) || !aligned(ids_host, 4) || !aligned(w_host, 4))
        return REDMOE_ERR_INVALID_ARG;
    if (!workspace || !aligned(workspace, 256)) return REDMOE_ERR_WORKSPACE;
    const HostStage h = host_stage_layout(L, T);
    if (workspace_bytes < h.total) return REDMOE_ERR_WORKSPACE;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    char* base = static_cast<char*>(workspace);
    if (host_x_ok(L, T)) {
        // decode rows with every buffer pinned: the kernels read x over the link once
        // (staged in the workspace) and store the results straight back, so no copy is
        // enqueued at all
        const void* xv = writable_view(const_cast<void*>(x_host));
        float* o = static_cast<float*>(writable_view(out_host));
        int32_t* i = static_cast<int32_t*>(writable_view(ids_host));
        float* w = static_cast<float*>(writable_view(w_host));
        if (xv && o && i && w) {
            const DecLayer d = dec_layer(L, xv, o, i, w);
            return launch_decode_host_x(L, &d, 1, T, workspace, base + h.x, s);
        }
    }
    const size_t xbytes = (L->x_dtype == DT_F32 ? 4ull : 2ull) * T * L->hidden;
    const void* xv = xbytes <= STAGE_KERNEL_MAX ? writable_view(const_cast<void*>(x_host)) : nullptr;
    if (xv) {
        const size_t n16 = xbytes / 16;  // hidden is a multiple of 32: whole chunks
        stage_from_host_kernel<<<unsigned((n16 + 255) / 256), 256, 0, s>>>(static_cast<const uint4*>(xv),
                                                                            reinterpret_cast<uint4*>(base + h.x), n16);
        if (cudaGetLastError() != cudaSuccess) return REDMOE_ERR_CUDA;
    } else if (cudaMemcpyAsync(base + h.x, x_host, xbytes, cudaMemcpyDefault, s) != cudaSuccess) {
        return REDMOE_ERR_CUDA;
    }
    if (T <= DECODE_MAX_T) {
        // the decode kernels store each result once: straight into mapped host memory
        float* o = static_cast<float*>(writable_view(out_host));
        int32_t* i = static_cast<int32_t*>(writable_view(ids_host));
        float* w = static_cast<float*>(writable_view(w_host));
        if (o && i && w)
            return redmoe_forward(L, base + h.x, T, o, i, w, workspace, workspace_bytes, nullptr, stream);
    }
    float* o = reinterpret_cast<float*>(base + h.out);
    int32_t* i = reinterpret_cast<int32_t*>(base + h.ids);
    float* w = reinterpret_cast<float*>(base + h.w);
    if ((st = redmoe_forward(L, base + h.x, T, o, i, w, workspace, workspace_bytes, nullptr, stream)) != REDMOE_OK)
        return st;
    const size_t kb = 4ull * T * L->top_k;
    if (cudaMemcpyAsync(out_host, o, 4ull * T * L->hidden, cudaMemcpyDefault, s) != cudaSuccess ||
        cudaMemcpyAsync(ids_host, i, kb, cudaMemcpyDefault, s) != cudaSuccess ||
        cudaMemcpyAsync(w_host, w, kb, cudaMemcpyDefault, s) != cudaSuccess)
        return REDMOE_ERR_CUDA;
    return REDMOE_OK;
}

redmoe_status redmoe_forward_cached(const redmoe_layer* L, const void* x, int32_t T, float* out, int32_t* topk_ids,
                                    float* topk_w, const uint8_t* cached, float lambda, void* workspace,
                                    size_t workspace_bytes, void* stream) {
    redmoe_status st = check_layer(L);
    if (st != REDMOE_OK) return st;
    if (T < 0 || !(lambda >= 0.0f) || !(lambda <= 3.0e38f)) return REDMOE_ERR_INVALID_ARG;
    if (T == 0) return REDMOE_OK;
    if (!x || !out || !topk_ids || !topk_w || !cached) return REDMOE_ERR_INVALID_ARG;
    if (!aligned(x, 16) || !aligned(out, 16) || !aligned(topk_ids, 4) || !aligned(topk_w, 4))
        return REDMOE_ERR_INVALID_ARG;
    if ((st = check_ws(L, T, workspace, workspace_bytes)) != REDMOE_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const CacheBias cb{cached, lambda};
    if (T > DECODE_MAX_T) {
        if (!batch_shape_ok(L)) return REDMOE_ERR_UNSUPPORTED;
        if ((long long)T * L->top_k + T > (1ll << 30)) return REDMOE_ERR_INVALID_ARG;
        return launch_batched(L, x, T, out, topk_ids, topk_w, workspace, nullptr, s, nullptr, cb);
    }
    const DecLayer d = dec_layer(L, x, out, topk_ids, topk_w);
    return launch_decode(L, &d, 1, T, workspace, s, nullptr, cb);
}

redmoe_status redmoe_router(const redmoe_layer* L, const void* x, int32_t T, int32_t* topk_ids, float* topk_w,
                            float* shared_gate, float* logits, void* workspace, size_t workspace_bytes,
                            void* stream) {
    redmoe_status st = check_layer(L);
    if (st != REDMOE_OK) return st;
    if (T < 0) return REDMOE_ERR_INVALID_ARG;
    if (T == 0) return REDMOE_OK;
    if (!x || !topk_ids || !topk_w || !shared_gate || !aligned(x, 16) || !aligned(topk_ids, 4) ||
        !aligned(topk_w, 4) || !aligned(shared_gate, 4) || (logits && !aligned(logits, 4)))
        return REDMOE_ERR_INVALID_ARG;
    if ((st = check_ws(L, T, workspace, workspace_bytes)) != REDMOE_OK) return st;
    const BatchWs b = batch_ws_layout(T, L->n_experts);
    float* lg = logits ? logits : reinterpret_cast<float*>(static_cast<char*>(workspace) + b.logits);
    return launch_router(L, x, T, lg, topk_ids, topk_w, shared_gate,
                         static_cast<cudaStream_t>(stream), nullptr);
}

redmoe_status redmoe_route_build(const int32_t* topk_ids, int32_t T, int32_t k, int32_t E, int32_t* counts,
                                 int32_t* offsets, int32_t* perm, void* workspace, size_t workspace_bytes,
                                 void* stream) {
    (void)workspace;
    (void)workspace_bytes;
    if (T < 0 || k <= 0 || E <= 0 || k > E || k > MAX_TOPK || E > MAX_EXPERTS) return REDMOE_ERR_INVALID_ARG;
    if (!counts || !offsets || !aligned(counts, 4) || !aligned(offsets, 4)) return REDMOE_ERR_INVALID_ARG;
    if (T > 0 && (!topk_ids || !perm || !aligned(topk_ids, 4) || !aligned(perm, 4))) return REDMOE_ERR_INVALID_ARG;
    if ((long long)T * k > (1ll << 30)) return REDMOE_ERR_INVALID_ARG;
    DevInfo di;
    if (!get_dev_info(&di)) return REDMOE_ERR_CUDA;
    if (route_build_smem_bytes(E) > di.max_smem_optin) return REDMOE_ERR_UNSUPPORTED;
    return launch_route_build(topk_ids, T, k, E, counts, offsets, perm, 0, nullptr,
                              static_cast<cudaStream_t>(stream), nullptr);
}

redmoe_status redmoe_forward_stack(const redmoe_layer* layers, int32_t n_layers, const void* const* xs, int32_t T,
                                   float* const* outs, int32_t* const* ids, float* const* ws, void* workspace,
                                   size_t workspace_bytes, void* stream) {
    if (!layers || n_layers < 0 || !xs || !outs || !ids || !ws) return REDMOE_ERR_INVALID_ARG;
    if (n_layers == 0 || T == 0) return T < 0 ? REDMOE_ERR_INVALID_ARG : REDMOE_OK;
    if (T < 0) return REDMOE_ERR_INVALID_ARG;
    redmoe_status st;
    for (int l = 0; l < n_layers; ++l) {
        if ((st = check_layer(&layers[l])) != REDMOE_OK) return st;
        const redmoe_layer& a = layers[0];
        const redmoe_layer& b = layers[l];
        if (a.hidden != b.hidden || a.n_experts != b.n_experts || a.top_k != b.top_k || a.inter != b.inter ||
            a.shared_inter != b.shared_inter || a.x_dtype != b.x_dtype || a.router_dtype != b.router_dtype ||
            a.expert_dtype != b.expert_dtype)
            return REDMOE_ERR_INVALID_ARG;
        if (!xs[l] || !outs[l] || !ids[l] || !ws[l] || !aligned(xs[l], 16) || !aligned(outs[l], 16) ||
            !aligned(ids[l], 4) || !aligned(ws[l], 4))
            return REDMOE_ERR_INVALID_ARG;
    }
    if ((st = check_ws(&layers[0], T, workspace, workspace_bytes)) != REDMOE_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (T > DECODE_MAX_T) {
        for (int l = 0; l < n_layers; ++l) {
            st = redmoe_forward(&layers[l], xs[l], T, outs[l], ids[l], ws[l], workspace, workspace_bytes, nullptr, stream);
            if (st != REDMOE_OK) return st;
        }
        return REDMOE_OK;
    }
    std::vector<DecLayer> d(n_layers);
    for (int l = 0; l < n_layers; ++l) d[l] = dec_layer(&layers[l], xs[l], outs[l], ids[l], ws[l]);
    return launch_decode(&layers[0], d.data(), n_layers, T, workspace, s, nullptr);
}

redmoe_status redmoe_forward_stack_host(const redmoe_layer* layers, int32_t n_layers, const void* const* xs,
                                        int32_t T, float* const* outs, int32_t* const* ids, float* const* ws,
                                        void* workspace, size_t workspace_bytes, void* stream) {
    if (!layers || n_layers < 0 || !xs || !outs || !ids || !ws) return REDMOE_ERR_INVALID_ARG;
    if (n_layers == 0 || T == 0) return T < 0 ? REDMOE_ERR_INVALID_ARG : REDMOE_OK;
    if (T < 0) return REDMOE_ERR_INVALID_ARG;
    redmoe_status st;
    for (int l = 0; l < n_layers; ++l) {
        if ((st = check_layer(&layers[l])) != REDMOE_OK) return st;
        const redmoe_layer& a = layers[0];
        const redmoe_layer& b = layers[l];
        if (a.hidden != b.hidden || a.n_experts != b.n_experts || a.top_k != b.top_k || a.inter != b.inter ||
            a.shared_inter != b.shared_inter || a.x_dtype != b.x_dtype || a.router_dtype != b.router_dtype ||
            a.expert_dtype != b.expert_dtype)
            return REDMOE_ERR_INVALID_ARG;
        if (!xs[l] || !outs[l] || !ids[l] || !ws[l] || !aligned(xs[l], 16) || !aligned(outs[l], 16) ||
            !aligned(ids[l], 4) || !aligned(ws[l], 4))
            return REDMOE_ERR_INVALID_ARG;
    }
    if (!workspace || !aligned(workspace, 256)) return REDMOE_ERR_WORKSPACE;
    const HostStage h = host_stage_layout(&layers[0], T);
    if (workspace_bytes < h.total) return REDMOE_ERR_WORKSPACE;
    if (host_x_ok(&layers[0], T)) {
        // one launch for the whole stack when every buffer is pinned: each layer's x is
        // read over the link by the kernel and its results stored straight back
        std::vector<DecLayer> d(n_layers);
        bool mapped = true;
        for (int l = 0; l < n_layers && mapped; ++l) {
            const void* xv = writable_view(const_cast<void*>(xs[l]));
            float* o = static_cast<float*>(writable_view(outs[l]));
            int32_t* i = static_cast<int32_t*>(writable_view(ids[l]));
            float* w = static_cast<float*>(writable_view(ws[l]));
            mapped = xv && o && i && w;
            if (mapped) d[l] = dec_layer(&layers[l], xv, o, i, w);
        }
        if (mapped)
            return launch_decode_host_x(&layers[0], d.data(), n_layers, T, workspace,
                                        static_cast<char*>(workspace) + h.x, static_cast<cudaStream_t>(stream));
    }
    // otherwise layer by layer, each as redmoe_forward_host
    for (int l = 0; l < n_layers; ++l)
        if ((st = redmoe_forward_host(&layers[l], xs[l], T, outs[l], ids[l], ws[l], workspace, workspace_bytes,
                                      stream)) != REDMOE_OK)
            return st;
    return REDMOE_OK;
}

redmoe_status redmoe_check_timeout(const void* workspace, void* stream) {
    if (!workspace) {  // the allocation-free scratch of this device
        workspace = noalloc_scratch_address();
        if (!workspace) return REDMOE_ERR_CUDA;
    }
    if (!aligned(workspace, 256)) return REDMOE_ERR_WORKSPACE;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (cudaStreamSynchronize(s) != cudaSuccess) return REDMOE_ERR_CUDA;
    Control c;
    if (cudaMemcpy(&c, workspace, sizeof(c), cudaMemcpyDeviceToHost) != cudaSuccess) return REDMOE_ERR_CUDA;
    if (c.err & ERRBIT_TIMEOUT) return REDMOE_ERR_TIMEOUT;
    return (c.err & ERRBIT_STATE) ? REDMOE_ERR_INVALID_ARG : REDMOE_OK;
}

}  // extern "C"
