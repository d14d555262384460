// redmoe_forward_noalloc: the decode-size layer forward with its scratch memory in a
// fixed array that is part of the library image, for callers that cannot allocate device
// memory.
//
// Who needs this: code that runs where cudaMalloc is not allowed or not acceptable, e.g.
// inside a CUDA stream capture in a strict capture mode (an allocation call there breaks
// the capture), a latency-critical loop that must never wait on the allocator or risk an
// out-of-memory failure in the middle of a step, or a plug-in hosted by a framework that
// owns the whole device memory budget and gives the plug-in none of it. Such callers can
// still hand over inputs and outputs, but not a workspace.
//
// How: the workspace that redmoe_forward takes from the caller lives here in a
// file-scope __device__ array of NOALLOC_SCRATCH_BYTES (1 MiB). Every GPU that loads the
// library keeps those bytes until the process exits. Host code cannot use the array's
// name as a device address, so the first call on each device looks the address up with
// cudaGetSymbolAddress while that device is current and caches it; make that first call
// outside any stream capture. Every call on a device shares the one array: calls that
// may overlap on the GPU (different streams without ordering) race on it and must not
// be issued. Each call clears the array's 256-byte control block with an asynchronous
// memset (no allocation) before the kernel, because the kernel's grid barrier expects it
// at zero.
#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace redmoe {

constexpr size_t NOALLOC_SCRATCH_BYTES = size_t(1) << 20;

namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[NOALLOC_SCRATCH_BYTES];

constexpr int MAX_DEVICES = 64;

// Device address of g_noalloc_scratch on the current device, looked up once per device.
void* scratch_address() {
    static std::mutex mu;
    static void* addr[MAX_DEVICES] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= MAX_DEVICES) return nullptr;
    std::lock_guard<std::mutex> lock(mu);
    if (!addr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess) return nullptr;
        addr[dev] = p;
    }
    return addr[dev];
}

}  // namespace

redmoe_status check_layer_for_noalloc(const redmoe_layer* L);

}  // namespace redmoe

using namespace redmoe;

extern "C" redmoe_status redmoe_forward_noalloc(const redmoe_layer* L, const void* x, int32_t T, float* out,
                                                int32_t* topk_ids, float* topk_w, void* stream) {
    redmoe_status st = check_layer_for_noalloc(L);
    if (st != REDMOE_OK) return st;
    if (T < 0) return REDMOE_ERR_INVALID_ARG;
    if (T == 0) return REDMOE_OK;
    if (!x || !out || !topk_ids || !topk_w) return REDMOE_ERR_INVALID_ARG;
    const uintptr_t ax = reinterpret_cast<uintptr_t>(x), ao = reinterpret_cast<uintptr_t>(out);
    if (ax % 16 || ao % 16 || reinterpret_cast<uintptr_t>(topk_ids) % 4 || reinterpret_cast<uintptr_t>(topk_w) % 4)
        return REDMOE_ERR_INVALID_ARG;
    if (T > DECODE_MAX_T) return REDMOE_ERR_UNSUPPORTED;
    const DecodeWs need = decode_ws_layout(T, L->n_experts, L->top_k, L->inter, L->shared_inter);
    if (need.total > NOALLOC_SCRATCH_BYTES) return REDMOE_ERR_WORKSPACE;
    void* ws = scratch_address();
    if (!ws) return REDMOE_ERR_CUDA;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (cudaMemsetAsync(ws, 0, 256, s) != cudaSuccess) return REDMOE_ERR_CUDA;
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
    d.ids = topk_ids;
    d.w = topk_w;
    return launch_decode(L, &d, 1, T, ws, s, nullptr);
}
