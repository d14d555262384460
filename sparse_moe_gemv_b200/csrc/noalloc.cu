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
// be issued.
//
// The array starts with the same 256-byte control block as a workspace. Before each
// launch a call clears the two grid-barrier counters (an asynchronous 8-byte memset, no
// allocation), so that a launch that failed part-way cannot leave them dirty. It does
// not clear the error word: a bounded in-kernel wait that gave up stays recorded until
// the caller reads it with redmoe_check_timeout(NULL, stream) and clears it with
// redmoe_workspace_init(NULL, 0, stream).
#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace redmoe {

constexpr size_t NOALLOC_SCRATCH_BYTES = size_t(1) << 20;

namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[NOALLOC_SCRATCH_BYTES];

constexpr int MAX_DEVICES = 64;

}  // namespace

// Device address of g_noalloc_scratch on the current device, looked up once per device.
void* noalloc_scratch_address() {
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

}  // namespace redmoe

using namespace redmoe;

extern "C" redmoe_status redmoe_forward_noalloc(const redmoe_layer* L, const void* x, int32_t T, float* out,
                                                int32_t* topk_ids, float* topk_w, void* stream) {
    redmoe_status st = check_layer(L);
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
    void* ws = noalloc_scratch_address();
    if (!ws) return REDMOE_ERR_CUDA;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    static_assert(offsetof(Control, err) == 8, "the barrier counters are the first 8 bytes");
    if (cudaMemsetAsync(ws, 0, offsetof(Control, err), s) != cudaSuccess) return REDMOE_ERR_CUDA;
    const DecLayer d = dec_layer(L, x, out, topk_ids, topk_w);
    return launch_decode(L, &d, 1, T, ws, s, nullptr);
}
