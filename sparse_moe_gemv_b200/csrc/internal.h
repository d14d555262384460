// Declarations shared between the .cu files of libredmoe (not part of the C ABI).
#pragma once

#include <vector>

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/redmoe.h"

namespace redmoe {

constexpr int DECODE_MAX_T = 4;        // decode kernel handles 1..4 token rows
constexpr int MAX_TOPK = 32;
constexpr int MAX_EXPERTS = 1024;
constexpr int MAX_STACK = 64;          // layers per persistent decode launch
constexpr uint64_t BARRIER_TIMEOUT_NS = 1000000000ull;  // 1 s
constexpr int ROUTE_MAX_BLOCKS = 256;  // blocks of the batched routing kernel, at most

inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// Opt-in cache-aware routing: the selection ranks z + lambda * (max z - min z) * cached[e];
// cached == nullptr is plain routing.
struct CacheBias {
    const uint8_t* cached;
    float lambda;
};

// One layer as the decode kernel sees it (pointers into caller memory).
struct DecLayer {
    const void* router_w;
    const float* router_bias;
    const void* shared_gate_w;
    const void* w_gate;
    const void* w_up;
    const void* w_down;
    const uint16_t* s_gate;
    const uint16_t* s_up;
    const uint16_t* s_down;
    const void* sh_gate;
    const void* sh_up;
    const void* sh_down;
    const uint16_t* sh_s_gate;
    const uint16_t* sh_s_up;
    const uint16_t* sh_s_down;
    const void* x;
    float* out;
    int32_t* ids;
    float* w;
    // One-row kernel only: routing taken from these arrays instead of computed (NULL:
    // computed), and routed expert e read from stack index slot_of[e] (NULL: index e).
    const int32_t* given_ids;
    const float* given_w;
    const int32_t* slot_of;
};

// The decode kernel's view of one redmoe_layer called on (x, out, ids, w).
DecLayer dec_layer(const redmoe_layer* L, const void* x, float* out, int32_t* ids, float* w);
// The same calls restricted to rows r0 .. of x, out, ids and w.
std::vector<DecLayer> dec_rows(const redmoe_layer* sh, const DecLayer* layers, int n_layers, int r0);
// Decode sizes run as rows 0-1 on the few-row kernel plus the rest on the one- or few-row
// kernel (T = 3, 4 on layers both take).
bool decode_split_ok(const redmoe_layer* sh, int T);

// Layer validation shared by every entry point (shape, dtype combination, pointers).
redmoe_status check_layer(const redmoe_layer* L);

// Device address of the allocation-free scratch array on the current device (looked up
// once per device); NULL on a CUDA error.
void* noalloc_scratch_address();

// Workspace carve-up of the decode path (byte offsets from the workspace base).
struct DecodeWs {
    size_t logits, sgate, hsh, hrt, total;
};
DecodeWs decode_ws_layout(int T, int E, int k, int I, int Is);

// The one-row kernel (T = 1, bf16 or int4 experts of the Qwen3-Next width): which layers
// it takes, and its launch over n_layers layers.
bool decode1_shape_ok(const redmoe_layer* sh);
// T = 1 layers whose x (layers[l].x) is the device mapping of pinned host memory: block 0
// copies each layer's x into xstage (device, 2 H bytes, 16-byte aligned) at the layer's
// start and every block reads it there.
redmoe_status launch_decode1_host_x(const redmoe_layer* sh, const DecLayer* layers, int n_layers, void* ws,
                                    void* xstage, cudaStream_t stream);
redmoe_status launch_decode1(const redmoe_layer* sh, const DecLayer* layers, int n_layers, void* ws,
                             cudaStream_t stream, int* launches, CacheBias cb);

// The few-row kernel (T = 2, 3; bf16 or int4 experts of the Qwen3-Next width).
bool decodefr_shape_ok(const redmoe_layer* sh, int T);
redmoe_status launch_decodefr(const redmoe_layer* sh, const DecLayer* layers, int n_layers, int T, void* ws,
                              cudaStream_t stream, int* launches, CacheBias cb);
// The same with every layer's x (layers[l].x, T rows) the device mapping of pinned host
// memory: blocks 0 .. 4T-1 copy it into xstage (device, T * 2 H bytes, 16-byte aligned)
// at each layer's start and every x read comes from there.
redmoe_status launch_decodefr_host_x(const redmoe_layer* sh, const DecLayer* layers, int n_layers, int T, void* ws,
                                     void* xstage, cudaStream_t stream);

// Launch the persistent decode kernel over n_layers layers (1..MAX_STACK).
redmoe_status launch_decode(const redmoe_layer* shape, const DecLayer* layers, int n_layers, int T,
                            void* workspace, cudaStream_t stream, int* launches, CacheBias cb = CacheBias{nullptr, 0.0f});

// Workspace carve-up of the batched (grouped-GEMM) path (byte offsets from the base).
struct BatchLayout {
    size_t logits, sgate, counts, offsets, perm, tiles, bhist, xg, h, total;
};
BatchLayout batch_layout(int T, int E, int k, int H, int I);
bool batch_shape_ok(const redmoe_layer* L);
redmoe_status launch_batched(const redmoe_layer* L, const void* x, int T, float* out, int32_t* ids, float* w,
                             void* ws, const redmoe_route_debug* dbg, cudaStream_t s, int* launches,
                             CacheBias cb = CacheBias{nullptr, 0.0f});

// Device attributes cached per device.
struct DevInfo {
    int sm_count;
    int max_smem_optin;
};
bool get_dev_info(DevInfo* out);

}  // namespace redmoe
