// Parameters of the grouped tensor-core GEMM kernels (shared by ggemm.cu and prefill.cu).
#pragma once

#include <cuda.h>
#include <stdint.h>

#include "common.cuh"

namespace redmoe {

enum : int { GM_ROUTER = 0, GM_SWIGLU = 1, GM_SCATTER = 2 };

struct GemmParams {
    CUtensorMap tmA;    // A rows [rows, K]
    CUtensorMap tmA2;   // SWIGLU: the shared expert's A rows (x itself, [T, K])
    CUtensorMap tmB0;   // routed B rows (SWIGLU: gate), or the router weights
    CUtensorMap tmB1;   // routed up rows (SWIGLU only)
    CUtensorMap tmS0;   // shared-expert B rows (SWIGLU: gate)
    CUtensorMap tmS1;   // shared-expert up rows (SWIGLU only)
    int E;              // routed groups; group E is the shared expert (grouped modes)
    int T, k;           // tokens, experts per token
    int N;              // output columns of the whole GEMM (router: E; SWIGLU: I; SCATTER: H)
    int Nb;             // rows of one routed group's B block (SWIGLU: I; SCATTER: H)
    int n_tiles;        // tiles along N
    int num_kb;         // K / 64
    const int* offsets; // [E + 1] group starts in the grouped row space (grouped modes)
    const int* tiles;   // [E + 2] prefix of m-tiles per group (grouped modes)
    float* out_f32;     // ROUTER: logits [T, N]; SCATTER: out [T, N]
    const float* bias;  // ROUTER: per-expert offset or null
    uint16_t* out_bf16; // SWIGLU: h [rows, N] bf16
    const int* perm;    // SCATTER: grouped row -> t*k + j
    const float* topk_w;// SCATTER: [T * k]
    const float* sgate; // SCATTER: [T]
    float* zero_out;    // ROUTER: zeroed by the epilogue warps before their tiles (or null)
    uint64_t zero_f4;   // ROUTER: float4 count of zero_out
    Control* ctl;
    uint64_t timeout_ns;
};

}  // namespace redmoe
