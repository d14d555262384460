// Bandwidth-bound matrix-vector building blocks (CUDA cores, 16-byte streaming loads).
//
// A weight row of K elements is read as 16-byte chunks (V elements: 4 fp32, 8 bf16 or
// 32 int4); lane L of a warp reads chunks L, L + 32, ... so that one warp instruction
// moves 512 contiguous bytes. The activation vectors the row is dotted with live in
// shared memory in a chunk-interleaved layout (see stage_vec) so that the matching
// activation reads are conflict-free for every weight type.
#pragma once

#include "common.cuh"

namespace redmoe {

constexpr int GEMV_G = 8;   // 16-byte chunks per lane per row group (loads in flight)

template <int W> struct Wv;
template <> struct Wv<DT_F32> { static constexpr int V = 4; };
template <> struct Wv<DT_BF16> { static constexpr int V = 8; };
template <> struct Wv<DT_INT4> { static constexpr int V = 32; };

template <int VT> struct Vb { static constexpr int bytes = (VT == DT_BF16) ? 2 : 4; };

template <int W, int VT> struct Pc { static constexpr int P = Wv<W>::V * Vb<VT>::bytes / 16; };

__host__ __device__ constexpr int wv(int w) { return w == DT_F32 ? 4 : (w == DT_BF16 ? 8 : 32); }
__host__ __device__ constexpr int vbytes(int vt) { return vt == DT_BF16 ? 2 : 4; }
// Bytes of one weight row of K elements (int4: packed bytes only).
__host__ __device__ constexpr long row_bytes(int w, int K) {
    return w == DT_F32 ? 4L * K : (w == DT_BF16 ? 2L * K : K / 2);
}
// Staged-activation bytes for a K-vector read against weight type w.
__host__ __device__ inline int staged_bytes(int K, int w, int vt) {
    const int nch = K / wv(w);
    const int P = wv(w) * vbytes(vt) / 16;
    return ((nch + 31) / 32) * 32 * P * 16;
}

// ------------------------------------------------------------------ staging
// Copy a K-vector (bf16 or f32 in global memory) into the chunk-interleaved layout for
// weight type W. `coherent` selects L2-only loads for data written earlier in this
// launch by other blocks.
template <int W, int VT>
__device__ void stage_vec(uint4* dst, const void* src, int K, bool coherent) {
    constexpr int V = Wv<W>::V;
    constexpr int P = Pc<W, VT>::P;
    constexpr int PER = 16 / Vb<VT>::bytes;  // elements per 16-byte piece
    const int nch = K / V;
    const int nslots = ((nch + 31) / 32) * 32 * P;
    for (int s = threadIdx.x; s < nslots; s += blockDim.x) {
        const int L = s & 31;
        const int q = (s >> 5) % P;
        const int ii = (s >> 5) / P;
        const int c = ii * 32 + L;
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (c < nch) {
            const uint4* p = reinterpret_cast<const uint4*>(static_cast<const char*>(src) +
                                                             size_t(c * V + q * PER) * Vb<VT>::bytes);
            v = coherent ? __ldcg(p) : *p;
        }
        dst[s] = v;
    }
}

// --------------------------------------------------------------- chunk dot
// Dot of one 16-byte weight chunk (iteration ii, lane position L) with its staged
// activations. int4: returns sum (nibble - 8) * x; the caller applies the group scale.
__device__ __forceinline__ float nib(uint32_t w, int n) {
    return __uint_as_float(0x4B000000u | ((w >> (4 * n)) & 15u)) - 8388616.0f;
}

template <int W, int VT>
__device__ __forceinline__ float chunk_dot(const uint4& w, const uint4* xs, int ii, int L) {
    constexpr int P = Pc<W, VT>::P;
    const uint4* b = xs + ii * P * 32 + L;
    float acc = 0.0f;
    if constexpr (W == DT_BF16 && VT == DT_BF16) {
        const uint4 x = b[0];
        acc = fmaf(bf16lo(w.x), bf16lo(x.x), acc); acc = fmaf(bf16hi(w.x), bf16hi(x.x), acc);
        acc = fmaf(bf16lo(w.y), bf16lo(x.y), acc); acc = fmaf(bf16hi(w.y), bf16hi(x.y), acc);
        acc = fmaf(bf16lo(w.z), bf16lo(x.z), acc); acc = fmaf(bf16hi(w.z), bf16hi(x.z), acc);
        acc = fmaf(bf16lo(w.w), bf16lo(x.w), acc); acc = fmaf(bf16hi(w.w), bf16hi(x.w), acc);
    } else if constexpr (W == DT_BF16 && VT == DT_F32) {
        const uint4 x0 = b[0], x1 = b[32];
        acc = fmaf(bf16lo(w.x), __uint_as_float(x0.x), acc); acc = fmaf(bf16hi(w.x), __uint_as_float(x0.y), acc);
        acc = fmaf(bf16lo(w.y), __uint_as_float(x0.z), acc); acc = fmaf(bf16hi(w.y), __uint_as_float(x0.w), acc);
        acc = fmaf(bf16lo(w.z), __uint_as_float(x1.x), acc); acc = fmaf(bf16hi(w.z), __uint_as_float(x1.y), acc);
        acc = fmaf(bf16lo(w.w), __uint_as_float(x1.z), acc); acc = fmaf(bf16hi(w.w), __uint_as_float(x1.w), acc);
    } else if constexpr (W == DT_F32 && VT == DT_F32) {
        const uint4 x = b[0];
        acc = fmaf(__uint_as_float(w.x), __uint_as_float(x.x), acc);
        acc = fmaf(__uint_as_float(w.y), __uint_as_float(x.y), acc);
        acc = fmaf(__uint_as_float(w.z), __uint_as_float(x.z), acc);
        acc = fmaf(__uint_as_float(w.w), __uint_as_float(x.w), acc);
    } else if constexpr (W == DT_INT4 && VT == DT_BF16) {
        const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const uint4 x = b[q * 32];
            const uint32_t xw[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
            for (int m = 0; m < 4; ++m) {
                acc = fmaf(nib(ws[q], 2 * m), bf16lo(xw[m]), acc);
                acc = fmaf(nib(ws[q], 2 * m + 1), bf16hi(xw[m]), acc);
            }
        }
    } else if constexpr (W == DT_INT4 && VT == DT_F32) {
        const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int p = 0; p < 8; ++p) {
            const uint4 x = b[p * 32];
            const uint32_t wq = ws[p >> 1];
            const int n0 = (p & 1) * 4;
            acc = fmaf(nib(wq, n0 + 0), __uint_as_float(x.x), acc);
            acc = fmaf(nib(wq, n0 + 1), __uint_as_float(x.y), acc);
            acc = fmaf(nib(wq, n0 + 2), __uint_as_float(x.z), acc);
            acc = fmaf(nib(wq, n0 + 3), __uint_as_float(x.w), acc);
        }
    }
    return acc;
}

// Lane-partial dots of one weight row (K elements, type W) with T staged vectors
// (vector t at xs + t * xstride uint4s). Row groups of G chunks per lane are loaded
// before use so that each lane has G 16-byte loads in flight.
template <int W, int VT, int NT>
__device__ __forceinline__ void row_dots(const void* row, const uint16_t* srow, int K, const uint4* xs,
                                         int xstride, int T, int lane, float (&acc)[NT]) {
    const int nch = K / Wv<W>::V;
    const int nit = (nch + 31) / 32;
    const uint4* r = static_cast<const uint4*>(row);
    for (int g0 = 0; g0 < nit; g0 += GEMV_G) {
        uint4 wc[GEMV_G];
        float sc[GEMV_G];
#pragma unroll
        for (int i = 0; i < GEMV_G; ++i) {
            const int c = (g0 + i) * 32 + lane;
            const bool ok = (g0 + i < nit) && c < nch;
            wc[i] = ok ? ld_stream(r + c) : make_uint4(0u, 0u, 0u, 0u);
            if constexpr (W == DT_INT4) sc[i] = ok ? bf16f(ld_stream_u16(srow + c)) : 0.0f;
        }
#pragma unroll
        for (int i = 0; i < GEMV_G; ++i) {
            if (g0 + i < nit) {
#pragma unroll
                for (int t = 0; t < NT; ++t) {
                    if (t < T) {
                        float d = chunk_dot<W, VT>(wc[i], xs + t * xstride, g0 + i, lane);
                        if constexpr (W == DT_INT4) d *= sc[i];
                        acc[t] += d;
                    }
                }
            }
        }
    }
}

// Gate and up rows of one expert row index together (both K = H), then SwiGLU.
template <int W, int VT, int NT>
__device__ __forceinline__ void pair_dots(const void* grow, const uint16_t* gs, const void* urow,
                                          const uint16_t* us, int K, const uint4* xs, int xstride,
                                          int T, int lane, float (&a)[NT], float (&u)[NT]) {
    const int nch = K / Wv<W>::V;
    const int nit = (nch + 31) / 32;
    const uint4* gr = static_cast<const uint4*>(grow);
    const uint4* ur = static_cast<const uint4*>(urow);
    for (int g0 = 0; g0 < nit; g0 += GEMV_G) {
        uint4 wg[GEMV_G], wu[GEMV_G];
        float sg[GEMV_G], su[GEMV_G];
#pragma unroll
        for (int i = 0; i < GEMV_G; ++i) {
            const int c = (g0 + i) * 32 + lane;
            const bool ok = (g0 + i < nit) && c < nch;
            wg[i] = ok ? ld_stream(gr + c) : make_uint4(0u, 0u, 0u, 0u);
            wu[i] = ok ? ld_stream(ur + c) : make_uint4(0u, 0u, 0u, 0u);
            if constexpr (W == DT_INT4) {
                sg[i] = ok ? bf16f(ld_stream_u16(gs + c)) : 0.0f;
                su[i] = ok ? bf16f(ld_stream_u16(us + c)) : 0.0f;
            }
        }
#pragma unroll
        for (int i = 0; i < GEMV_G; ++i) {
            if (g0 + i < nit) {
#pragma unroll
                for (int t = 0; t < NT; ++t) {
                    if (t < T) {
                        float da = chunk_dot<W, VT>(wg[i], xs + t * xstride, g0 + i, lane);
                        float du = chunk_dot<W, VT>(wu[i], xs + t * xstride, g0 + i, lane);
                        if constexpr (W == DT_INT4) { da *= sg[i]; du *= su[i]; }
                        a[t] += da;
                        u[t] += du;
                    }
                }
            }
        }
    }
}

__device__ __forceinline__ float silu_mul(float a, float u) { return a / (1.0f + expf(-a)) * u; }

}  // namespace redmoe
