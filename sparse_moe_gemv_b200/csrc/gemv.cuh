// Bandwidth-bound matrix-vector building blocks (CUDA cores, 16-byte streaming loads).
//
// A weight row of K elements is read as 16-byte chunks (V elements: 4 fp32, 8 bf16 or
// 32 int4); lane L of a warp reads chunks L, L + 32, ... so that one warp instruction
// moves 512 contiguous bytes. The activation vectors the row is dotted with live in
// shared memory in a chunk-interleaved layout (see stage_vec) so that the matching
// activation reads are conflict-free for every weight type. Products accumulate in
// fp32 (packed f32x2 fused multiply-adds, two partial sums per lane).
#pragma once

#include "common.cuh"

namespace redmoe {

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
// weight type W: the P 16-byte pieces of the activations matching weight chunk c sit at
// slots ((c / 32) * P + q) * 32 + c % 32. `coherent` selects L2-only loads for data
// written earlier in this launch by other blocks.
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

// --------------------------------------------------------------- f32x2 math
// Paired fp32 arithmetic (two fp32 operations per instruction), through the CUDA
// intrinsics, which take float2 by value (no type punning of registers).
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) { return __ffma2_rn(a, b, c); }
__device__ __forceinline__ float2 fadd2(float2 a, float2 b) { return __fadd2_rn(a, b); }
__device__ __forceinline__ float2 bf2(uint32_t w) { return make_float2(bf16lo(w), bf16hi(w)); }
__device__ __forceinline__ float2 f2(uint32_t a, uint32_t b) { return make_float2(__uint_as_float(a), __uint_as_float(b)); }
// int4 nibbles n and n+1 of w as floats (nibble - 8): exponent-trick conversion, exact.
__device__ __forceinline__ float2 nib2(uint32_t w, int n) {
    const float2 m = make_float2(__uint_as_float(0x4B000000u | ((w >> (4 * n)) & 15u)),
                                 __uint_as_float(0x4B000000u | ((w >> (4 * n + 4)) & 15u)));
    return fadd2(m, make_float2(-8388616.0f, -8388616.0f));
}

// --------------------------------------------------------------- chunk dot
// Accumulate the dot of one 16-byte weight chunk (iteration ii, lane position L) with its
// staged activations into acc (two partial sums). int4: acc gets sum (nibble - 8) * x; the
// caller applies the group scale.
template <int W, int VT>
__device__ __forceinline__ float2 chunk_dot(const uint4& w, const uint4* xs, int ii, int L, float2 acc) {
    constexpr int P = Pc<W, VT>::P;
    const uint4* b = xs + ii * P * 32 + L;
    if constexpr (W == DT_BF16 && VT == DT_BF16) {
        const uint4 x = b[0];
        acc = ffma2(bf2(w.x), bf2(x.x), acc);
        acc = ffma2(bf2(w.y), bf2(x.y), acc);
        acc = ffma2(bf2(w.z), bf2(x.z), acc);
        acc = ffma2(bf2(w.w), bf2(x.w), acc);
    } else if constexpr (W == DT_BF16 && VT == DT_F32) {
        const uint4 x0 = b[0], x1 = b[32];
        acc = ffma2(bf2(w.x), f2(x0.x, x0.y), acc);
        acc = ffma2(bf2(w.y), f2(x0.z, x0.w), acc);
        acc = ffma2(bf2(w.z), f2(x1.x, x1.y), acc);
        acc = ffma2(bf2(w.w), f2(x1.z, x1.w), acc);
    } else if constexpr (W == DT_F32 && VT == DT_F32) {
        const uint4 x = b[0];
        acc = ffma2(f2(w.x, w.y), f2(x.x, x.y), acc);
        acc = ffma2(f2(w.z, w.w), f2(x.z, x.w), acc);
    } else if constexpr (W == DT_INT4 && VT == DT_BF16) {
        const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const uint4 x = b[q * 32];
            acc = ffma2(nib2(ws[q], 0), bf2(x.x), acc);
            acc = ffma2(nib2(ws[q], 2), bf2(x.y), acc);
            acc = ffma2(nib2(ws[q], 4), bf2(x.z), acc);
            acc = ffma2(nib2(ws[q], 6), bf2(x.w), acc);
        }
    } else if constexpr (W == DT_INT4 && VT == DT_F32) {
        const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int p = 0; p < 8; ++p) {
            const uint4 x = b[p * 32];
            const uint32_t wq = ws[p >> 1];
            const int n0 = (p & 1) * 4;
            acc = ffma2(nib2(wq, n0), f2(x.x, x.y), acc);
            acc = ffma2(nib2(wq, n0 + 2), f2(x.z, x.w), acc);
        }
    }
    return acc;
}

// Scaled accumulation: acc += s * (chunk . x) for int4, acc += chunk . x otherwise.
template <int W, int VT>
__device__ __forceinline__ float2 chunk_dot_s(const uint4& w, float s, const uint4* xs, int ii, int L, float2 acc) {
    if constexpr (W == DT_INT4) {
        const float2 d = chunk_dot<W, VT>(w, xs, ii, L, make_float2(0.f, 0.f));
        return ffma2(make_float2(s, s), d, acc);
    } else {
        (void)s;
        return chunk_dot<W, VT>(w, xs, ii, L, acc);
    }
}

// Weighted accumulation: acc += s * (chunk . x) for every weight type (s carries the
// int4 group scale times a routing weight, or just the routing weight).
template <int W, int VT>
__device__ __forceinline__ float2 chunk_dot_w(const uint4& w, float s, const uint4* xs, int ii, int L, float2 acc) {
    const float2 d = chunk_dot<W, VT>(w, xs, ii, L, make_float2(0.f, 0.f));
    return ffma2(make_float2(s, s), d, acc);
}

// 16-byte chunks per lane loaded before use in a row job (loads in flight per lane)
template <int W> struct RowGroup { static constexpr int G = (W == DT_BF16) ? 8 : 2; };

// Lane-partial dots of one weight row (nch 16-byte chunks) with the T staged vectors
// (vector t at xs + t * xstride uint4s).
template <int W, int VT, int T>
__device__ __forceinline__ void row_dots(const void* row, const uint16_t* srow, int nch, const uint4* xs,
                                         int xstride, int lane, float2 (&acc)[T]) {
    constexpr int G = RowGroup<W>::G;
    const int nit = (nch + 31) >> 5;
    const uint4* r = static_cast<const uint4*>(row);
    for (int g0 = 0; g0 < nit; g0 += G) {
        uint4 wc[G];
        float sc[G];
#pragma unroll
        for (int i = 0; i < G; ++i) {
            const int c = (g0 + i) * 32 + lane;
            const bool ok = (g0 + i < nit) && c < nch;
            wc[i] = ok ? ld_stream(r + c) : make_uint4(0u, 0u, 0u, 0u);
            sc[i] = 0.0f;
            if constexpr (W == DT_INT4) sc[i] = ok ? bf16f(ld_stream_u16(srow + c)) : 0.0f;
        }
#pragma unroll
        for (int i = 0; i < G; ++i) {
            if (g0 + i < nit) {
#pragma unroll
                for (int t = 0; t < T; ++t)
                    acc[t] = chunk_dot_s<W, VT>(wc[i], sc[i], xs + t * xstride, g0 + i, lane, acc[t]);
            }
        }
    }
}

// Gate and up rows of one expert row index together (both K = H).
template <int W, int VT, int T>
__device__ __forceinline__ void pair_dots(const void* grow, const uint16_t* gs, const void* urow, const uint16_t* us,
                                          int nch, const uint4* xs, int xstride, int lane, float2 (&a)[T],
                                          float2 (&u)[T]) {
    constexpr int G = RowGroup<W>::G;
    const int nit = (nch + 31) >> 5;
    const uint4* gr = static_cast<const uint4*>(grow);
    const uint4* ur = static_cast<const uint4*>(urow);
    for (int g0 = 0; g0 < nit; g0 += G) {
        uint4 wg[G], wu[G];
        float sg[G], su[G];
#pragma unroll
        for (int i = 0; i < G; ++i) {
            const int c = (g0 + i) * 32 + lane;
            const bool ok = (g0 + i < nit) && c < nch;
            wg[i] = ok ? ld_stream(gr + c) : make_uint4(0u, 0u, 0u, 0u);
            wu[i] = ok ? ld_stream(ur + c) : make_uint4(0u, 0u, 0u, 0u);
            sg[i] = su[i] = 0.0f;
            if constexpr (W == DT_INT4) {
                sg[i] = ok ? bf16f(ld_stream_u16(gs + c)) : 0.0f;
                su[i] = ok ? bf16f(ld_stream_u16(us + c)) : 0.0f;
            }
        }
#pragma unroll
        for (int i = 0; i < G; ++i) {
            if (g0 + i < nit) {
#pragma unroll
                for (int t = 0; t < T; ++t) {
                    a[t] = chunk_dot_s<W, VT>(wg[i], sg[i], xs + t * xstride, g0 + i, lane, a[t]);
                    u[t] = chunk_dot_s<W, VT>(wu[i], su[i], xs + t * xstride, g0 + i, lane, u[t]);
                }
            }
        }
    }
}

__device__ __forceinline__ float silu_mul(float a, float u) { return a / (1.0f + expf(-a)) * u; }

}  // namespace redmoe
