// Row and dot helpers of the register-resident decode kernels (decode1.cu for one token
// row, decode_fr.cu for two to four): a lane holds its slice of x in registers in the
// layout its 16-byte weight chunks need, loads weight rows with 16-byte streaming loads
// and dots them without going through shared memory.
#pragma once

#include "common.cuh"
#include "gemv.cuh"

namespace redmoe {
namespace {

constexpr int D1_THREADS = 256;
constexpr int D1_WARPS = D1_THREADS / 32;
constexpr int D1_XPL = 64;        // x elements per lane (H = 2048 at most)
constexpr int D1_HPL = 16;        // h elements per lane (I = 512)
constexpr int D1_MAXK = 11;       // routed experts per token (plus the shared one)
constexpr int D1_MAXE = 512;      // experts (16 router logits per lane in the top-k)
constexpr int D1_RB_MAX = 16;     // output rows per block
constexpr int D1_G = 2;           // routed gate/up row pairs in flight per warp (bf16)
constexpr int D1_GQ = 5;          // the same for int4 / int2 (all of a warp's pairs at Qwen3-Next size)

__host__ __device__ constexpr int a16(int x) { return (x + 15) & ~15; }

// Elements of one 16-byte weight chunk.
template <int W> struct ChunkElems { static constexpr int n = 8; };
template <> struct ChunkElems<DT_INT4> { static constexpr int n = 32; };
template <> struct ChunkElems<DT_INT2> { static constexpr int n = 64; };

// x slice of a lane as fp32, in the layout a weight type's 16-byte chunks need:
//   bf16 rows: chunk c = lane + 32 j (j < H / 256) covers elements 8c .. 8c + 7 -> xf[8j + m]
//   int4 rows: chunk c = lane + 32 j (j < H / 1024) covers elements 32c .. 32c + 31 -> xf[32j + m]
//   int2 rows: chunk c = lane (H = 2048) covers elements 64c .. 64c + 63 -> xf[m]
// SM: x is a copy in shared memory (plain loads) rather than in global memory.
template <int W, bool SM = false>
__device__ __forceinline__ void load_x(const uint16_t* x, int H, int lane, float (&xf)[D1_XPL]) {
    constexpr int PER = ChunkElems<W>::n;  // elements per chunk
    constexpr int NJ = D1_XPL / PER;
    uint4 v[D1_XPL / 8];
#pragma unroll
    for (int j = 0; j < NJ; ++j) {
        const int c = lane + 32 * j;
#pragma unroll
        for (int q = 0; q < PER / 8; ++q) {
            const bool ok = (c * PER + q * 8) < H;
            const uint4* px = reinterpret_cast<const uint4*>(x + size_t(c) * PER + q * 8);
            v[j * (PER / 8) + q] = ok ? (SM ? *px : __ldg(px)) : make_uint4(0u, 0u, 0u, 0u);
        }
    }
#pragma unroll
    for (int i = 0; i < D1_XPL / 8; ++i) {
        const uint32_t w[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            xf[8 * i + 2 * q] = bf16lo(w[q]);
            xf[8 * i + 2 * q + 1] = bf16hi(w[q]);
        }
    }
}

// One bf16 row of H elements, in the bf16 chunk layout: NJ = H / 256 16-byte loads per lane.
struct RowBF {
    uint4 w[D1_XPL / 8];
};
__device__ __forceinline__ void ld_row_bf(RowBF& r, const void* row, int H, int lane) {
    const uint4* p = static_cast<const uint4*>(row);
#pragma unroll
    for (int j = 0; j < D1_XPL / 8; ++j) {
        const int c = lane + 32 * j;
        r.w[j] = (c * 8 < H) ? ld_stream(p + c) : make_uint4(0u, 0u, 0u, 0u);
    }
}
__device__ __forceinline__ float2 dot_row_bf(const RowBF& r, const float (&xf)[D1_XPL]) {
    float2 a = make_float2(0.f, 0.f), b = make_float2(0.f, 0.f);
#pragma unroll
    for (int j = 0; j < D1_XPL / 8; ++j) {
        a = ffma2(bf2(r.w[j].x), make_float2(xf[8 * j + 0], xf[8 * j + 1]), a);
        b = ffma2(bf2(r.w[j].y), make_float2(xf[8 * j + 2], xf[8 * j + 3]), b);
        a = ffma2(bf2(r.w[j].z), make_float2(xf[8 * j + 4], xf[8 * j + 5]), a);
        b = ffma2(bf2(r.w[j].w), make_float2(xf[8 * j + 6], xf[8 * j + 7]), b);
    }
    return fadd2(a, b);
}

// Packed codes to fp32 with one byte permute per element: a code c in the low bits of
// byte b of `v` (the other bits zero) becomes the float 2^23 + c (bytes {c, 0, 0, 0x4B});
// subtracting 2^23 + bias then gives c - bias exactly.
__device__ __forceinline__ float code_f(uint32_t v, uint32_t b) {
    return __uint_as_float(__byte_perm(v, 0x4B000000u, 0x7650u | b));
}

// 8 int4 elements (one word: element n in bits 4n .. 4n+3) dotted with xv[0..8)
__device__ __forceinline__ float2 dot8_q4(uint32_t w, const float* xv, float2 a) {
    const uint32_t lo = w & 0x0F0F0F0Fu;         // elements 0, 2, 4, 6 in bytes 0..3
    const uint32_t hi = (w >> 4) & 0x0F0F0F0Fu;  // elements 1, 3, 5, 7
    const float2 off = make_float2(-8388616.0f, -8388616.0f);  // -(2^23 + 8)
#pragma unroll
    for (uint32_t b = 0; b < 4; ++b)
        a = ffma2(fadd2(make_float2(code_f(lo, b), code_f(hi, b)), off), make_float2(xv[2 * b], xv[2 * b + 1]), a);
    return a;
}

// 16 int2 elements (one word: element n in bits 2n, 2n+1) dotted with xv[0..16)
__device__ __forceinline__ float2 dot16_q2(uint32_t w, const float* xv) {
    const uint32_t c0 = w & 0x03030303u, c1 = (w >> 2) & 0x03030303u;  // elements 4b, 4b+1
    const uint32_t c2 = (w >> 4) & 0x03030303u, c3 = (w >> 6) & 0x03030303u;  // 4b+2, 4b+3
    const float2 off = make_float2(-8388610.0f, -8388610.0f);  // -(2^23 + 2)
    float2 a = make_float2(0.f, 0.f), b2 = make_float2(0.f, 0.f);
#pragma unroll
    for (uint32_t b = 0; b < 4; ++b) {
        a = ffma2(fadd2(make_float2(code_f(c0, b), code_f(c1, b)), off), make_float2(xv[4 * b], xv[4 * b + 1]), a);
        b2 = ffma2(fadd2(make_float2(code_f(c2, b), code_f(c3, b)), off), make_float2(xv[4 * b + 2], xv[4 * b + 3]), b2);
    }
    return fadd2(a, b2);
}

// One int4 group-32 row of H elements, in the int4 chunk layout: H / 1024 chunks of 32
// elements (16 bytes, one scale group) per lane.
struct RowQ4 {
    uint4 w[D1_XPL / 32];
    uint16_t s[D1_XPL / 32];
};
__device__ __forceinline__ void ld_row_q4(RowQ4& r, const void* row, const uint16_t* sc, int H, int lane) {
    const uint4* p = static_cast<const uint4*>(row);
#pragma unroll
    for (int j = 0; j < D1_XPL / 32; ++j) {
        const int c = lane + 32 * j;
        const bool ok = c * 32 < H;
        r.w[j] = ok ? ld_stream(p + c) : make_uint4(0u, 0u, 0u, 0u);
        r.s[j] = ok ? ld_stream_u16(sc + c) : uint16_t(0);
    }
}
__device__ __forceinline__ float2 dot_row_q4(const RowQ4& r, const float (&xf)[D1_XPL]) {
    float2 acc = make_float2(0.f, 0.f);
#pragma unroll
    for (int j = 0; j < D1_XPL / 32; ++j) {
        const uint32_t w[4] = {r.w[j].x, r.w[j].y, r.w[j].z, r.w[j].w};
        float2 a = make_float2(0.f, 0.f), b = make_float2(0.f, 0.f);
        a = dot8_q4(w[0], xf + 32 * j, a);
        b = dot8_q4(w[1], xf + 32 * j + 8, b);
        a = dot8_q4(w[2], xf + 32 * j + 16, a);
        b = dot8_q4(w[3], xf + 32 * j + 24, b);
        const float s = bf16f(r.s[j]);
        acc = ffma2(make_float2(s, s), fadd2(a, b), acc);
    }
    return acc;
}

// One int2 group-32 row of H elements, in the int2 chunk layout: one chunk of 64
// elements (16 bytes, two scale groups) per lane.
struct RowQ2 {
    uint4 w[D1_XPL / 64];
    uint32_t s[D1_XPL / 64];  // the chunk's two bf16 scales
};
__device__ __forceinline__ void ld_row_q2(RowQ2& r, const void* row, const uint16_t* sc, int H, int lane) {
    const uint4* p = static_cast<const uint4*>(row);
#pragma unroll
    for (int j = 0; j < D1_XPL / 64; ++j) {
        const int c = lane + 32 * j;
        const bool ok = c * 64 < H;
        r.w[j] = ok ? ld_stream(p + c) : make_uint4(0u, 0u, 0u, 0u);
        r.s[j] = ok ? ld_stream_u32(sc + 2 * c) : 0u;
    }
}
__device__ __forceinline__ float2 dot_row_q2(const RowQ2& r, const float (&xf)[D1_XPL]) {
    float2 acc = make_float2(0.f, 0.f);
#pragma unroll
    for (int j = 0; j < D1_XPL / 64; ++j) {
        const float* xv = xf + 64 * j;
        const float2 g0 = fadd2(dot16_q2(r.w[j].x, xv), dot16_q2(r.w[j].y, xv + 16));
        const float2 g1 = fadd2(dot16_q2(r.w[j].z, xv + 32), dot16_q2(r.w[j].w, xv + 48));
        const float s0 = bf16lo(r.s[j]), s1 = bf16hi(r.s[j]);
        acc = ffma2(make_float2(s0, s0), g0, acc);
        acc = ffma2(make_float2(s1, s1), g1, acc);
    }
    return acc;
}

// Word of h element i (I = 512) in an h row as the down projection reads it. There lane l
// holds the 16 elements its chunk of a down row covers: l*16 .. l*16+15 for int4 and int2
// rows (one 8- or 4-byte load), and l*8 .. l*8+7 with 256+l*8 .. 256+l*8+7 for bf16 rows
// (two 16-byte loads 512 bytes apart, each conflict-free over the warp). Element m of
// lane l sits at word 128*(m/4) + 4*l + m%4, so that the lane's four 16-byte loads of h
// are conflict-free (in shared memory) and coalesced (in global memory) too.
template <int WT>
__device__ __forceinline__ int hpos(int i) {
    int l, m;
    if constexpr (WT == DT_BF16) {
        l = (i & 255) >> 3;
        m = (i & 7) | ((i >> 8) << 3);
    } else {
        l = i >> 4;
        m = i & 15;
    }
    return 128 * (m >> 2) + 4 * l + (m & 3);
}

template <int W> struct RowOf { using type = RowBF; };
template <> struct RowOf<DT_INT4> { using type = RowQ4; };
template <> struct RowOf<DT_INT2> { using type = RowQ2; };

template <int W>
__device__ __forceinline__ void ld_row(typename RowOf<W>::type& r, const void* row, const uint16_t* sc, int H, int lane) {
    if constexpr (W == DT_INT4) ld_row_q4(r, row, sc, H, lane);
    else if constexpr (W == DT_INT2) ld_row_q2(r, row, sc, H, lane);
    else { (void)sc; ld_row_bf(r, row, H, lane); }
}
template <int W>
__device__ __forceinline__ float2 dot_row(const typename RowOf<W>::type& r, const float (&xf)[D1_XPL]) {
    if constexpr (W == DT_INT4) return dot_row_q4(r, xf);
    else if constexpr (W == DT_INT2) return dot_row_q2(r, xf);
    else return dot_row_bf(r, xf);
}

// bytes of one stored row of K elements (codes only) and of its group scales
__host__ __device__ constexpr int d1_row_bytes(int wt, int K) {
    return wt == DT_INT4 ? K / 2 : (wt == DT_INT2 ? K / 4 : 2 * K);
}
__host__ __device__ constexpr int d1_scale_bytes(int wt, int K) { return wt == DT_BF16 ? 0 : K / 16; }


// x rows as packed bf16 pairs in the layout of weight type W: word m of row t is
// elements 2m, 2m + 1 of the lane's slice (bf16: chunk c = lane + 32 j covers elements
// 8c .. 8c + 7 -> words 4j .. 4j + 3; int4: chunk c covers 32c .. 32c + 31 -> words
// 16j .. 16j + 15).
// CG: coherent loads (x written earlier in the same launch), not the read-only path.
template <int W, int T, bool CG = false>
__device__ __forceinline__ void load_xp(const uint16_t* x, int H, int lane, uint32_t (&xp)[T][32]) {
    constexpr int PER = ChunkElems<W>::n;
    constexpr int NJ = D1_XPL / PER;
#pragma unroll
    for (int t = 0; t < T; ++t) {
#pragma unroll
        for (int j = 0; j < NJ; ++j) {
            const int c = lane + 32 * j;
#pragma unroll
            for (int q = 0; q < PER / 8; ++q) {
                const int idx = c * PER + q * 8;
                const uint4* px = reinterpret_cast<const uint4*>(x + size_t(t) * H + idx);
                const uint4 v = idx < H ? (CG ? __ldcg(px) : __ldg(px)) : make_uint4(0u, 0u, 0u, 0u);
                const int w = (j * (PER / 8) + q) * 4;
                xp[t][w] = v.x;
                xp[t][w + 1] = v.y;
                xp[t][w + 2] = v.z;
                xp[t][w + 3] = v.w;
            }
        }
    }
}

// A packed bf16 pair of x widened to fp32 where it is used: the conversion is kept inside
// the loop (volatile), so the compiler does not hoist the widened copies of all T rows of
// x out of phase B's loop and run out of registers.
__device__ __forceinline__ float2 bf2x(uint32_t w) {
    uint32_t lo, hi;
    asm volatile("shl.b32 %0, %2, 16;\n\tand.b32 %1, %2, 0xffff0000;" : "=r"(lo), "=r"(hi) : "r"(w));
    return make_float2(__uint_as_float(lo), __uint_as_float(hi));
}

// acc[t] += row . x_t for the rows t with bit t of `mask`
template <int T>
__device__ __forceinline__ void dotT_bf(const RowBF& r, const uint32_t (&xp)[T][32], unsigned mask, float2 (&acc)[T]) {
#pragma unroll
    for (int j = 0; j < D1_XPL / 8; ++j) {
        const float2 w0 = bf2(r.w[j].x), w1 = bf2(r.w[j].y), w2 = bf2(r.w[j].z), w3 = bf2(r.w[j].w);
#pragma unroll
        for (int t = 0; t < T; ++t) {
            if (mask >> t & 1u) {
                float2 a = acc[t];
                a = ffma2(w0, bf2x(xp[t][4 * j]), a);
                a = ffma2(w1, bf2x(xp[t][4 * j + 1]), a);
                a = ffma2(w2, bf2x(xp[t][4 * j + 2]), a);
                acc[t] = ffma2(w3, bf2x(xp[t][4 * j + 3]), a);
            }
        }
    }
}
template <int T>
__device__ __forceinline__ void dotT_q4(const RowQ4& r, const uint32_t (&xp)[T][32], unsigned mask, float2 (&acc)[T]) {
    const float2 off = make_float2(-8388616.0f, -8388616.0f);  // -(2^23 + 8)
#pragma unroll
    for (int j = 0; j < D1_XPL / 32; ++j) {
        const uint32_t w[4] = {r.w[j].x, r.w[j].y, r.w[j].z, r.w[j].w};
        float2 d[T];
#pragma unroll
        for (int t = 0; t < T; ++t) d[t] = make_float2(0.f, 0.f);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const uint32_t lo = w[q] & 0x0F0F0F0Fu, hi = (w[q] >> 4) & 0x0F0F0F0Fu;
#pragma unroll
            for (uint32_t b = 0; b < 4; ++b) {
                const float2 wf = fadd2(make_float2(code_f(lo, b), code_f(hi, b)), off);
#pragma unroll
                for (int t = 0; t < T; ++t)
                    if (mask >> t & 1u) d[t] = ffma2(wf, bf2x(xp[t][16 * j + 4 * q + b]), d[t]);
            }
        }
        const float s = bf16f(r.s[j]);
#pragma unroll
        for (int t = 0; t < T; ++t)
            if (mask >> t & 1u) acc[t] = ffma2(make_float2(s, s), d[t], acc[t]);
    }
}
template <int W, int T>
__device__ __forceinline__ void dotT(const typename RowOf<W>::type& r, const uint32_t (&xp)[T][32], unsigned mask,
                                     float2 (&acc)[T]) {
    if constexpr (W == DT_INT4) dotT_q4<T>(r, xp, mask, acc);
    else dotT_bf<T>(r, xp, mask, acc);
}

}  // namespace
}  // namespace redmoe
