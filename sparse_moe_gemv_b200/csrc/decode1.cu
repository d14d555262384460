// Decode path for one token row (T = 1) with bf16 or int4 group-32 experts: one
// persistent cooperative kernel per call (or per stack of layers).
//
// At T = 1 a layer is a pure stream: every weight byte the token needs is read once from
// HBM and used for one multiply-add. What costs time is not arithmetic but the three
// dependent steps (router -> routed gate/up -> down) and how fast each one reaches full
// bandwidth. This kernel is organised around that:
//
//   * Every lane keeps its slice of x in registers as fp32 for the whole layer, so a weight
//     chunk is dotted straight out of the registers it was loaded into: no shared-memory
//     traffic for activations or for gate/up weights.
//   * Phase A: warps stream the router rows, the shared-gate row and the shared expert's
//     gate/up rows (the shared expert needs no routing: the "extra slot" of the DwarfStar
//     MoE kernel, "Research notes, October 2026", section 1) with 16-byte vector loads.
//     Meanwhile one thread per block starts a bulk copy of the block's rows of the shared
//     expert's down matrix into shared memory.
//   * Grid barrier; every warp then computes the top-k of the 512 logits in registers
//     (router, top-k and shared gate form one stage, as in the same section). One thread
//     per block immediately starts bulk copies of the block's rows of the k routed
//     experts' down matrices: all of phase C's weights stream into shared memory while
//     phase B runs, since they do not depend on h.
//   * Phase B: each block takes an equal contiguous share of the k * I routed gate/up row
//     pairs; each warp keeps G pairs of loads in flight and writes h = silu(a) * u.
//   * Grid barrier; phase C computes the block's output rows from the down rows already
//     in shared memory and h (read from L2 into registers). Each output row is summed over
//     the experts in a fixed order: the result is deterministic.
//
// Down rows are only I = 512 elements long (1 KiB bf16, 256 B + 32 B int4): the block's
// rows of one expert form one contiguous range, copied in one piece, which is the lesson
// of the narrow-row kernel in "Research notes, October 2026", section 4.
#include <mutex>
#include <new>
#include <vector>

#include "common.cuh"
#include "gemv.cuh"
#include "internal.h"
#include "topk.cuh"

namespace redmoe {

namespace {

constexpr int D1_THREADS = 256;
constexpr int D1_WARPS = D1_THREADS / 32;
constexpr int D1_XPL = 64;        // x elements per lane (H = 2048 at most)
constexpr int D1_HPL = 16;        // h elements per lane (I = 512)
constexpr int D1_MAXK = 16;       // routed experts per token (plus the shared one)
constexpr int D1_RB_MAX = 16;     // output rows per block
constexpr int D1_G = 2;           // routed gate/up row pairs in flight per warp (bf16)

__host__ __device__ constexpr int a16(int x) { return (x + 15) & ~15; }

// Elements of one 16-byte weight chunk.
template <int W> struct ChunkElems { static constexpr int n = 8; };
template <> struct ChunkElems<DT_INT4> { static constexpr int n = 32; };
template <> struct ChunkElems<DT_INT2> { static constexpr int n = 64; };

// x slice of a lane as fp32, in the layout a weight type's 16-byte chunks need:
//   bf16 rows: chunk c = lane + 32 j (j < H / 256) covers elements 8c .. 8c + 7 -> xf[8j + m]
//   int4 rows: chunk c = lane + 32 j (j < H / 1024) covers elements 32c .. 32c + 31 -> xf[32j + m]
//   int2 rows: chunk c = lane (H = 2048) covers elements 64c .. 64c + 63 -> xf[m]
template <int W>
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
            v[j * (PER / 8) + q] = ok ? __ldg(reinterpret_cast<const uint4*>(x + size_t(c) * PER + q * 8))
                                      : make_uint4(0u, 0u, 0u, 0u);
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
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const float* xv = xf + 32 * j + 8 * q;
            a = ffma2(nib2(w[q], 0), make_float2(xv[0], xv[1]), a);
            b = ffma2(nib2(w[q], 2), make_float2(xv[2], xv[3]), b);
            a = ffma2(nib2(w[q], 4), make_float2(xv[4], xv[5]), a);
            b = ffma2(nib2(w[q], 6), make_float2(xv[6], xv[7]), b);
        }
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
// 16 consecutive int2 elements (one word) dotted with xv[0..16)
__device__ __forceinline__ float2 dot16_q2(uint32_t w, const float* xv) {
    float2 a = make_float2(0.f, 0.f), b = make_float2(0.f, 0.f);
#pragma unroll
    for (int n = 0; n < 16; n += 4) {
        a = ffma2(crumb2(w, n), make_float2(xv[n], xv[n + 1]), a);
        b = ffma2(crumb2(w, n + 2), make_float2(xv[n + 2], xv[n + 3]), b);
    }
    return fadd2(a, b);
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

__device__ __forceinline__ float hsum2(float2 v) { return warp_sum(v.x + v.y); }

// Shared-memory plan of the kernel (byte offsets). `dreg` holds the block's rows of the
// down matrix of k + 1 experts (routed slots 0..k-1 in selection order, the shared
// expert in slot k), each slot RB rows (int4: codes, then scales).
struct D1Smem {
    int dreg, slot, sc_off, bars, part, total;
};
__host__ __device__ inline D1Smem d1_smem(int wt, int k, int I, int RB) {
    D1Smem s;
    const int drow = d1_row_bytes(wt, I);
    s.sc_off = a16(RB * drow);
    s.slot = a16(s.sc_off + RB * d1_scale_bytes(wt, I));
    int o = 0;
    s.dreg = o; o += (k + 1) * s.slot;
    s.bars = o; o += 8 * (D1_MAXK + 1);
    s.part = o; o += 4 * D1_WARPS * D1_RB_MAX;
    s.total = a16(o);
    return s;
}

template <int NL>
struct D1Params {
    int H, E, k, I, n_layers, RB;
    Control* ctl;
    float* logits;  // [E]
    float* sgate;   // 2 x [1]
    float* hsh;     // 2 x [Is]
    float* hrt;     // [k, I]
    uint64_t timeout_ns;
    CacheBias cb;
    DecLayer L[NL];
};

template <int WT, int NL>
__global__ void __launch_bounds__(D1_THREADS, 1) decode1_kernel(const __grid_constant__ D1Params<NL> p) {
    extern __shared__ __align__(128) unsigned char smem[];
    using Row = typename RowOf<WT>::type;
    const int H = p.H, E = p.E, k = p.k, I = p.I, RB = p.RB;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int nblocks = gridDim.x;
    const int Wtot = nblocks * D1_WARPS;
    int* err = &p.ctl->err;
    const uint64_t to = p.timeout_ns;
    const D1Smem S = d1_smem(WT, k, I, RB);
    unsigned char* dreg = smem + S.dreg;
    uint64_t* dbar = reinterpret_cast<uint64_t*>(smem + S.bars);
    float* part = reinterpret_cast<float*>(smem + S.part);
    constexpr bool PACKED = WT != DT_BF16;           // int4 / int2: codes plus group scales
    const int drow = d1_row_bytes(WT, I);            // bytes of one down row (codes)
    const int dsc = d1_scale_bytes(WT, I);           // bytes of its scales
    const long grow = d1_row_bytes(WT, H);           // bytes of one gate/up row
    const int r0 = blockIdx.x * RB;
    const int nrows = max(0, min(RB, H - r0));
    unsigned bar_idx = 0;

    if (threadIdx.x == 0) {
        for (int i = 0; i <= k; ++i) mbar_init(dbar + i, 1);
        fence_mbar_init();
    }
    __syncthreads();

    // bulk copy of the block's rows of one down matrix (and int4 scales) into slot `s`
    auto issue_down = [&](int s, const void* wd, const uint16_t* sd) {
        unsigned char* dst = dreg + s * S.slot;
        const uint32_t bytes = uint32_t(nrows * drow), sbytes = uint32_t(nrows * dsc);
        mbar_arrive_expect_tx(dbar + s, bytes + sbytes);
        bulk_g2s(dst, static_cast<const char*>(wd) + size_t(r0) * drow, bytes, dbar + s);
        if (PACKED) bulk_g2s(dst + S.sc_off, reinterpret_cast<const char*>(sd) + size_t(r0) * dsc, sbytes, dbar + s);
    };

    for (int l = 0; l < p.n_layers; ++l) {
        const DecLayer& Ly = p.L[l];
        const uint16_t* x = static_cast<const uint16_t*>(Ly.x);
        float* sgate = p.sgate + (l & 1);
        float* hsh = p.hsh + size_t(l & 1) * I;
        const uint32_t par = uint32_t(l & 1);

        // ------------------------------------------------------------ phase A
        if (threadIdx.x == 0 && nrows > 0) {
            fence_proxy_async_smem();  // the previous layer's reads of dreg come first
            issue_down(k, Ly.sh_down, Ly.sh_s_down);
        }
        // job q < E: router row q; q == E: shared-gate row; q > E: shared gate/up row q-E-1.
        // Warp w of block b takes q = w * nblocks + b (+ Wtot ...): every block gets a few
        // of each kind.
        const int jobsA = E + 1 + I;
        for (int q = warp * nblocks + blockIdx.x; q < jobsA; q += Wtot) {
            if (q <= E) {
                float xf[D1_XPL];
                RowBF r;
                const void* row = q < E ? static_cast<const void*>(static_cast<const char*>(Ly.router_w) + size_t(q) * 2 * H)
                                        : Ly.shared_gate_w;
                ld_row_bf(r, row, H, lane);
                load_x<DT_BF16>(x, H, lane, xf);
                const float v = hsum2(dot_row_bf(r, xf));
                if (lane == 0) {
                    if (q < E) p.logits[q] = v + (Ly.router_bias ? Ly.router_bias[q] : 0.0f);
                    else *sgate = 1.0f / (1.0f + expf(-v));
                }
            } else {
                const int i = q - E - 1;
                float xf[D1_XPL];
                Row g, u;
                ld_row<WT>(g, static_cast<const char*>(Ly.sh_gate) + size_t(i) * grow,
                           PACKED ? Ly.sh_s_gate + size_t(i) * (H / 32) : nullptr, H, lane);
                ld_row<WT>(u, static_cast<const char*>(Ly.sh_up) + size_t(i) * grow,
                           PACKED ? Ly.sh_s_up + size_t(i) * (H / 32) : nullptr, H, lane);
                load_x<WT>(x, H, lane, xf);
                const float a = hsum2(dot_row<WT>(g, xf)), b = hsum2(dot_row<WT>(u, xf));
                if (lane == 0) hsh[i] = silu_mul(a, b);
            }
        }
        grid_barrier(p.ctl, nblocks, bar_idx++, to);

        // ------------------------------------------------------------ phase B
        // top-k of the logits by every warp, in registers: lane j < k ends with the id and
        // the renormalised weight of selection j
        int sel_id;
        float sel_w;
        if (E <= 512) warp_route<16>(p.logits, E, k, p.cb.cached, p.cb.lambda, sel_id, sel_w);
        else warp_route<MAX_EXPERTS / 32>(p.logits, E, k, p.cb.cached, p.cb.lambda, sel_id, sel_w);
        if (blockIdx.x == 0 && warp == 0 && lane < k) {
            Ly.ids[lane] = sel_id;
            Ly.w[lane] = sel_w;
        }
        if (warp == 0 && nrows > 0) {
            // phase C's routed down rows do not depend on h: start their copies now
            for (int j = 0; j < k; ++j) {
                const int e = __shfl_sync(FULL, sel_id, j);
                if (lane == 0)
                    issue_down(j, static_cast<const char*>(Ly.w_down) + size_t(e) * H * drow,
                               PACKED ? Ly.s_down + size_t(e) * H * (I / 32) : nullptr);
            }
        }
        {
            float xf[D1_XPL];
            load_x<WT>(x, H, lane, xf);
            // this block's share [j0, j1) of the k * I routed row pairs (u-major)
            const int J = k * I;
            const int j0 = int((long long)J * blockIdx.x / nblocks), j1 = int((long long)J * (blockIdx.x + 1) / nblocks);
            constexpr int G = (WT == DT_INT2) ? 8 : ((WT == DT_INT4) ? 4 : D1_G);
            for (int jb = j0 + warp; jb < j1; jb += D1_WARPS * G) {
                Row g[G], u[G];
#pragma unroll
                for (int t = 0; t < G; ++t) {
                    const int j = jb + t * D1_WARPS;
                    const int uu = j / I, i = j - (j / I) * I;
                    const int e = __shfl_sync(FULL, sel_id, uu < k ? uu : 0);
                    if (j < j1) {
                        const size_t rowi = size_t(e) * I + i;
                        ld_row<WT>(g[t], static_cast<const char*>(Ly.w_gate) + rowi * grow,
                                   PACKED ? Ly.s_gate + rowi * (H / 32) : nullptr, H, lane);
                        ld_row<WT>(u[t], static_cast<const char*>(Ly.w_up) + rowi * grow,
                                   PACKED ? Ly.s_up + rowi * (H / 32) : nullptr, H, lane);
                    }
                }
#pragma unroll
                for (int t = 0; t < G; ++t) {
                    const int j = jb + t * D1_WARPS;
                    if (j < j1) {
                        const float a = hsum2(dot_row<WT>(g[t], xf)), b = hsum2(dot_row<WT>(u[t], xf));
                        if (lane == 0) p.hrt[j] = silu_mul(a, b);
                    }
                }
            }
        }
        grid_barrier(p.ctl, nblocks, bar_idx++, to);

        // ------------------------------------------------------------ phase C
        if (l + 1 < p.n_layers && threadIdx.x < 32) {
            // L2 prefetch of the next layer's router rows and shared gate/up rows (this
            // block's phase-A jobs of that layer)
            const DecLayer& Nx = p.L[l + 1];
            for (int q = lane * nblocks + blockIdx.x; q < E + 1 + I; q += 32 * nblocks) {
                if (q < E) prefetch_l2(static_cast<const char*>(Nx.router_w) + size_t(q) * 2 * H, 2 * H);
                else if (q > E) {
                    prefetch_l2(static_cast<const char*>(Nx.sh_gate) + size_t(q - E - 1) * grow, grow);
                    prefetch_l2(static_cast<const char*>(Nx.sh_up) + size_t(q - E - 1) * grow, grow);
                }
            }
        }
        // units (slot u, half hf of the block's rows): 2 (k + 1) units over the warps; each
        // warp accumulates its rows' weighted partials in registers
        const int half = (nrows + 1) / 2;
        float2 acc[D1_RB_MAX / 2];
#pragma unroll
        for (int r = 0; r < D1_RB_MAX / 2; ++r) acc[r] = make_float2(0.f, 0.f);
        const float sg = __ldcg(sgate);
        for (int unit = warp; nrows > 0 && unit < 2 * (k + 1); unit += D1_WARPS) {
            const int u = unit >> 1, hf = unit & 1;
            const int ra = hf * half, rn = min(half, nrows - ra);
            const float* hv = (u < k ? p.hrt + size_t(u) * I : hsh) + lane * D1_HPL;
            float hf32[D1_HPL];
#pragma unroll
            for (int i = 0; i < D1_HPL / 4; ++i) {
                const float4 v = __ldcg(reinterpret_cast<const float4*>(hv) + i);
                hf32[4 * i] = v.x; hf32[4 * i + 1] = v.y; hf32[4 * i + 2] = v.z; hf32[4 * i + 3] = v.w;
            }
            const float wu = u < k ? __shfl_sync(FULL, sel_w, u) : sg;
            mbar_wait(dbar + u, par, err, to);
            const unsigned char* slot = dreg + u * S.slot;
#pragma unroll
            for (int r = 0; r < D1_RB_MAX / 2; ++r) {
                if (r < rn) {
                    float2 d = make_float2(0.f, 0.f);
                    if constexpr (WT == DT_INT2) {
                        const uint32_t wv = *reinterpret_cast<const uint32_t*>(slot + (ra + r) * drow + lane * 4);
                        const float s = bf16f(*reinterpret_cast<const uint16_t*>(slot + S.sc_off + (ra + r) * dsc + (lane >> 1) * 2));
                        d = ffma2(make_float2(s, s), dot16_q2(wv, hf32), d);
                    } else if constexpr (WT == DT_INT4) {
                        const uint2 wv = *reinterpret_cast<const uint2*>(slot + (ra + r) * drow + lane * 8);
                        const float s = bf16f(*reinterpret_cast<const uint16_t*>(slot + S.sc_off + (ra + r) * dsc + (lane >> 1) * 2));
                        float2 a = make_float2(0.f, 0.f);
                        a = ffma2(nib2(wv.x, 0), make_float2(hf32[0], hf32[1]), a);
                        a = ffma2(nib2(wv.x, 2), make_float2(hf32[2], hf32[3]), a);
                        a = ffma2(nib2(wv.x, 4), make_float2(hf32[4], hf32[5]), a);
                        a = ffma2(nib2(wv.x, 6), make_float2(hf32[6], hf32[7]), a);
                        a = ffma2(nib2(wv.y, 0), make_float2(hf32[8], hf32[9]), a);
                        a = ffma2(nib2(wv.y, 2), make_float2(hf32[10], hf32[11]), a);
                        a = ffma2(nib2(wv.y, 4), make_float2(hf32[12], hf32[13]), a);
                        a = ffma2(nib2(wv.y, 6), make_float2(hf32[14], hf32[15]), a);
                        d = ffma2(make_float2(s, s), a, d);
                    } else {
                        const uint4* wr = reinterpret_cast<const uint4*>(slot + (ra + r) * drow + lane * 32);
                        const uint4 w0 = wr[0], w1 = wr[1];
                        d = ffma2(bf2(w0.x), make_float2(hf32[0], hf32[1]), d);
                        d = ffma2(bf2(w0.y), make_float2(hf32[2], hf32[3]), d);
                        d = ffma2(bf2(w0.z), make_float2(hf32[4], hf32[5]), d);
                        d = ffma2(bf2(w0.w), make_float2(hf32[6], hf32[7]), d);
                        d = ffma2(bf2(w1.x), make_float2(hf32[8], hf32[9]), d);
                        d = ffma2(bf2(w1.y), make_float2(hf32[10], hf32[11]), d);
                        d = ffma2(bf2(w1.z), make_float2(hf32[12], hf32[13]), d);
                        d = ffma2(bf2(w1.w), make_float2(hf32[14], hf32[15]), d);
                    }
                    acc[r] = ffma2(make_float2(wu, wu), d, acc[r]);
                }
            }
            // a warp's units all share its half: unit = warp + 8 m keeps hf = warp & 1
        }
        // per row: reduce the lanes, then sum the warps' partials in a fixed order
        {
            const int hf = warp & 1;
            const int ra = hf * half, rn = nrows > 0 ? min(half, nrows - ra) : 0;
#pragma unroll
            for (int r = 0; r < D1_RB_MAX / 2; ++r) {
                const float v = warp_sum(acc[r].x + acc[r].y);
                if (lane == 0 && r < rn) part[warp * D1_RB_MAX + ra + r] = v;
            }
        }
        __syncthreads();
        if (threadIdx.x < nrows) {
            const int r = threadIdx.x, hf = r >= half ? 1 : 0;
            float o = 0.0f;
            for (int w = hf; w < D1_WARPS; w += 2) o += part[w * D1_RB_MAX + r];
            Ly.out[r0 + r] = o;
        }
        if (l + 1 < p.n_layers) grid_barrier(p.ctl, nblocks, bar_idx++, to);
    }
    grid_exit(p.ctl, nblocks);
}

int d1_blocks_per_sm(const void* kern, int smem) {
    struct Entry {
        int dev;
        const void* kern;
        int smem;
        int per_sm;
    };
    static std::mutex mu;
    static std::vector<Entry> cache;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return -1;
    std::lock_guard<std::mutex> lock(mu);
    for (const Entry& e : cache)
        if (e.dev == dev && e.kern == kern && e.smem == smem) return e.per_sm;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess) return -1;
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, D1_THREADS, smem) != cudaSuccess) return -1;
    per_sm = per_sm > 1 ? 1 : per_sm;
    cache.push_back({dev, kern, smem, per_sm});
    return per_sm;
}

template <int WT, int NL>
redmoe_status d1_launch(const redmoe_layer* sh, const DecLayer* layers, int n_layers, void* ws, cudaStream_t stream,
                        CacheBias cb) {
    DevInfo di;
    if (!get_dev_info(&di)) return REDMOE_ERR_CUDA;
    const int RB = (sh->hidden + di.sm_count - 1) / di.sm_count;
    if (RB > D1_RB_MAX) return REDMOE_ERR_UNSUPPORTED;
    const D1Smem S = d1_smem(WT, sh->top_k, sh->inter, RB);
    if (S.total > di.max_smem_optin) return REDMOE_ERR_UNSUPPORTED;
    auto kern = decode1_kernel<WT, NL>;
    const int per_sm = d1_blocks_per_sm(reinterpret_cast<const void*>(kern), S.total);
    if (per_sm < 0) return REDMOE_ERR_CUDA;
    if (per_sm == 0) return REDMOE_ERR_UNSUPPORTED;

    D1Params<NL>* pp = new (std::nothrow) D1Params<NL>();
    if (!pp) return REDMOE_ERR_CUDA;
    D1Params<NL>& q = *pp;
    q.H = sh->hidden; q.E = sh->n_experts; q.k = sh->top_k; q.I = sh->inter;
    q.n_layers = n_layers;
    q.RB = RB;
    const DecodeWs L = decode_ws_layout(1, q.E, q.k, q.I, sh->shared_inter);
    char* base = static_cast<char*>(ws);
    q.ctl = reinterpret_cast<Control*>(base);
    q.logits = reinterpret_cast<float*>(base + L.logits);
    q.sgate = reinterpret_cast<float*>(base + L.sgate);
    q.hsh = reinterpret_cast<float*>(base + L.hsh);
    q.hrt = reinterpret_cast<float*>(base + L.hrt);
    q.timeout_ns = BARRIER_TIMEOUT_NS;
    q.cb = cb;
    for (int i = 0; i < n_layers; ++i) q.L[i] = layers[i];

    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(di.sm_count * per_sm);
    cfg.blockDim = dim3(D1_THREADS);
    cfg.dynamicSmemBytes = S.total;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const cudaError_t err = cudaLaunchKernelEx(&cfg, kern, q);
    delete pp;
    return err == cudaSuccess ? REDMOE_OK : REDMOE_ERR_CUDA;
}

template <int WT>
redmoe_status d1_launch_all(const redmoe_layer* sh, const DecLayer* layers, int n_layers, void* ws, cudaStream_t stream,
                            int* launches, CacheBias cb) {
    redmoe_status st = REDMOE_OK;
    if (n_layers == 1) {
        st = d1_launch<WT, 1>(sh, layers, 1, ws, stream, cb);
        if (st == REDMOE_OK && launches) *launches += 1;
        return st;
    }
    for (int l0 = 0; l0 < n_layers && st == REDMOE_OK; l0 += MAX_STACK) {
        const int n = n_layers - l0 < MAX_STACK ? n_layers - l0 : MAX_STACK;
        st = d1_launch<WT, MAX_STACK>(sh, layers + l0, n, ws, stream, cb);
        if (st == REDMOE_OK && launches) *launches += 1;
    }
    return st;
}

}  // namespace

// Layers the one-row kernel takes: bf16 x and router, bf16 or int4 experts, the
// Qwen3-Next expert width (I = Is = 512), H up to 2048 in whole chunks per lane, k up to
// D1_MAXK, and at most D1_RB_MAX output rows per block.
bool decode1_shape_ok(const redmoe_layer* sh) {
    const int H = sh->hidden, wt = sh->expert_dtype;
    if (sh->x_dtype != DT_BF16 || sh->router_dtype != DT_BF16) return false;
    if (sh->inter != 512 || sh->shared_inter != 512) return false;
    if (wt != DT_BF16 && wt != DT_INT4 && wt != DT_INT2) return false;
    if (H > 32 * D1_XPL || H % (wt == DT_INT2 ? 2048 : (wt == DT_INT4 ? 1024 : 256))) return false;
    if (sh->top_k > D1_MAXK || sh->n_experts > MAX_EXPERTS) return false;
    return true;
}

redmoe_status launch_decode1(const redmoe_layer* sh, const DecLayer* layers, int n_layers, void* ws,
                             cudaStream_t stream, int* launches, CacheBias cb) {
    if (sh->expert_dtype == DT_INT4) return d1_launch_all<DT_INT4>(sh, layers, n_layers, ws, stream, launches, cb);
    if (sh->expert_dtype == DT_INT2) return d1_launch_all<DT_INT2>(sh, layers, n_layers, ws, stream, launches, cb);
    return d1_launch_all<DT_BF16>(sh, layers, n_layers, ws, stream, launches, cb);
}

}  // namespace redmoe
