// Decode path for two or three token rows with bf16 or int4 experts: the few-row matvec of
// parallel-2 serving and 2- or 3-row speculative verify ("Research notes, October 2026",
// section 1, MTP "Verify" bullet: the draft is verified as a 2- or 3-row forward on the
// decode kernels). One persistent cooperative kernel per call (or per stack of layers).
//
// The organisation is that of the one-row kernel (decode1.cu), with T activation rows:
//
//   * Every lane keeps its slice of each row of x in registers as packed bf16 pairs (32
//     words per row), in the layout its 16-byte weight chunks need; a weight chunk is
//     widened once and dotted with every row that needs it.
//   * Phase A: router rows, the shared-gate row and the shared expert's gate/up rows, one
//     job per warp; one thread per block bulk-copies its rows of the shared expert's down
//     matrix into shared-memory slot 0.
//   * Grid barrier; warps 0 .. T-1 each take the top-k of one row of logits; warps 4 and 5
//     take phase C's two units of the shared expert. One warp then finds the distinct
//     experts of the T * k selections with one warp-wide match (T * k <= 32), and one
//     thread starts bulk copies of the block's rows of the first distinct experts' down
//     matrices into the remaining slots, and L2 prefetches of the rows of the others.
//   * Phase B: the U * I gate/up row pairs of the U distinct experts, interleaved over all
//     warps; each pair is dotted with the rows of x that selected its expert.
//   * Grid barrier; the h rows are bulk-copied into shared memory; phase C computes the
//     block's output rows (down rows from the slots, or from L2 for the experts that did
//     not fit) and sums each output over the experts in a fixed order: deterministic.
#include <mutex>
#include <new>
#include <vector>

#include "common.cuh"
#include "gemv.cuh"
#include "internal.h"
#include "rowdot.cuh"
#include "topk.cuh"

namespace redmoe {

namespace {

constexpr int FR_MAXT = 3;
constexpr int FR_MAXSEL = 32;                 // routed selections of a call, T * k (one warp)
constexpr int FR_MAXSLOT = 48;                // shared-memory down slots (shared expert in 0)

__device__ __forceinline__ float hsum_fr(float2 v) { return warp_sum(v.x + v.y); }

struct FrSmem {
    int dreg, slot, sc_off, nslot, hbuf, bars, part, psh, sel, total;
};
// Shared memory of the kernel: nslot down slots (slot 0 the shared expert, then the
// first distinct routed experts), the routed h rows, barriers, per-warp partial sums and
// the selection tables.
__host__ __device__ inline FrSmem fr_smem(int wt, int T, int k, int I, int RB, int max_smem) {
    FrSmem s;
    const int drow = d1_row_bytes(wt, I);
    s.sc_off = a16(RB * drow);
    s.slot = a16(s.sc_off + RB * d1_scale_bytes(wt, I));
    const int sel = a16(4 * (4 * FR_MAXSEL + 2 * FR_MAXSEL * FR_MAXT + 4));
    const int fixed = a16(4 * T * k * I) + 8 * (FR_MAXSLOT + 1) + a16(4 * D1_WARPS * D1_RB_MAX * T) +
                      a16(4 * D1_RB_MAX * T) + sel;
    int n = (max_smem - fixed) / s.slot;
    if (n > FR_MAXSLOT) n = FR_MAXSLOT;
    if (n > T * k + 1) n = T * k + 1;
    s.nslot = n;
    int o = 0;
    s.dreg = o; o += n * s.slot;
    s.hbuf = o; o += a16(4 * T * k * I);
    s.bars = o; o += 8 * (FR_MAXSLOT + 1);
    s.part = o; o += a16(4 * D1_WARPS * D1_RB_MAX * T);
    s.psh = o; o += a16(4 * D1_RB_MAX * T);  // the shared expert's partials, per row and token
    s.sel = o; o += sel;
    s.total = a16(o);
    return s;
}

template <int NL>
struct FrParams {
    int H, E, k, I, n_layers, RB, max_smem;
    Control* ctl;
    float* logits;  // [T, E]
    float* sgate;   // 2 x [T]
    float* hsh;     // 2 x [T, I]
    float* hrt;     // [T * k, I]   (row t * k + j: selection j of token t)
    uint64_t timeout_ns;
    CacheBias cb;
    // non-null: every layer's x is pinned host memory (its device mapping in L[l].x); at
    // each layer's start warp 7 of blocks 0 .. 4T-1 copies a quarter row each here and counts
    // on Control::x_ready, and every x read of the layer comes from here
    uint16_t* xstage;
    DecLayer L[NL];
};

// A quarter of one row of x (H/4 bf16 elements) from pinned host memory into the
// workspace copy, by one warp: cache-volatile loads (the host rewrites x between calls),
// every load of a lane issued before its first store (one link round trip), then a count
// on x_ready with a release.
__device__ __forceinline__ void fetch_host_quarter(const uint4* src_row, uint4* dst_row, int quarter, int H, int lane,
                                                   unsigned* x_ready) {
    constexpr int PER = D1_XPL / 32;  // 16-byte chunks per lane: a quarter row per warp
    const int c0 = quarter * (H / 32) + lane;
    uint4 v[PER];
#pragma unroll
    for (int j = 0; j < PER; ++j)
        if (32 * j + lane < H / 32) v[j] = __ldcv(src_row + c0 + 32 * j);
#pragma unroll
    for (int j = 0; j < PER; ++j)
        if (32 * j + lane < H / 32) dst_row[c0 + 32 * j] = v[j];
    __threadfence();
    __syncwarp();
    if (lane == 0) asm volatile("red.release.gpu.global.add.u32 [%0], 1;" :: "l"(x_ready) : "memory");
}

// XR: x comes from pinned host memory through p.xstage (a separate instantiation, so
// that calls on device buffers run without its waits and coherent loads).
template <int WT, int T, int NL, bool XR>
__global__ void __launch_bounds__(D1_THREADS, 1) decodefr_kernel(const __grid_constant__ FrParams<NL> p) {
    extern __shared__ __align__(128) unsigned char smem[];
    using Row = typename RowOf<WT>::type;
    constexpr bool PACKED = WT != DT_BF16;
    const int H = p.H, E = p.E, k = p.k, I = p.I, RB = p.RB;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int nblocks = gridDim.x;
    const int Wtot = nblocks * D1_WARPS;
    int* err = &p.ctl->err;
    const uint64_t to = p.timeout_ns;
    const FrSmem S = fr_smem(WT, T, k, I, RB, p.max_smem);
    unsigned char* dreg = smem + S.dreg;
    uint64_t* dbar = reinterpret_cast<uint64_t*>(smem + S.bars);
    uint64_t* hbar = dbar + FR_MAXSLOT;
    const float* hbuf = reinterpret_cast<const float*>(smem + S.hbuf);
    float* part = reinterpret_cast<float*>(smem + S.part);  // [warp][row][t]
    float* psh = reinterpret_cast<float*>(smem + S.psh);    // [row][t]
    int* s_ids = reinterpret_cast<int*>(smem + S.sel);          // [T * k] expert of selection i
    float* s_w = reinterpret_cast<float*>(s_ids + FR_MAXSEL);    // [T * k] its weight
    int* s_ue = s_ids + 2 * FR_MAXSEL;                          // [U] expert of distinct index u
    int* s_um = s_ids + 3 * FR_MAXSEL;                          // [U] rows of x that selected it
    int* s_us = s_ids + 4 * FR_MAXSEL;                          // [U][T] its selection per row, or -1
    float* s_uw = reinterpret_cast<float*>(s_us + FR_MAXSEL * FR_MAXT);  // [U][T] its weight per row
    int* s_nu = s_us + 2 * FR_MAXSEL * FR_MAXT;                 // U
    const int drow = d1_row_bytes(WT, I), dsc = d1_scale_bytes(WT, I);
    const long grow = d1_row_bytes(WT, H);
    const int r0 = blockIdx.x * RB;
    const int nrows = max(0, min(RB, H - r0));
    const int half = (nrows + 1) / 2;
    const int ra = (warp & 1) * half, rn = nrows > 0 ? min(half, nrows - ra) : 0;
    unsigned bar_idx = 0;

    if (threadIdx.x == 0) {
        for (int i = 0; i < S.nslot; ++i) mbar_init(dbar + i, 1);
        mbar_init(hbar, 1);
        fence_mbar_init();
    }
    __syncthreads();

    auto issue_down = [&](int s, const void* wd, const uint16_t* sd) {
        unsigned char* dst = dreg + s * S.slot;
        const uint32_t bytes = uint32_t(nrows * drow), sbytes = uint32_t(nrows * dsc);
        mbar_arrive_expect_tx(dbar + s, bytes + sbytes);
        bulk_g2s(dst, static_cast<const char*>(wd) + size_t(r0) * drow, bytes, dbar + s);
        if (PACKED) bulk_g2s(dst + S.sc_off, reinterpret_cast<const char*>(sd) + size_t(r0) * dsc, sbytes, dbar + s);
    };

    for (int l = 0; l < p.n_layers; ++l) {
        const DecLayer& Ly = p.L[l];
        constexpr bool xremote = XR;
        const uint16_t* x = xremote ? p.xstage : static_cast<const uint16_t*>(Ly.x);
        float* sgate = p.sgate + (l & 1) * T;
        float* hsh = p.hsh + size_t(l & 1) * T * I;
        const uint32_t par = uint32_t(l & 1);

        // ------------------------------------------------------------ phase A
        if (threadIdx.x == 0 && nrows > 0) {
            fence_proxy_async_smem();  // the previous layer's reads of the slots come first
            issue_down(0, Ly.sh_down, Ly.sh_s_down);
        }
        bool xready = !xremote;  // this warp has seen the layer's x published
        if (xremote && (NL == 1 || l == 0 || 4 * T > D1_WARPS) && blockIdx.x < 4 * T && warp == D1_WARPS - 1) {
            // x from host memory: a quarter of row blockIdx.x / 4 per block, read once over
            // the link with cache-volatile loads (the host rewrites it between calls), every
            // load of a lane issued before its first store (one link round trip). A later
            // stacked layer's x is fetched ahead, during the layer before (phase C).
            constexpr int PER = D1_XPL / 32;  // 16-byte chunks per lane: a quarter row per warp
            const uint4* src = static_cast<const uint4*>(Ly.x) + size_t(blockIdx.x >> 2) * (H / 8);
            uint4* dst = reinterpret_cast<uint4*>(p.xstage) + size_t(blockIdx.x >> 2) * (H / 8);
            const int c0 = (blockIdx.x & 3) * (H / 32) + lane;
            uint4 v[PER];
#pragma unroll
            for (int j = 0; j < PER; ++j)
                if (32 * j + lane < H / 32) v[j] = __ldcv(src + c0 + 32 * j);
#pragma unroll
            for (int j = 0; j < PER; ++j)
                if (32 * j + lane < H / 32) dst[c0 + 32 * j] = v[j];
            __threadfence();
            __syncwarp();
            if (lane == 0) asm volatile("red.release.gpu.global.add.u32 [%0], 1;" :: "l"(&p.ctl->x_ready) : "memory");
        }
        // a warp's first x read of the layer waits until all 4T quarters are published
        auto wait_x = [&]() {
            if (xready) return;
            if (lane == 0) {
                const uint64_t t0 = globaltimer_ns();
                for (uint32_t spins = 0; ld_acquire_gpu(&p.ctl->x_ready) < 4u * T * unsigned(l + 1); ++spins) {
                    if ((spins & 63u) == 63u && (globaltimer_ns() - t0 > to || spins > (1u << 26))) {
                        atomicOr(err, ERRBIT_TIMEOUT);
                        break;
                    }
                }
            }
            __syncwarp();
            xready = true;
        };
        for (int q = warp * nblocks + blockIdx.x; q < E + 1 + I; q += Wtot) {
            float2 a[T], b[T];
#pragma unroll
            for (int t = 0; t < T; ++t) a[t] = b[t] = make_float2(0.f, 0.f);
            if (q <= E) {
                uint32_t xp[T][32];
                RowBF r;
                const void* row = q < E ? static_cast<const void*>(static_cast<const char*>(Ly.router_w) + size_t(q) * 2 * H)
                                        : Ly.shared_gate_w;
                ld_row_bf(r, row, H, lane);
                wait_x();
                load_xp<DT_BF16, T, XR>(x, H, lane, xp);
                dotT_bf<T>(r, xp, (1u << T) - 1u, a);
#pragma unroll
                for (int t = 0; t < T; ++t) {
                    const float v = hsum_fr(a[t]);
                    if (lane == 0) {
                        if (q < E) p.logits[t * E + q] = v + (Ly.router_bias ? Ly.router_bias[q] : 0.0f);
                        else sgate[t] = 1.0f / (1.0f + expf(-v));
                    }
                }
            } else {
                const int i = q - E - 1;
                uint32_t xp[T][32];
                Row g, u;
                ld_row<WT>(g, static_cast<const char*>(Ly.sh_gate) + size_t(i) * grow,
                           PACKED ? Ly.sh_s_gate + size_t(i) * (H / 32) : nullptr, H, lane);
                ld_row<WT>(u, static_cast<const char*>(Ly.sh_up) + size_t(i) * grow,
                           PACKED ? Ly.sh_s_up + size_t(i) * (H / 32) : nullptr, H, lane);
                wait_x();
                load_xp<WT, T, XR>(x, H, lane, xp);
                dotT<WT, T>(g, xp, (1u << T) - 1u, a);
                dotT<WT, T>(u, xp, (1u << T) - 1u, b);
#pragma unroll
                for (int t = 0; t < T; ++t) {
                    const float av = hsum_fr(a[t]), bv = hsum_fr(b[t]);
                    if (lane == 0) hsh[size_t(t) * I + hpos<WT>(i)] = silu_mul(av, bv);
                }
            }
        }
        grid_barrier(p.ctl, nblocks, bar_idx++, to);

        // weighted row dots of one unit (expert rows ra .. ra + rn of the block at `rows`,
        // int4 scales at `scl`, row stride `rstride` bytes): acc[r][t] += w_t * row . h_t
        // for the rows t of `mask`, h_t at hv[t]
        auto unit_dots = [&](float2 (&acc)[D1_RB_MAX / 2][T], const unsigned char* rows, const unsigned char* scl,
                             long rstride, long sstride, unsigned mask, const float (&wt)[T],
                             const float* const (&hv)[T], bool h_global) {
            float hh[T][D1_HPL];
#pragma unroll
            for (int t = 0; t < T; ++t) {
                if (mask >> t & 1u) {
                    const float4* h4 = reinterpret_cast<const float4*>(hv[t]) + lane;
#pragma unroll
                    for (int i = 0; i < D1_HPL / 4; ++i) {
                        const float4 v = h_global ? __ldcg(h4 + 32 * i) : h4[32 * i];
                        hh[t][4 * i] = v.x; hh[t][4 * i + 1] = v.y; hh[t][4 * i + 2] = v.z; hh[t][4 * i + 3] = v.w;
                    }
                }
            }
#pragma unroll
            for (int r = 0; r < D1_RB_MAX / 2; ++r) {
                {
                    // rows past rn dot a valid row: no branch per row, the result is unused
                    const int rr = min(ra + r, nrows - 1);
                    const unsigned char* row = rows + rr * rstride;
                    if constexpr (WT == DT_INT4) {
                        const uint2 wv = *reinterpret_cast<const uint2*>(row + lane * 8);
                        const float s = bf16f(*reinterpret_cast<const uint16_t*>(scl + rr * sstride + (lane >> 1) * 2));
#pragma unroll
                        for (int t = 0; t < T; ++t) {
                            if (mask >> t & 1u) {
                                const float2 a = dot8_q4(wv.x, hh[t], make_float2(0.f, 0.f));
                                const float2 b = dot8_q4(wv.y, hh[t] + 8, make_float2(0.f, 0.f));
                                acc[r][t] = ffma2(make_float2(s * wt[t], s * wt[t]), fadd2(a, b), acc[r][t]);
                            }
                        }
                    } else {
                        const uint4 w0 = *reinterpret_cast<const uint4*>(row + lane * 16);
                        const uint4 w1 = *reinterpret_cast<const uint4*>(row + 512 + lane * 16);
                        const float2 f[8] = {bf2(w0.x), bf2(w0.y), bf2(w0.z), bf2(w0.w),
                                             bf2(w1.x), bf2(w1.y), bf2(w1.z), bf2(w1.w)};
#pragma unroll
                        for (int t = 0; t < T; ++t) {
                            if (mask >> t & 1u) {
                                float2 d = make_float2(0.f, 0.f), e = make_float2(0.f, 0.f);
#pragma unroll
                                for (int m = 0; m < 8; m += 2) {
                                    d = ffma2(f[m], make_float2(hh[t][2 * m], hh[t][2 * m + 1]), d);
                                    e = ffma2(f[m + 1], make_float2(hh[t][2 * m + 2], hh[t][2 * m + 3]), e);
                                }
                                acc[r][t] = ffma2(make_float2(wt[t], wt[t]), fadd2(d, e), acc[r][t]);
                            }
                        }
                    }
                }
            }
        };

        // ------------------------------------------------------------ phase B
        if (warp < T) {
            // the top-k of row `warp` of the logits
            int id;
            float wv;
            warp_route<D1_MAXE / 32>(p.logits + size_t(warp) * E, E, k, p.cb.cached, p.cb.lambda, id, wv);
            if (lane < k) {
                s_ids[warp * k + lane] = id;
                s_w[warp * k + lane] = wv;
                if (blockIdx.x == 0) {
                    Ly.ids[warp * k + lane] = id;
                    Ly.w[warp * k + lane] = wv;
                }
            }
        } else if ((warp == 4 || warp == 5) && nrows > 0) {
            // phase C's two units of the shared expert: its h rows and down rows are ready
            mbar_wait(dbar + 0, par, err, to);
            float wt[T];
            const float* hv[T];
#pragma unroll
            for (int t = 0; t < T; ++t) {
                wt[t] = __ldcg(sgate + t);
                hv[t] = hsh + size_t(t) * I;
            }
            float2 accs[D1_RB_MAX / 2][T];
#pragma unroll
            for (int r = 0; r < D1_RB_MAX / 2; ++r)
#pragma unroll
                for (int t = 0; t < T; ++t) accs[r][t] = make_float2(0.f, 0.f);
            unit_dots(accs, dreg, dreg + S.sc_off, drow, dsc, (1u << T) - 1u, wt, hv, true);
#pragma unroll
            for (int r = 0; r < D1_RB_MAX / 2; ++r) {
#pragma unroll
                for (int t = 0; t < T; ++t) {
                    const float v = warp_sum(accs[r][t].x + accs[r][t].y);
                    if (lane == 0 && r < rn) psh[(ra + r) * T + t] = v;
                }
            }
        }
        __syncthreads();
        if (warp == 0) {
            // distinct experts of the T * k selections: one match over the warp
            const int ns = T * k;
            const int e = lane < ns ? s_ids[lane] : -1 - lane;
            const unsigned peers = __match_any_sync(FULL, e);
            const int leader = __ffs(peers) - 1;
            const unsigned leads = __ballot_sync(FULL, lane < ns && lane == leader);
            const int u = __popc(leads & ((1u << leader) - 1u));
            if (lane < ns && lane == leader) {
                unsigned m = 0;
                for (unsigned rest = peers; rest; rest &= rest - 1) m |= 1u << ((__ffs(rest) - 1) / k);
                s_ue[u] = e;
                s_um[u] = int(m);
#pragma unroll
                for (int t = 0; t < T; ++t) s_us[u * T + t] = -1;
            }
            __syncwarp();
            if (lane < ns) {
                const int t = lane / k;
                s_us[u * T + t] = lane;
                s_uw[u * T + t] = s_w[lane];
            }
            if (lane == 0) *s_nu = __popc(leads);
        }
        __syncthreads();
        const int U = *s_nu;
        const int nds = min(U + 1, S.nslot);  // slots in use: the shared expert, then u = 0 .. nds - 2
        if (threadIdx.x == 0 && nrows > 0) {
            // phase C's routed down rows do not depend on h: the first ones into the slots,
            // the others' rows into L2
            for (int u = 0; u < U; ++u) {
                const int e = s_ue[u];
                const char* wd = static_cast<const char*>(Ly.w_down) + size_t(e) * H * drow;
                const uint16_t* sd = PACKED ? Ly.s_down + size_t(e) * H * (I / 32) : nullptr;
                if (u + 1 < nds) {
                    issue_down(u + 1, wd, sd);
                } else {
                    prefetch_l2(wd + size_t(r0) * drow, uint64_t(nrows) * drow);
                    if (PACKED) prefetch_l2(reinterpret_cast<const char*>(sd) + size_t(r0) * dsc, uint64_t(nrows) * dsc);
                }
            }
        }
        {
            uint32_t xp[T][32];
            // (past the grid barrier: the layer's x is published whichever way it came; the
            // staged x is written in this launch, hence coherent loads)
            load_xp<WT, T, XR>(x, H, lane, xp);
            constexpr int G = (WT == DT_BF16) ? 1 : (T == 2 ? 3 : 2);
            const int J = U * I;
            const int gw = blockIdx.x * D1_WARPS + warp;
            for (int jb = gw; jb < J; jb += G * Wtot) {
                Row g[G], u[G];
#pragma unroll
                for (int t = 0; t < G; ++t) {
                    const int j = jb + t * Wtot;
                    if (j < J) {
                        const int uu = j / I, i = j - uu * I;
                        const size_t rowi = size_t(s_ue[uu]) * I + i;
                        ld_row<WT>(g[t], static_cast<const char*>(Ly.w_gate) + rowi * grow,
                                   PACKED ? Ly.s_gate + rowi * (H / 32) : nullptr, H, lane);
                        ld_row<WT>(u[t], static_cast<const char*>(Ly.w_up) + rowi * grow,
                                   PACKED ? Ly.s_up + rowi * (H / 32) : nullptr, H, lane);
                    }
                }
#pragma unroll
                for (int t = 0; t < G; ++t) {
                    const int j = jb + t * Wtot;
                    if (j < J) {
                        const int uu = j / I, i = j - uu * I;
                        const unsigned mask = unsigned(s_um[uu]);
                        float2 a[T], b[T];
#pragma unroll
                        for (int tt = 0; tt < T; ++tt) a[tt] = b[tt] = make_float2(0.f, 0.f);
                        dotT<WT, T>(g[t], xp, mask, a);
                        dotT<WT, T>(u[t], xp, mask, b);
#pragma unroll
                        for (int tt = 0; tt < T; ++tt) {
                            if (mask >> tt & 1u) {
                                const float av = hsum_fr(a[tt]), bv = hsum_fr(b[tt]);
                                if (lane == 0) p.hrt[size_t(s_us[uu * T + tt]) * I + hpos<WT>(i)] = silu_mul(av, bv);
                            }
                        }
                    }
                }
            }
        }
        grid_barrier(p.ctl, nblocks, bar_idx++, to);
        if constexpr (XR && NL > 1 && 4 * T <= D1_WARPS) {
            // the next stacked layer's x, fetched ahead by the last block (at the Qwen3-Next
            // size it has no output rows, hence no phase-C work), one quarter row per warp:
            // every block's phase-B reads of this layer's staged x are behind the barrier
            if (blockIdx.x == nblocks - 1 && warp < 4 * T && l + 1 < p.n_layers)
                fetch_host_quarter(static_cast<const uint4*>(p.L[l + 1].x) + size_t(warp >> 2) * (H / 8),
                                   reinterpret_cast<uint4*>(p.xstage) + size_t(warp >> 2) * (H / 8), warp & 3, H, lane,
                                   &p.ctl->x_ready);
        }

        // ------------------------------------------------------------ phase C
        if (l + 1 < p.n_layers && threadIdx.x < 32) {
            const DecLayer& Nx = p.L[l + 1];
            for (int q = lane * nblocks + blockIdx.x; q < E; q += 32 * nblocks)
                prefetch_l2(static_cast<const char*>(Nx.router_w) + size_t(q) * 2 * H, 2 * H);
            for (int i = lane * nblocks + blockIdx.x; i < I; i += 32 * nblocks) {
                prefetch_l2(static_cast<const char*>(Nx.sh_gate) + size_t(i) * grow, grow);
                prefetch_l2(static_cast<const char*>(Nx.sh_up) + size_t(i) * grow, grow);
            }
        }
        if (nrows > 0) {
            if (threadIdx.x == 0) {
                // the routed h rows (written by every block before the barrier), one bulk copy
                fence_proxy_async_global();
                fence_proxy_async_smem();
                mbar_arrive_expect_tx(hbar, uint32_t(4 * T * k * I));
                bulk_g2s(smem + S.hbuf, p.hrt, uint32_t(4 * T * k * I), hbar);
            }
        }
        // the launch's last barrier: count the block out (after the h copy is on its way)
        if (l + 1 == p.n_layers) grid_release(p.ctl, nblocks);
        if (nrows > 0) mbar_wait(hbar, par, err, to);
        float2 acc[D1_RB_MAX / 2][T];
#pragma unroll
        for (int r = 0; r < D1_RB_MAX / 2; ++r)
#pragma unroll
            for (int t = 0; t < T; ++t) acc[r][t] = make_float2(0.f, 0.f);
        if (nrows > 0) {
#pragma unroll 1
            for (int unit = warp; unit < 2 * U; unit += D1_WARPS) {
                const int u = unit >> 1;
                const unsigned mask = unsigned(s_um[u]);
                float wt[T];
                const float* hv[T];
#pragma unroll
                for (int t = 0; t < T; ++t) {
                    const int si = s_us[u * T + t];
                    wt[t] = si >= 0 ? s_uw[u * T + t] : 0.0f;
                    hv[t] = hbuf + size_t(si >= 0 ? si : 0) * I;
                }
                if (u + 1 < nds) {
                    mbar_wait(dbar + u + 1, par, err, to);
                    const unsigned char* slot = dreg + (u + 1) * S.slot;
                    unit_dots(acc, slot, slot + S.sc_off, drow, dsc, mask, wt, hv, false);
                } else {
                    // not in a slot: the block's rows straight from global memory (L2)
                    const int e = s_ue[u];
                    const unsigned char* rows = static_cast<const unsigned char*>(Ly.w_down) + (size_t(e) * H + r0) * drow;
                    const unsigned char* scl = PACKED ? reinterpret_cast<const unsigned char*>(Ly.s_down + (size_t(e) * H + r0) * (I / 32))
                                                      : nullptr;
                    unit_dots(acc, rows, scl, drow, dsc, mask, wt, hv, false);
                }
            }
        }
        // per row and token: reduce the lanes, then sum the warps' partials in a fixed order
#pragma unroll
        for (int r = 0; r < D1_RB_MAX / 2; ++r) {
#pragma unroll
            for (int t = 0; t < T; ++t) {
                const float v = warp_sum(acc[r][t].x + acc[r][t].y);
                if (lane == 0 && r < rn) part[(warp * D1_RB_MAX + ra + r) * T + t] = v;
            }
        }
        __syncthreads();
        for (int i = threadIdx.x; i < nrows * T; i += D1_THREADS) {
            const int r = i / T, t = i - (i / T) * T, hf = r >= half ? 1 : 0;
            float o = psh[r * T + t];  // the shared expert first, then the warps in order
            for (int w = hf; w < D1_WARPS; w += 2) o += part[(w * D1_RB_MAX + r) * T + t];
            Ly.out[size_t(t) * H + r0 + r] = o;
        }
        if (l + 1 < p.n_layers) grid_barrier(p.ctl, nblocks, bar_idx++, to);
    }
}

int fr_blocks_per_sm(const void* kern, int smem) {
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

template <int WT, int T, int NL, bool XR>
redmoe_status fr_launch(const redmoe_layer* sh, const DecLayer* layers, int n_layers, void* ws, cudaStream_t stream,
                        CacheBias cb, void* xstage) {
    DevInfo di;
    if (!get_dev_info(&di)) return REDMOE_ERR_CUDA;
    const int RB = (sh->hidden + di.sm_count - 1) / di.sm_count;
    if (RB > D1_RB_MAX) return REDMOE_ERR_UNSUPPORTED;
    const int max_smem = di.max_smem_optin;
    const FrSmem S = fr_smem(WT, T, sh->top_k, sh->inter, RB, max_smem);
    if (S.nslot < 1 || S.total > max_smem) return REDMOE_ERR_UNSUPPORTED;
    auto kern = decodefr_kernel<WT, T, NL, XR>;
    const int per_sm = fr_blocks_per_sm(reinterpret_cast<const void*>(kern), S.total);
    if (per_sm < 0) return REDMOE_ERR_CUDA;
    if (per_sm == 0) return REDMOE_ERR_UNSUPPORTED;
    FrParams<NL>* pp = new (std::nothrow) FrParams<NL>();
    if (!pp) return REDMOE_ERR_CUDA;
    FrParams<NL>& q = *pp;
    q.H = sh->hidden; q.E = sh->n_experts; q.k = sh->top_k; q.I = sh->inter;
    q.n_layers = n_layers;
    q.RB = RB;
    q.max_smem = max_smem;
    const DecodeWs L = decode_ws_layout(T, q.E, q.k, q.I, sh->shared_inter);
    char* base = static_cast<char*>(ws);
    q.ctl = reinterpret_cast<Control*>(base);
    q.logits = reinterpret_cast<float*>(base + L.logits);
    q.sgate = reinterpret_cast<float*>(base + L.sgate);
    q.hsh = reinterpret_cast<float*>(base + L.hsh);
    q.hrt = reinterpret_cast<float*>(base + L.hrt);
    q.timeout_ns = BARRIER_TIMEOUT_NS;
    q.cb = cb;
    q.xstage = static_cast<uint16_t*>(xstage);
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

template <int WT, int T, bool XR>
redmoe_status fr_launch_all(const redmoe_layer* sh, const DecLayer* layers, int n_layers, void* ws, cudaStream_t stream,
                            int* launches, CacheBias cb, void* xstage) {
    redmoe_status st = REDMOE_OK;
    if (n_layers == 1) {
        st = fr_launch<WT, T, 1, XR>(sh, layers, 1, ws, stream, cb, xstage);
        if (st == REDMOE_OK && launches) *launches += 1;
        return st;
    }
    for (int l0 = 0; l0 < n_layers && st == REDMOE_OK; l0 += MAX_STACK) {
        const int n = n_layers - l0 < MAX_STACK ? n_layers - l0 : MAX_STACK;
        st = fr_launch<WT, T, MAX_STACK, XR>(sh, layers + l0, n, ws, stream, cb, xstage);
        if (st == REDMOE_OK && launches) *launches += 1;
    }
    return st;
}

template <int WT>
redmoe_status fr_launch_t(const redmoe_layer* sh, const DecLayer* layers, int n_layers, int T, void* ws,
                          cudaStream_t stream, int* launches, CacheBias cb) {
    switch (T) {
        case 2: return fr_launch_all<WT, 2, false>(sh, layers, n_layers, ws, stream, launches, cb, nullptr);
        case 3: return fr_launch_all<WT, 3, false>(sh, layers, n_layers, ws, stream, launches, cb, nullptr);
        default: return REDMOE_ERR_UNSUPPORTED;
    }
}

}  // namespace

// Layers the few-row kernel takes: those of the one-row kernel with bf16 or int4 experts,
// at 2 token rows (T * k <= 32, so that one warp finds the distinct experts). The kernel
// is written for T = 2 and 3.
bool decodefr_shape_ok(const redmoe_layer* sh, int T) {
    // T = 3 measured slower here than on the ring kernel (111 against 82 us per bf16 call:
    // 19 of its 29 distinct experts' down rows miss the shared-memory slots), so the
    // dispatch sends only T = 2 to this kernel
    if (T != 2 || T * sh->top_k > 32) return false;
    if (sh->expert_dtype != DT_BF16 && sh->expert_dtype != DT_INT4) return false;
    return decode1_shape_ok(sh);
}

redmoe_status launch_decodefr(const redmoe_layer* sh, const DecLayer* layers, int n_layers, int T, void* ws,
                              cudaStream_t stream, int* launches, CacheBias cb) {
    if (sh->expert_dtype == DT_INT4) return fr_launch_t<DT_INT4>(sh, layers, n_layers, T, ws, stream, launches, cb);
    return fr_launch_t<DT_BF16>(sh, layers, n_layers, T, ws, stream, launches, cb);
}

redmoe_status launch_decodefr_host_x(const redmoe_layer* sh, const DecLayer* layers, int n_layers, int T, void* ws,
                                     void* xstage, cudaStream_t stream) {
    const CacheBias cb{nullptr, 0.0f};
    if (T != 2) return REDMOE_ERR_UNSUPPORTED;  // the host-memory x instantiations are built for T = 2
    if (sh->expert_dtype == DT_INT4)
        return fr_launch_all<DT_INT4, 2, true>(sh, layers, n_layers, ws, stream, nullptr, cb, xstage);
    return fr_launch_all<DT_BF16, 2, true>(sh, layers, n_layers, ws, stream, nullptr, cb, xstage);
}

}  // namespace redmoe
