// Decode path for one token row (T = 1) with bf16 or int4 group-32 experts: one
// persistent cooperative kernel per call (or per stack of layers).
//
// At T = 1 a layer is a pure stream: every weight byte the token needs is read once from
// HBM and used for one multiply-add. What costs time is not arithmetic but the three
// dependent steps (router -> routed gate/up -> down) and how fast each one reaches full
// bandwidth. This kernel is organised around that:
//
//   * x is bulk-copied into shared memory once per layer; every lane keeps its slice in
//     registers as fp32 while it streams rows, so a weight chunk is dotted straight out of
//     the registers it was loaded into: no shared-memory traffic for gate/up weights.
//   * Phase A: warps stream the router rows and the shared-gate row with 16-byte vector
//     loads, and nothing else: they are all that stands between the launch and the top-k.
//     Meanwhile one thread per block starts a bulk copy of the block's rows of the shared
//     expert's down matrix into shared memory.
//   * Split grid barrier: each block publishes its logits (arrive); then warps 1..7
//     stream the block's share of the shared expert's gate/up rows (the shared expert
//     needs no routing: the "extra slot" of the DwarfStar MoE kernel, "Research notes,
//     October 2026", section 1) while warp 0 alone waits for the other blocks.
//   * Warp 0 computes the top-k of the 512 logits in registers (router, top-k and shared
//     gate form one stage: same section). Then one thread per block starts bulk
//     copies of the block's rows of the k routed experts' down matrices: phase C's weights
//     stream into shared memory during phase B, since they do not depend on h.
//   * Phase B: the k * I routed gate/up row pairs, interleaved over all warps; bf16 warps
//     keep two pairs of loads in flight, int4/int2 warps issue all of theirs at once;
//     h = silu(a) * u.
//   * Grid barrier; the routed and shared h rows are bulk-copied into shared memory and
//     phase C computes the block's output rows from the down rows already there (the
//     shared expert is slot k). Each output row is summed over the experts in a fixed
//     order: the result is deterministic.
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
#include "rowdot.cuh"
#include "topk.cuh"

namespace redmoe {

namespace {

__device__ __forceinline__ float hsum2(float2 v) { return warp_sum(v.x + v.y); }

// Shared-memory plan of the kernel (byte offsets). `dreg` holds the block's rows of the
// down matrix of k + 1 experts (routed slots 0..k-1 in selection order, the shared
// expert in slot k), each slot RB rows (int4: codes, then scales).
struct D1Smem {
    int dreg, slot, sc_off, hbuf, xs, bars, part, sel, total;
};
__host__ __device__ inline D1Smem d1_smem(int wt, int k, int I, int RB, int H) {
    D1Smem s;
    const int drow = d1_row_bytes(wt, I);
    s.sc_off = a16(RB * drow);
    s.slot = a16(s.sc_off + RB * d1_scale_bytes(wt, I));
    int o = 0;
    s.dreg = o; o += (k + 1) * s.slot;
    s.hbuf = o; o += a16(4 * (k + 1) * I);  // the routed and the shared h rows, staged for phase C
    s.xs = o; o += a16(2 * H);  // the layer's x (bf16), one bulk copy per layer
    s.bars = o; o += 8 * (D1_MAXK + 3);
    s.part = o; o += 4 * D1_WARPS * D1_RB_MAX;
    s.sel = o; o += 12 * D1_MAXK + 4;  // the block's top-k: ids, weights, stack indices; the shared gate
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
    // non-null: every layer's x is pinned host memory (its device mapping in L[l].x); at
    // the start of each layer block 0 copies it here and counts on Control::x_ready, and
    // every block reads it from here (one buffer: the barrier between stacked layers keeps
    // a layer's copy from overwriting x that another block still reads)
    uint16_t* xstage;
    DecLayer L[NL];
};

// x of one layer from pinned host memory into the workspace copy `xstage`, by warps 4..7
// of one block (warps without a router row): each reads a quarter of x once over the link
// with cache-volatile loads (the host rewrites it between calls), every load of a lane
// issued before its first store so that the copy costs one link round trip, then counts
// itself on x_ready with a release.
__device__ __forceinline__ void fetch_host_x(const void* x, uint16_t* xstage, unsigned* x_ready, int H, int warp,
                                             int lane) {
    constexpr int PER = D1_XPL / 32;  // 16-byte chunks per lane: a quarter of x per warp
    const uint4* src = static_cast<const uint4*>(x);
    uint4* dst = reinterpret_cast<uint4*>(xstage);
    const int c0 = (warp - 4) * 32 * PER + lane;
    uint4 v[PER];
#pragma unroll
    for (int j = 0; j < PER; ++j)
        if (c0 + 32 * j < H / 8) v[j] = __ldcv(src + c0 + 32 * j);
#pragma unroll
    for (int j = 0; j < PER; ++j)
        if (c0 + 32 * j < H / 8) dst[c0 + 32 * j] = v[j];
    __threadfence();
    __syncwarp();
    if (lane == 0) asm volatile("red.release.gpu.global.add.u32 [%0], 1;" :: "l"(x_ready) : "memory");
}

// XR: every layer's x comes from pinned host memory through p.xstage (a separate
// instantiation, so that calls on device buffers carry none of that code).
template <int WT, int NL, bool XR>
__global__ void __launch_bounds__(D1_THREADS, 1) decode1_kernel(const __grid_constant__ D1Params<NL> p) {
    extern __shared__ __align__(128) unsigned char smem[];
    using Row = typename RowOf<WT>::type;
    const int H = p.H, E = p.E, k = p.k, I = p.I, RB = p.RB;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int nblocks = gridDim.x;
    const int Wtot = nblocks * D1_WARPS;
    int* err = &p.ctl->err;
    const uint64_t to = p.timeout_ns;
    const D1Smem S = d1_smem(WT, k, I, RB, H);
    unsigned char* dreg = smem + S.dreg;
    uint64_t* dbar = reinterpret_cast<uint64_t*>(smem + S.bars);
    uint64_t* hbar = dbar + D1_MAXK + 1;
    uint64_t* xbar = dbar + D1_MAXK + 2;
    const float* hbuf = reinterpret_cast<const float*>(smem + S.hbuf);
    float* part = reinterpret_cast<float*>(smem + S.part);
    int* s_sel_id = reinterpret_cast<int*>(smem + S.sel);
    float* s_sel_w = reinterpret_cast<float*>(smem + S.sel) + D1_MAXK;
    int* s_sel_slot = reinterpret_cast<int*>(smem + S.sel) + 2 * D1_MAXK;
    float* s_wsh = reinterpret_cast<float*>(smem + S.sel) + 3 * D1_MAXK;
    constexpr bool PACKED = WT != DT_BF16;           // int4 / int2: codes plus group scales
    const int drow = d1_row_bytes(WT, I);            // bytes of one down row (codes)
    const int dsc = d1_scale_bytes(WT, I);           // bytes of its scales
    const long grow = d1_row_bytes(WT, H);           // bytes of one gate/up row
    const int r0 = blockIdx.x * RB;
    const int nrows = max(0, min(RB, H - r0));
    unsigned bar_idx = 0;

    if (threadIdx.x == 0) {
        for (int i = 0; i <= k; ++i) mbar_init(dbar + i, 1);
        mbar_init(hbar, 1);
        mbar_init(xbar, 1);
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
        constexpr bool xremote = XR;
        if (xremote && (NL == 1 || l == 0) && blockIdx.x == 0 && warp >= 4) {
            // x from host memory, as in fetch_host_x: the first layer's is fetched by block 0
            // at the start of the launch, each later stacked layer's ahead of time (phase
            // C); written out here rather than called, which keeps the single-layer build's
            // registers as they were
            constexpr int PER = D1_XPL / 32;
            const uint4* src = reinterpret_cast<const uint4*>(x);
            uint4* dst = reinterpret_cast<uint4*>(p.xstage);
            const int c0 = (warp - 4) * 32 * PER + lane;
            uint4 v[PER];
#pragma unroll
            for (int j = 0; j < PER; ++j)
                if (c0 + 32 * j < H / 8) v[j] = __ldcv(src + c0 + 32 * j);
#pragma unroll
            for (int j = 0; j < PER; ++j)
                if (c0 + 32 * j < H / 8) dst[c0 + 32 * j] = v[j];
            __threadfence();
            __syncwarp();
            if (lane == 0) asm volatile("red.release.gpu.global.add.u32 [%0], 1;" :: "l"(&p.ctl->x_ready) : "memory");
        }
        if (threadIdx.x == (xremote ? 32 * (D1_WARPS - 1) : 0)) {
            // (with x in host memory an idle warp's lane waits for it, so that warp 0's
            // router row is not held up)
            const void* xsrc = x;
            if (xremote) {
                const uint64_t t0 = globaltimer_ns();
                for (uint32_t spins = 0; ld_acquire_gpu(&p.ctl->x_ready) < 4u * unsigned(l + 1); ++spins) {
                    if ((spins & 63u) == 63u && (globaltimer_ns() - t0 > to || spins > (1u << 26))) {
                        atomicOr(err, ERRBIT_TIMEOUT);
                        break;
                    }
                }
                fence_proxy_async_global();  // generic stores of block 0, read by the bulk copy
                xsrc = p.xstage;
            }
            fence_proxy_async_smem();  // the previous layer's reads of xs come first
            mbar_arrive_expect_tx(xbar, uint32_t(2 * H));
            bulk_g2s(smem + S.xs, xsrc, uint32_t(2 * H), xbar);
        }
        if (threadIdx.x == 0 && nrows > 0) {
            fence_proxy_async_smem();  // the previous layer's reads of dreg come first
            issue_down(k, Ly.sh_down, Ly.sh_s_down);
        }
        // job q < E: router row q; q == E: shared-gate row. Warp w of block b takes
        // q = w * nblocks + b: the jobs go to the low warps of every block. Only these rows
        // stand between the launch and the top-k, so nothing else is streamed before them.
        for (int q = warp * nblocks + blockIdx.x; q < E + 1; q += Wtot) {
            if (Ly.given_ids && q < E) continue;  // routing given: no router rows
            float xr[D1_XPL];
            RowBF r;
            const void* row = q < E ? static_cast<const void*>(static_cast<const char*>(Ly.router_w) + size_t(q) * 2 * H)
                                    : Ly.shared_gate_w;
            ld_row_bf(r, row, H, lane);
            mbar_wait(xbar, par, err, to);
            load_x<DT_BF16, true>(reinterpret_cast<const uint16_t*>(smem + S.xs), H, lane, xr);
            const float v = hsum2(dot_row_bf(r, xr));
            if (lane == 0) {
                if (q < E) p.logits[q] = v + (Ly.router_bias ? Ly.router_bias[q] : 0.0f);
                else *sgate = 1.0f / (1.0f + expf(-v));
            }
        }
        // the logits are published; while the other blocks finish theirs, warps 1..7 stream
        // the shared expert's gate/up rows (it needs no routing: the extra expert slot of the
        // DwarfStar MoE kernel) and warp 0 alone waits for the barrier, then takes the top-k.
        // Pair i goes to block i % nblocks; its slot i / nblocks (mod 7) picks the warp:
        // slots 0..3 are warps 4..7, which had no router row, slots 4..6 warps 1..3.
        grid_arrive(p.ctl);
        const unsigned bar1 = bar_idx++;
        const int shslot = warp >= 4 ? warp - 4 : (warp > 0 ? warp + 3 : -1);
        for (int i = shslot < 0 ? I : shslot * nblocks + blockIdx.x; i < I; i += 7 * nblocks) {
            float xr[D1_XPL];
            Row g, u;
            ld_row<WT>(g, static_cast<const char*>(Ly.sh_gate) + size_t(i) * grow,
                       PACKED ? Ly.sh_s_gate + size_t(i) * (H / 32) : nullptr, H, lane);
            ld_row<WT>(u, static_cast<const char*>(Ly.sh_up) + size_t(i) * grow,
                       PACKED ? Ly.sh_s_up + size_t(i) * (H / 32) : nullptr, H, lane);
            mbar_wait(xbar, par, err, to);
            load_x<WT, true>(reinterpret_cast<const uint16_t*>(smem + S.xs), H, lane, xr);
            const float a = hsum2(dot_row<WT>(g, xr)), b = hsum2(dot_row<WT>(u, xr));
            if (lane == 0) hsh[hpos<WT>(i)] = silu_mul(a, b);
        }

        // Phase C's work comes in units (slot u, half hf of the block's rows): 2 (k + 1)
        // units, slots 0 .. k-1 the routed experts and slot k the shared one (unit = warp +
        // 8 m, every unit of a warp has hf = warp & 1). Each warp accumulates its rows'
        // weighted partials in registers.
        constexpr int MU = (2 * (D1_MAXK + 1) + D1_WARPS - 1) / D1_WARPS;  // units per warp, at most
        const int half = (nrows + 1) / 2;
        const int ra = (warp & 1) * half, rn = nrows > 0 ? min(half, nrows - ra) : 0;
        float2 acc[D1_RB_MAX / 2];
        // weighted row dots of one unit: acc[r] += wu * (row ra + r of slot u) . h
        auto unit_dots = [&](int u, float wu, const float (&hf32)[D1_HPL]) {
            mbar_wait(dbar + u, par, err, to);
            const unsigned char* slot = dreg + u * S.slot;
#pragma unroll
            for (int r = 0; r < D1_RB_MAX / 2; ++r) {
                {
                    // rows past rn dot a valid row: no branch per row, the result is unused
                    const int rr = min(ra + r, nrows - 1);
                    float2 d = make_float2(0.f, 0.f);
                    if constexpr (WT == DT_INT2) {
                        const uint32_t wv = *reinterpret_cast<const uint32_t*>(slot + rr * drow + lane * 4);
                        const float s = bf16f(*reinterpret_cast<const uint16_t*>(slot + S.sc_off + rr * dsc + (lane >> 1) * 2));
                        d = ffma2(make_float2(s, s), dot16_q2(wv, hf32), d);
                    } else if constexpr (WT == DT_INT4) {
                        const uint2 wv = *reinterpret_cast<const uint2*>(slot + rr * drow + lane * 8);
                        const float s = bf16f(*reinterpret_cast<const uint16_t*>(slot + S.sc_off + rr * dsc + (lane >> 1) * 2));
                        const float2 a = dot8_q4(wv.x, hf32, make_float2(0.f, 0.f));
                        const float2 b = dot8_q4(wv.y, hf32 + 8, make_float2(0.f, 0.f));
                        d = ffma2(make_float2(s, s), fadd2(a, b), d);
                    } else {
                        const unsigned char* wr = slot + rr * drow + lane * 16;
                        const uint4 w0 = *reinterpret_cast<const uint4*>(wr);
                        const uint4 w1 = *reinterpret_cast<const uint4*>(wr + 512);
                        float2 e = make_float2(0.f, 0.f);
                        d = ffma2(bf2(w0.x), make_float2(hf32[0], hf32[1]), d);
                        e = ffma2(bf2(w0.y), make_float2(hf32[2], hf32[3]), e);
                        d = ffma2(bf2(w0.z), make_float2(hf32[4], hf32[5]), d);
                        e = ffma2(bf2(w0.w), make_float2(hf32[6], hf32[7]), e);
                        d = ffma2(bf2(w1.x), make_float2(hf32[8], hf32[9]), d);
                        e = ffma2(bf2(w1.y), make_float2(hf32[10], hf32[11]), e);
                        d = ffma2(bf2(w1.z), make_float2(hf32[12], hf32[13]), d);
                        e = ffma2(bf2(w1.w), make_float2(hf32[14], hf32[15]), e);
                        d = fadd2(d, e);
                    }
                    acc[r] = ffma2(make_float2(wu, wu), d, acc[r]);
                }
            }
        };
        // ------------------------------------------------------------ phase B
        if (warp == 0) {
            // one warp per block takes the top-k of the logits (lane j < k: id and
            // renormalised weight of selection j) and shares it
            grid_wait_warp(p.ctl, nblocks, bar1, to);
            const float sg = __ldcg(sgate);  // the shared expert's gate, read beside the logits
            int id = 0;
            float wv = 0.0f;
            if (Ly.given_ids) {
                if (lane < k) {
                    id = __ldcg(Ly.given_ids + lane);
                    wv = __ldcg(Ly.given_w + lane);
                }
            } else {
                warp_route<D1_MAXE / 32>(p.logits, E, k, p.cb.cached, p.cb.lambda, id, wv);
            }
            if (lane < k) {
                int slot = id;
                if (Ly.slot_of) {
                    slot = __ldcg(Ly.slot_of + id);
                    if (slot < 0) {  // not resident: a caller error; read slot 0 and report it
                        atomicOr(err, ERRBIT_STATE);
                        slot = 0;
                    }
                }
                s_sel_id[lane] = id;
                s_sel_w[lane] = wv;
                s_sel_slot[lane] = slot;
                if (lane == 0) *s_wsh = sg;
                if (blockIdx.x == 0) {
                    Ly.ids[lane] = id;
                    Ly.w[lane] = wv;
                }
            }
        }
        __syncthreads();
#pragma unroll
        for (int r = 0; r < D1_RB_MAX / 2; ++r) acc[r] = make_float2(0.f, 0.f);
        // x in the layout of the expert weights (from the shared copy: no memory latency)
        float xf[D1_XPL];
        mbar_wait(xbar, par, err, to);
        load_x<WT, true>(reinterpret_cast<const uint16_t*>(smem + S.xs), H, lane, xf);
        const int sel_id = lane < k ? s_sel_slot[lane] : 0;  // stack index of selection j
        const float sel_w = lane < k ? s_sel_w[lane] : 0.0f;
        if (warp == 0 && nrows > 0) {
            // phase C's routed down rows do not depend on h: start their copies now
            for (int j = 0; j < k; ++j) {
                const int e = __shfl_sync(FULL, sel_id, j);
                if (lane == 0)
                    issue_down(j, static_cast<const char*>(Ly.w_down) + size_t(e) * H * drow,
                               PACKED ? Ly.s_down + size_t(e) * H * (I / 32) : nullptr);
            }
        }
        // the k * I routed gate/up row pairs (u-major)
        const int J = k * I;
        auto job_rows = [&](int j, Row& g, Row& u) {
            const int uu = j / I, i = j - (j / I) * I;
            const int e = __shfl_sync(FULL, sel_id, uu < k ? uu : 0);
            if (j < J) {
                const size_t rowi = size_t(e) * I + i;
                ld_row<WT>(g, static_cast<const char*>(Ly.w_gate) + rowi * grow,
                           PACKED ? Ly.s_gate + rowi * (H / 32) : nullptr, H, lane);
                ld_row<WT>(u, static_cast<const char*>(Ly.w_up) + rowi * grow,
                           PACKED ? Ly.s_up + rowi * (H / 32) : nullptr, H, lane);
            }
        };
        {
            // each warp takes the pairs j = gw, gw + Wtot, ... and keeps G of them in flight
            // (bf16 rows are 4 KB: 2 pairs; packed rows are 1 KB int4 or 512 B int2: all of a
            // warp's pairs at the Qwen3-Next size, so one memory latency covers them)
            constexpr int G = WT == DT_BF16 ? D1_G : D1_GQ;
            const int gw = blockIdx.x * D1_WARPS + warp;
            for (int jb = gw; jb < J; jb += G * Wtot) {
                Row g[G], u[G];
#pragma unroll
                for (int t = 0; t < G; ++t) job_rows(jb + t * Wtot, g[t], u[t]);
#pragma unroll
                for (int t = 0; t < G; ++t) {
                    const int j = jb + t * Wtot;
                    if (j < J) {
                        const float a = hsum2(dot_row<WT>(g[t], xf)), b = hsum2(dot_row<WT>(u[t], xf));
                        if (lane == 0) p.hrt[j - (j % I) + hpos<WT>(j % I)] = silu_mul(a, b);
                    }
                }
            }
        }

        // ------------------------------------------------------------ phase C
        grid_barrier(p.ctl, nblocks, bar_idx++, to);
        if constexpr (NL > 1) {
            // the next stacked layer's x, fetched ahead by the last block (at the Qwen3-Next
            // size it has no output rows, hence no phase-C work): every block copied this
            // layer's staged x before the first barrier, so it may be overwritten now
            if (XR && blockIdx.x == nblocks - 1 && warp >= 4 && l + 1 < p.n_layers)
                fetch_host_x(p.L[l + 1].x, p.xstage, &p.ctl->x_ready, H, warp, lane);
        }
        if (nrows > 0 && threadIdx.x == 0) {
            // the routed and the shared h rows (written by every block before the barrier)
            // into shared memory, two bulk copies
            fence_proxy_async_global();
            fence_proxy_async_smem();
            mbar_arrive_expect_tx(hbar, uint32_t(4 * (k + 1) * I));
            bulk_g2s(smem + S.hbuf, p.hrt, uint32_t(4 * k * I), hbar);
            bulk_g2s(smem + S.hbuf + 4 * k * I, hsh, uint32_t(4 * I), hbar);
        }
        // the launch's last barrier: count the block out (after the h copies are on their way)
        if (l + 1 == p.n_layers) grid_release(p.ctl, nblocks);
        if (l + 1 < p.n_layers && threadIdx.x < 32) {
            // L2 prefetch of the next layer's router rows and shared gate/up rows (the rows
            // this block streams first in that layer)
            const DecLayer& Nx = p.L[l + 1];
            for (int q = lane * nblocks + blockIdx.x; q < E; q += 32 * nblocks)
                prefetch_l2(static_cast<const char*>(Nx.router_w) + size_t(q) * 2 * H, 2 * H);
            for (int i = lane * nblocks + blockIdx.x; i < I; i += 32 * nblocks) {
                prefetch_l2(static_cast<const char*>(Nx.sh_gate) + size_t(i) * grow, grow);
                prefetch_l2(static_cast<const char*>(Nx.sh_up) + size_t(i) * grow, grow);
            }
        }
        if (nrows > 0) {
            mbar_wait(hbar, par, err, to);
            const float wsh = *s_wsh;
#pragma unroll 1
            for (int m = 0; m < MU; ++m) {
                const int unit = warp + D1_WARPS * m;
                if (unit < 2 * (k + 1)) {
                    const int u = unit >> 1;
                    float hh[D1_HPL];
                    const float4* hv = reinterpret_cast<const float4*>(hbuf + size_t(u) * I) + lane;
#pragma unroll
                    for (int i = 0; i < D1_HPL / 4; ++i) {
                        const float4 v = hv[32 * i];
                        hh[4 * i] = v.x; hh[4 * i + 1] = v.y; hh[4 * i + 2] = v.z; hh[4 * i + 3] = v.w;
                    }
                    const float wr = __shfl_sync(FULL, sel_w, u < k ? u : 0);
                    unit_dots(u, u < k ? wr : wsh, hh);
                }
            }
        }
        // per row: reduce the lanes, then sum the warps' partials in a fixed order
#pragma unroll
        for (int r = 0; r < D1_RB_MAX / 2; ++r) {
            const float v = warp_sum(acc[r].x + acc[r].y);
            if (lane == 0 && r < rn) part[warp * D1_RB_MAX + ra + r] = v;
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

template <int WT, int NL, bool XR>
redmoe_status d1_launch(const redmoe_layer* sh, const DecLayer* layers, int n_layers, void* ws, cudaStream_t stream,
                        CacheBias cb, void* xstage) {
    DevInfo di;
    if (!get_dev_info(&di)) return REDMOE_ERR_CUDA;
    const int RB = (sh->hidden + di.sm_count - 1) / di.sm_count;
    if (RB > D1_RB_MAX) return REDMOE_ERR_UNSUPPORTED;
    const D1Smem S = d1_smem(WT, sh->top_k, sh->inter, RB, sh->hidden);
    if (S.total > di.max_smem_optin) return REDMOE_ERR_UNSUPPORTED;
    auto kern = decode1_kernel<WT, NL, XR>;
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

template <int WT, bool XR = false>
redmoe_status d1_launch_all(const redmoe_layer* sh, const DecLayer* layers, int n_layers, void* ws, cudaStream_t stream,
                            int* launches, CacheBias cb, void* xstage = nullptr) {
    redmoe_status st = REDMOE_OK;
    if (n_layers == 1) {
        st = d1_launch<WT, 1, XR>(sh, layers, 1, ws, stream, cb, xstage);
        if (st == REDMOE_OK && launches) *launches += 1;
        return st;
    }
    for (int l0 = 0; l0 < n_layers && st == REDMOE_OK; l0 += MAX_STACK) {
        const int n = n_layers - l0 < MAX_STACK ? n_layers - l0 : MAX_STACK;
        st = d1_launch<WT, MAX_STACK, XR>(sh, layers + l0, n, ws, stream, cb, xstage);
        if (st == REDMOE_OK && launches) *launches += 1;
    }
    return st;
}

}  // namespace

// Layers the one-row kernel takes: bf16 x and router, bf16, int4 or int2 experts, the
// Qwen3-Next expert width (I = Is = 512), H up to 2048 in whole chunks per lane, at most
// D1_MAXE experts and D1_MAXK per token, and at most D1_RB_MAX output rows per block.
bool decode1_shape_ok(const redmoe_layer* sh) {
    const int H = sh->hidden, wt = sh->expert_dtype;
    if (sh->x_dtype != DT_BF16 || sh->router_dtype != DT_BF16) return false;
    if (sh->inter != 512 || sh->shared_inter != 512) return false;
    if (wt != DT_BF16 && wt != DT_INT4 && wt != DT_INT2) return false;
    if (H > 32 * D1_XPL || H % (wt == DT_INT2 ? 2048 : (wt == DT_INT4 ? 1024 : 256))) return false;
    if (sh->top_k > D1_MAXK || sh->n_experts > D1_MAXE) return false;
    return true;
}

redmoe_status launch_decode1(const redmoe_layer* sh, const DecLayer* layers, int n_layers, void* ws,
                             cudaStream_t stream, int* launches, CacheBias cb) {
    if (sh->expert_dtype == DT_INT4) return d1_launch_all<DT_INT4>(sh, layers, n_layers, ws, stream, launches, cb);
    if (sh->expert_dtype == DT_INT2) return d1_launch_all<DT_INT2>(sh, layers, n_layers, ws, stream, launches, cb);
    return d1_launch_all<DT_BF16>(sh, layers, n_layers, ws, stream, launches, cb);
}

redmoe_status launch_decode1_host_x(const redmoe_layer* sh, const DecLayer* layers, int n_layers, void* ws,
                                    void* xstage, cudaStream_t stream) {
    const CacheBias cb{nullptr, 0.0f};
    if (sh->expert_dtype == DT_INT4) return d1_launch_all<DT_INT4, true>(sh, layers, n_layers, ws, stream, nullptr, cb, xstage);
    if (sh->expert_dtype == DT_INT2) return d1_launch_all<DT_INT2, true>(sh, layers, n_layers, ws, stream, nullptr, cb, xstage);
    return d1_launch_all<DT_BF16, true>(sh, layers, n_layers, ws, stream, nullptr, cb, xstage);
}

}  // namespace redmoe
