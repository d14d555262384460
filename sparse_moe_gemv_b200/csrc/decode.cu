// Decode path (1..4 token rows): one persistent cooperative kernel per call.
//
// A layer at decode size is a bandwidth problem: every routed expert row is read once
// from HBM and dotted with 1..4 activation rows. The kernel streams the layer in three
// phases separated by grid barriers, with every block of the grid resident:
//
//   A  router logits (E rows of Wr), the shared gate (row g) and the shared expert's
//      gate/up rows with SwiGLU (the shared expert needs no routing, so it overlaps
//      the router, like the "extra slot" of the DwarfStar MoE kernel in "Research
//      notes, October 2026", section 1).
//   B  every block computes the top-k of every token from the logits (a warp per
//      token), the renormalised weights and the list of distinct experts, then streams
//      the routed gate/up rows and writes h = silu(a) * u.
//   C  each warp owns two output rows: it sums weight * (Wd[n, :] . h) over every
//      distinct expert and the shared expert and writes out[t, n] once (the weighted
//      combine happens in registers, deterministically, with no atomics).
//
// Weight bytes move with 1-D bulk copies (cp.async.bulk, completion on an mbarrier): each
// warp owns a ring of 3-5 stages of 4 KiB (phases A and B add the stages that fit the h
// buffer, idle until phase C) and keeps them in flight while it computes on the oldest, so
// a few instructions keep 100-200 KB per SM in flight. bf16 activations are widened to fp32
// in shared memory once per layer (T <= 3) for the dots. Compute
// reads the staged rows from shared memory with conflict-free 16-byte accesses ("pieces":
// 16 bytes of activations and the weight bytes that multiply them), in short rolled
// loops: at this size the cost is latency and instruction fetch, not arithmetic. The first
// stages of phase C (whose weights do not depend on h) are issued before the barrier that
// precedes it. (Prefetching all of phase C's rows into L2 during phase B measured slower at
// T = 1: the prefetch competes with the gate/up stream for HBM.)
//
// Down rows are only 512 elements long (1 KiB in bf16, 256 B in int4): a phase-C stage
// holds two rows of one expert, the lesson of the narrow-row kernel in "Research notes,
// October 2026", section 4 ("Narrow-row IQ mul_mv", 512-column expert down rows).
#include <mutex>
#include <new>
#include <vector>

#include "common.cuh"
#include "gemv.cuh"
#include "internal.h"
#include "topk.cuh"

namespace redmoe {

namespace {

constexpr int THREADS = 256;
constexpr int WARPS = THREADS / 32;
constexpr int SB = 4096 + 256;  // stage bytes: a 4 KiB weight segment plus int4 scales
constexpr int SEG_MAX = 4096;   // largest single weight segment
constexpr int RQ_MAX = 8;       // phase-C rows per stage, at most
constexpr int MAX_SLOTS = DECODE_MAX_T * MAX_TOPK;
static_assert(MAX_SLOTS <= THREADS, "one thread per routed slot");

// Stages per warp ring in phase C; phases A and B add the stages that fit the h buffer,
// which is idle until phase C (up to NS_MAX).
template <int T> struct Stages { static constexpr int NS = (T == 1) ? 5 : ((T == 2) ? 4 : 3); };
constexpr int NS_MAX = 8;

__host__ __device__ constexpr int align16(int x) { return (x + 15) & ~15; }
__host__ __device__ constexpr int align128(int x) { return (x + 127) & ~127; }
// int4 scale bytes of a K-element row (one bf16 per 32 elements)
__host__ __device__ constexpr int scale_bytes(int wt, int K) { return wt == DT_INT4 ? K / 16 : 0; }

struct Smem {
    int ring, xs, xf, hs, bars, keys, ids, wts, first, uidx, wcnt, ue, umask, uslot, uw, sg, nu, part, jobq, total;
    int nsb;  // ring depth of phases A and B
};

// bf16 activations are widened to fp32 once per layer (xf) when T <= 3, so that the many
// weight rows dotted with them do not each convert them again; at T = 4 the fp32 copy does
// not fit next to the stage ring, and the dots read the bf16 activations.
template <int XT, int T>
struct XWide {
    static constexpr bool on = XT == DT_BF16 && T <= 3;
    static constexpr int vt = on ? DT_F32 : XT;  // activation type the dots read
};

__host__ __device__ inline Smem smem_layout(int T, int NS, int H, int E, int k, int I, int Is, int xt, int RB,
                                            bool xwide) {
    Smem s;
    int o = 0;
    s.ring = o; o += WARPS * NS * SB;
    s.xs = o; o = align128(o + T * H * vbytes(xt));
    s.xf = o; o = align128(o + (xwide ? T * H * 4 : 0));
    s.hs = o; o = align128(o + 4 * (T * k * I + T * Is));
    s.nsb = NS + (4 * (T * k * I + T * Is)) / (WARPS * SB);
    if (s.nsb > NS_MAX) s.nsb = NS_MAX;
    s.bars = o; o += 8 * (WARPS * NS_MAX + 2);
    // phase-B scratch (keys, first) and phase-C scratch (part) share one region
    s.keys = o;
    s.first = o + 4 * T * E;
    s.part = o;
    o += (4 * T * E + 4 * E > 4 * WARPS * RB * T) ? 4 * T * E + 4 * E : 4 * WARPS * RB * T;
    s.ids = o; o += 4 * T * k;
    s.wts = o; o += 4 * T * k;
    s.uidx = o; o += 4 * T * k;
    s.wcnt = o; o += 4 * (MAX_SLOTS / 32);
    s.ue = o; o += 4 * T * k;
    s.umask = o; o += 4 * T * k;
    s.uslot = o; o += 4 * T * k * T;
    s.uw = o; o += 4 * T * k * T;
    s.sg = o; o += 4 * T;
    s.nu = o; o += 16;
    s.jobq = o; o += 4 * WARPS * 8;
    s.total = align128(o);
    return s;
}

// ------------------------------------------------------------ staged dots
// acc[t] += row . v_t for one row of K elements staged at w (int4: scales at sc),
// activations (bf16 or fp32, natural layout) at vs + t * vstride bytes. Lane L handles
// the 16-byte activation pieces L, L + 32, ...; the matching weight bytes are contiguous
// across lanes, so both shared-memory reads are conflict-free.
template <int W, int VT, int T>
__device__ __forceinline__ void staged_dot(const unsigned char* w, const unsigned char* sc, int K,
                                           const unsigned char* vs, int vstride, int lane, float2 (&acc)[T]) {
    constexpr int PE = 16 / Vb<VT>::bytes;  // activation elements per piece
    const int np = K / PE;
#pragma unroll 2
    for (int p = lane; p < np; p += 32) {
        if constexpr (W == DT_BF16 && VT == DT_BF16) {
            const uint4 wv = *reinterpret_cast<const uint4*>(w + p * 16);
#pragma unroll
            for (int t = 0; t < T; ++t) {
                const uint4 x = *reinterpret_cast<const uint4*>(vs + t * vstride + p * 16);
                float2 a = acc[t];
                a = ffma2(bf2(wv.x), bf2(x.x), a);
                a = ffma2(bf2(wv.y), bf2(x.y), a);
                a = ffma2(bf2(wv.z), bf2(x.z), a);
                acc[t] = ffma2(bf2(wv.w), bf2(x.w), a);
            }
        } else if constexpr (W == DT_F32 && VT == DT_F32) {
            const uint4 wv = *reinterpret_cast<const uint4*>(w + p * 16);
#pragma unroll
            for (int t = 0; t < T; ++t) {
                const uint4 x = *reinterpret_cast<const uint4*>(vs + t * vstride + p * 16);
                acc[t] = ffma2(f2(wv.z, wv.w), f2(x.z, x.w), ffma2(f2(wv.x, wv.y), f2(x.x, x.y), acc[t]));
            }
        } else if constexpr (W == DT_BF16 && VT == DT_F32) {
            const uint2 wv = *reinterpret_cast<const uint2*>(w + p * 8);
#pragma unroll
            for (int t = 0; t < T; ++t) {
                const uint4 x = *reinterpret_cast<const uint4*>(vs + t * vstride + p * 16);
                acc[t] = ffma2(bf2(wv.y), f2(x.z, x.w), ffma2(bf2(wv.x), f2(x.x, x.y), acc[t]));
            }
        } else if constexpr (W == DT_INT4 && VT == DT_BF16) {
            const uint32_t wv = *reinterpret_cast<const uint32_t*>(w + p * 4);
            const float s = bf16f(reinterpret_cast<const uint16_t*>(sc)[p >> 2]);
            const float2 n0 = nib2(wv, 0), n1 = nib2(wv, 2), n2 = nib2(wv, 4), n3 = nib2(wv, 6);
#pragma unroll
            for (int t = 0; t < T; ++t) {
                const uint4 x = *reinterpret_cast<const uint4*>(vs + t * vstride + p * 16);
                float2 d = make_float2(0.f, 0.f);
                d = ffma2(n0, bf2(x.x), d);
                d = ffma2(n1, bf2(x.y), d);
                d = ffma2(n2, bf2(x.z), d);
                d = ffma2(n3, bf2(x.w), d);
                acc[t] = ffma2(make_float2(s, s), d, acc[t]);
            }
        } else if constexpr (W == DT_INT4 && VT == DT_F32) {
            const uint32_t wv = *reinterpret_cast<const uint16_t*>(w + p * 2);
            const float s = bf16f(reinterpret_cast<const uint16_t*>(sc)[p >> 3]);
            const float2 n0 = nib2(wv, 0), n1 = nib2(wv, 2);
#pragma unroll
            for (int t = 0; t < T; ++t) {
                const uint4 x = *reinterpret_cast<const uint4*>(vs + t * vstride + p * 16);
                const float2 d = ffma2(n1, f2(x.z, x.w), ffma2(n0, f2(x.x, x.y), make_float2(0.f, 0.f)));
                acc[t] = ffma2(make_float2(s, s), d, acc[t]);
            }
        }
    }
}

__device__ __forceinline__ float hsum(float2 v) { return warp_sum(v.x + v.y); }

// ------------------------------------------------------------------- ring
// Up to four contiguous global ranges copied into one stage.
struct Seg {
    const void* src[4];
    uint32_t bytes[4];
    uint32_t off[4];
    int n;
};

__device__ __forceinline__ void seg_add(Seg& s, const void* src, uint32_t bytes, uint32_t off) {
#pragma unroll
    for (int i = 0; i < 4; ++i)
        if (i == s.n) {
            s.src[i] = src;
            s.bytes[i] = bytes;
            s.off[i] = off;
        }
    ++s.n;
}

// A warp-private ring of stages. Lane 0 issues the bulk copies of a stage; every lane waits
// on the stage's mbarrier; the stage is refilled only after the warp has finished reading it
// (__syncwarp, then a proxy fence before the async-proxy write). Stages 0 .. nsc-1 live in
// the ring region, the others in the h buffer; the depth may change only when the ring is
// drained. Each stage's next completion parity is one bit of `phase`.
struct Ring {
    unsigned char* buf0;  // stages 0 .. nsc-1
    unsigned char* buf1;  // stages nsc .. (h buffer)
    uint64_t* bar;
    uint32_t issued, consumed, phase;
    int ns, nsc, si, sc;  // depth, ring-region depth, next stage to issue, next to consume

    __device__ __forceinline__ unsigned char* stage(int st) const { return st < nsc ? buf0 + st * SB : buf1 + (st - nsc) * SB; }
    __device__ __forceinline__ void issue(const Seg& s, int lane) {
        const int st = si;
        if (lane == 0) {
            fence_proxy_async_smem();
            uint32_t tot = 0;
#pragma unroll
            for (int i = 0; i < 4; ++i) tot += (i < s.n) ? s.bytes[i] : 0u;
            mbar_arrive_expect_tx(bar + st, tot);
            unsigned char* dst = stage(st);
#pragma unroll
            for (int i = 0; i < 4; ++i)
                if (i < s.n) bulk_g2s(dst + s.off[i], s.src[i], s.bytes[i], bar + st);
        }
        si = (si + 1 == ns) ? 0 : si + 1;
        ++issued;
    }
    __device__ __forceinline__ const unsigned char* wait(int* err, uint64_t timeout_ns) {
        mbar_wait(bar + sc, (phase >> sc) & 1u, err, timeout_ns);
        return stage(sc);
    }
    __device__ __forceinline__ void release() {
        __syncwarp();
        phase ^= 1u << sc;
        sc = (sc + 1 == ns) ? 0 : sc + 1;
        ++consumed;
    }
    __device__ __forceinline__ bool full() const { return issued - consumed >= uint32_t(ns); }
    __device__ __forceinline__ void set_depth(int n) { ns = n; si = sc = 0; }  // drained rings only
};

template <int NL>
struct DecParams {
    int H, E, k, I, Is, n_layers;
    int RB, RQ;      // phase C: output rows per block, rows per stage
    Control* ctl;
    float* logits;   // [T, E]
    float* sgate;    // 2 x [T]        (double-buffered across layers)
    float* hsh;      // 2 x [T, Is]
    float* hrt;      // [T * k, I]     (slot t*k + j)
    uint64_t timeout_ns;
    CacheBias cb;
    DecLayer L[NL];
};

template <int XT, int RT, int WT, int T, int NL>
__global__ void __launch_bounds__(THREADS, 1) decode_kernel(const __grid_constant__ DecParams<NL> p) {
    constexpr int NS = Stages<T>::NS;
    extern __shared__ __align__(128) unsigned char smem[];
    const int H = p.H, E = p.E, k = p.k, I = p.I, Is = p.Is;
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int nblocks = gridDim.x;
    const int gw = blockIdx.x * WARPS + warp;
    const int Wtot = nblocks * WARPS;
    int* err = &p.ctl->err;
    const uint64_t to = p.timeout_ns;
    using XW = XWide<XT, T>;
    const Smem S = smem_layout(T, NS, H, E, k, I, Is, XT, p.RB, XW::on);
    unsigned char* xs = smem + S.xs;
    unsigned char* hs = smem + S.hs;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S.bars);
    uint64_t* xbar = bars + WARPS * NS_MAX;
    uint64_t* hbar = xbar + 1;
    uint32_t* s_keys = reinterpret_cast<uint32_t*>(smem + S.keys);
    int* s_ids = reinterpret_cast<int*>(smem + S.ids);
    float* s_w = reinterpret_cast<float*>(smem + S.wts);
    int* s_first = reinterpret_cast<int*>(smem + S.first);
    int* s_uidx = reinterpret_cast<int*>(smem + S.uidx);
    int* s_wcnt = reinterpret_cast<int*>(smem + S.wcnt);
    int* s_ue = reinterpret_cast<int*>(smem + S.ue);
    unsigned* s_um = reinterpret_cast<unsigned*>(smem + S.umask);
    int* s_us = reinterpret_cast<int*>(smem + S.uslot);
    float* s_uw = reinterpret_cast<float*>(smem + S.uw);
    float* s_sg = reinterpret_cast<float*>(smem + S.sg);
    int* s_nu = reinterpret_cast<int*>(smem + S.nu);
    float* s_part = reinterpret_cast<float*>(smem + S.part);
    int* s_jobq = reinterpret_cast<int*>(smem + S.jobq) + warp * 8;  // job code of each ring stage

    Ring ring;
    ring.buf0 = smem + S.ring + warp * NS * SB;
    ring.buf1 = smem + S.hs + warp * (S.nsb - NS) * SB;
    ring.bar = bars + warp * NS_MAX;
    ring.issued = ring.consumed = ring.phase = 0u;
    ring.nsc = NS;
    ring.set_depth(S.nsb);
    if (lane == 0)
        for (int i = 0; i < NS_MAX; ++i) mbar_init(ring.bar + i, 1);
    if (threadIdx.x == 0) {
        mbar_init(xbar, 1);
        mbar_init(hbar, 1);
    }
    fence_mbar_init();
    __syncthreads();

    const int xrow = H * vbytes(XT);                 // bytes of one activation row
    const unsigned char* xv = XW::on ? smem + S.xf : xs;  // activations as the dots read them
    const int xvrow = XW::on ? H * 4 : xrow;
    const int rrow = int(row_bytes(RT, H));          // router / shared-gate row
    const int grow = int(row_bytes(WT, H));          // gate or up row
    const int gsc = scale_bytes(WT, H);
    const int gtot = align16(grow) + gsc;            // one gate/up row with its scales
    const bool pair1 = 2 * gtot <= SB;               // gate and up of one row fit one stage
    const int pparts = pair1 ? 1 : 2;
    const int drow = int(row_bytes(WT, I)), dsc = scale_bytes(WT, I);
    const int srow = int(row_bytes(WT, Is)), ssc = scale_bytes(WT, Is);
    const int nslot = T * k;
    const int jobsA = E + 1;
    const int RB = p.RB, RQ = p.RQ;
    unsigned bar_idx = 0;

    // stage segment of one gate/up row (with scales) at offset `off`
    auto add_row = [&](Seg& s, const void* row, const void* scl, uint32_t off) {
        seg_add(s, row, grow, off);
        if (WT == DT_INT4) seg_add(s, scl, gsc, off + align16(grow));
    };

    if (threadIdx.x == 0) {
        mbar_arrive_expect_tx(xbar, T * xrow);
        bulk_g2s(xs, p.L[0].x, T * xrow, xbar);
    }

    for (int l = 0; l < p.n_layers; ++l) {
        const DecLayer& Ly = p.L[l];
        float* sgate = p.sgate + (l & 1) * T;
        float* hsh = p.hsh + size_t(l & 1) * T * Is;
        const char* sh_gate = static_cast<const char*>(Ly.sh_gate);
        const char* sh_up = static_cast<const char*>(Ly.sh_up);

        ring.set_depth(S.nsb);  // drained: phases A and B borrow the h buffer
        // ---------------------------------------------------------- phase A
        // Router rows 0..E-1 and the shared gate row (job E), by warps 1..7 of every block
        // (warp 0 only starts copies of its phase-B rows).
        // Phase B's job list: the shared expert's gate/up rows (jobs 0..Is-1, no routing
        // needed, so their copies start here), then the routed rows (u, i) of the U distinct
        // experts; job j belongs to warp j mod Wtot.
        auto segB = [&](int job, int part, int U_) {
            Seg s;
            s.n = 0;
            const char *g, *u;
            const uint16_t *gs = nullptr, *us = nullptr;
            if (job < Is) {
                g = sh_gate + size_t(job) * grow;
                u = sh_up + size_t(job) * grow;
                if (WT == DT_INT4) { gs = Ly.sh_s_gate + size_t(job) * (H / 32); us = Ly.sh_s_up + size_t(job) * (H / 32); }
            } else {
                const int r = job - Is, uu = r / I, i = r - uu * I;
                const size_t rowi = size_t(s_ue[uu]) * I + i;
                g = static_cast<const char*>(Ly.w_gate) + rowi * grow;
                u = static_cast<const char*>(Ly.w_up) + rowi * grow;
                if (WT == DT_INT4) { gs = Ly.s_gate + rowi * (H / 32); us = Ly.s_up + rowi * (H / 32); }
            }
            (void)U_;
            if (pair1 || part == 0) add_row(s, g, gs, 0);
            if (pair1 || part == 1) add_row(s, u, us, pair1 ? gtot : 0);
            return s;
        };
        // Issue cursor of phase B: this warp's jobs gw, gw + Wtot, ... of the list [shared
        // rows 0..Is-1 | routed rows]; the shared ones can start before the routing is known
        // (routed_ok), the routed ones only after.
        int bj = gw, bp = 0, bcur = 0;
        bool routed_ok = false;
        int Ucur = 0;
        auto issueB = [&]() -> bool {
            if (bp == 0) {
                if (bj >= Is && (!routed_ok || bj >= Is + Ucur * I)) return false;
                bcur = bj;
                bj += Wtot;
            }
            if (lane == 0) s_jobq[ring.si] = (bcur << 1) | bp;
            ring.issue(segB(bcur, bp, Ucur), lane);
            if (++bp == pparts) bp = 0;
            return true;
        };
        {
            auto segA = [&](int job) {
                Seg s;
                s.n = 0;
                seg_add(s, job < E ? static_cast<const void*>(static_cast<const char*>(Ly.router_w) + size_t(job) * rrow)
                                   : Ly.shared_gate_w,
                        rrow, 0);
                return s;
            };
            const int WA = nblocks * (WARPS - 1);
            const int wA = warp == 0 ? jobsA : blockIdx.x + nblocks * (warp - 1);
            int aj = wA;
            while (!ring.full() && aj < jobsA) { ring.issue(segA(aj), lane); aj += WA; }
            while (!ring.full() && aj >= jobsA && issueB()) {}  // shared gate/up copies ahead of routing
            mbar_wait(xbar, l & 1, err, to);
            if (XW::on) {  // widen this layer's activations once
                const uint32_t* x2 = reinterpret_cast<const uint32_t*>(xs);
                float2* xw = reinterpret_cast<float2*>(smem + S.xf);
                for (int i = threadIdx.x; i < T * H / 2; i += THREADS) xw[i] = bf2(x2[i]);
                __syncthreads();
            }
            for (int job = wA; job < jobsA; job += WA) {
                float2 a[T];
#pragma unroll
                for (int t = 0; t < T; ++t) a[t] = make_float2(0.f, 0.f);
                const unsigned char* d = ring.wait(err, to);
                staged_dot<RT, XW::vt, T>(d, nullptr, H, xv, xvrow, lane, a);
                ring.release();
                if (aj < jobsA) {
                    ring.issue(segA(aj), lane);
                    aj += WA;
                } else {
                    issueB();
                }
                if (job < E) {
                    const float b = Ly.router_bias ? Ly.router_bias[job] : 0.0f;
#pragma unroll
                    for (int t = 0; t < T; ++t) {
                        const float v = hsum(a[t]);
                        if (lane == 0) p.logits[t * E + job] = v + b;
                    }
                } else {
#pragma unroll
                    for (int t = 0; t < T; ++t) {
                        const float v = hsum(a[t]);
                        if (lane == 0) sgate[t] = 1.0f / (1.0f + expf(-v));
                    }
                }
            }
        }
        grid_barrier(p.ctl, nblocks, bar_idx++, to);

        // ---------------------------------------------------------- phase B
        if (p.cb.cached == nullptr) {
            for (int i = threadIdx.x; i < T * E; i += THREADS) s_keys[i] = order_key(__ldcg(p.logits + i));
            __syncthreads();
            if (warp < T) warp_topk_keys(E, k, s_keys + warp * E, s_ids + warp * k, s_w + warp * k);
        } else if (warp < T) {  // opt-in cache-aware routing
            int id;
            float wv;
            warp_route_any(p.logits + warp * E, E, k, p.cb.cached, p.cb.lambda, id, wv);
            if (lane < k) {
                s_ids[warp * k + lane] = id;
                s_w[warp * k + lane] = wv;
            }
        }
        __syncthreads();
        // distinct experts over the T*k routed slots: u numbers the first occurrences in
        // slot order; slot t*k + j of token t maps to u with weight w[t][j]
        if constexpr (T == 1) {
            if (threadIdx.x < k) {
                s_ue[threadIdx.x] = s_ids[threadIdx.x];
                s_um[threadIdx.x] = 1u;
                s_us[threadIdx.x] = threadIdx.x;
                s_uw[threadIdx.x] = s_w[threadIdx.x];
            }
            if (threadIdx.x == 0) *s_nu = k;
        } else {
            const int i = threadIdx.x;
            if (i < nslot) s_first[s_ids[i]] = 0x7fffffff;
            __syncthreads();
            if (i < nslot) atomicMin(&s_first[s_ids[i]], i);
            __syncthreads();
            bool lead = false;
            int rank = 0;
            if (warp < MAX_SLOTS / 32) {
                lead = i < nslot && s_first[s_ids[i]] == i;
                const unsigned bal = __ballot_sync(FULL, lead);
                rank = __popc(bal & ((1u << lane) - 1u));
                if (lane == 0) s_wcnt[warp] = __popc(bal);
            }
            __syncthreads();
            if (lead) {
                int base = 0;
                for (int w2 = 0; w2 < warp; ++w2) base += s_wcnt[w2];
                const int u = base + rank;
                s_uidx[i] = u;
                s_ue[u] = s_ids[i];
                s_um[u] = 0u;
#pragma unroll
                for (int t = 0; t < T; ++t) { s_us[u * T + t] = 0; s_uw[u * T + t] = 0.0f; }
            }
            if (i == 0) {
                int nu = 0;
                for (int w2 = 0; w2 < MAX_SLOTS / 32; ++w2) nu += s_wcnt[w2];
                *s_nu = nu;
            }
            __syncthreads();
            if (i < nslot) {
                const int t = i / k;
                const int u = s_uidx[s_first[s_ids[i]]];
                atomicOr(&s_um[u], 1u << t);
                s_us[u * T + t] = i;
                s_uw[u * T + t] = s_w[i];
            }
        }
        if (blockIdx.x == 0) {
            for (int i = threadIdx.x; i < nslot; i += blockDim.x) {
                Ly.ids[i] = s_ids[i];
                Ly.w[i] = s_w[i];
            }
        }
        __syncthreads();
        const int U = *s_nu;
        // Phase C: block b owns output rows [r0, r0 + nrows), cut into nq chunks of rq rows
        // (nq a divisor of 8). Warp w works on chunk q = w mod nq for the expert slots
        // u = w / nq, w / nq + 8 / nq, ... (u == U: the shared expert), accumulating the
        // weighted lane partials in registers and reducing once. The 8 / nq warp groups of a
        // chunk are then summed in a fixed order: the combine stays deterministic.
        const int r0 = blockIdx.x * RB;
        const int nrows = max(0, min(RB, H - r0));
        const int nq0 = (nrows + RQ - 1) / RQ;
        const int nq = nq0 <= 1 ? 1 : (nq0 <= 2 ? 2 : (nq0 <= 4 ? 4 : 8));
        const int rq = (nrows + nq - 1) / nq;
        const int gpc = WARPS / nq;             // warp groups per chunk
        const int cq = warp % nq, cgrp = warp / nq;
        const int jobsC = U + 1;                // this warp's experts: u = cgrp + gpc * m
        auto segC = [&](int u) {
            Seg s;
            s.n = 0;
            const int n0 = r0 + cq * rq, nr = max(0, min(rq, r0 + nrows - n0));
            if (u < U) {
                const size_t row = size_t(s_ue[u]) * H + n0;
                seg_add(s, static_cast<const char*>(Ly.w_down) + row * drow, nr * drow, 0);
                if (WT == DT_INT4) seg_add(s, Ly.s_down + row * (I / 32), nr * dsc, align16(RQ * drow));
            } else {
                seg_add(s, static_cast<const char*>(Ly.sh_down) + size_t(n0) * srow, nr * srow, 0);
                if (WT == DT_INT4) seg_add(s, Ly.sh_s_down + size_t(n0) * (Is / 32), nr * ssc, align16(RQ * srow));
            }
            return s;
        };
        {
            routed_ok = true;
            Ucur = U;
            while (!ring.full() && issueB()) {}
            __syncwarp();
            float2 a[T], b[T];
#pragma unroll
            for (int t = 0; t < T; ++t) a[t] = b[t] = make_float2(0.f, 0.f);
            while (ring.consumed != ring.issued) {
                const int code = s_jobq[ring.sc];
                const int job = code >> 1, part = code & 1;
                const unsigned char* d = ring.wait(err, to);
                if (pair1 || part == 0) staged_dot<WT, XW::vt, T>(d, d + align16(grow), H, xv, xvrow, lane, a);
                if (pair1 || part == 1) {
                    const unsigned char* du = d + (pair1 ? gtot : 0);
                    staged_dot<WT, XW::vt, T>(du, du + align16(grow), H, xv, xvrow, lane, b);
                }
                ring.release();
                issueB();
                if (part == pparts - 1) {
                    if (job < Is) {
#pragma unroll
                        for (int t = 0; t < T; ++t) {
                            const float av = hsum(a[t]), bv = hsum(b[t]);
                            if (lane == 0) hsh[t * Is + job] = silu_mul(av, bv);
                        }
                    } else {
                        const int r = job - Is, u = r / I, i = r - u * I;
                        const unsigned mask = s_um[u];
#pragma unroll
                        for (int t = 0; t < T; ++t) {
                            const float av = hsum(a[t]), bv = hsum(b[t]);
                            if (lane == 0 && (mask >> t & 1u)) p.hrt[size_t(s_us[u * T + t]) * I + i] = silu_mul(av, bv);
                        }
                    }
#pragma unroll
                    for (int t = 0; t < T; ++t) a[t] = b[t] = make_float2(0.f, 0.f);
                }
            }
        }
        // arrive, then start the first phase-C copies (they do not depend on h), then wait
        grid_arrive(p.ctl);
        int cj = cgrp;  // issue cursor of phase C (expert slot)
        const bool has_rows = cq * rq < nrows;
        ring.set_depth(NS);  // drained: phase C keeps the h buffer for h
        while (has_rows && !ring.full() && cj < jobsC) { ring.issue(segC(cj), lane); cj += gpc; }
        grid_wait(p.ctl, nblocks, bar_idx++, to);
        if (l + 1 == p.n_layers) grid_release(p.ctl, nblocks);  // the launch's last barrier

        // ---------------------------------------------------------- phase C
        if (threadIdx.x == 0) {
            fence_proxy_async_global();
            fence_proxy_async_smem();
            mbar_arrive_expect_tx(hbar, 4 * (nslot * I + T * Is));
            bulk_g2s(hs, p.hrt, 4 * nslot * I, hbar);
            bulk_g2s(hs + 4 * nslot * I, hsh, 4 * T * Is, hbar);
            if (l + 1 < p.n_layers) {  // x of the next layer: phase B no longer reads xs
                mbar_arrive_expect_tx(xbar, T * xrow);
                bulk_g2s(xs, p.L[l + 1].x, T * xrow, xbar);
            }
        }
        if (threadIdx.x < T) s_sg[threadIdx.x] = __ldcg(sgate + threadIdx.x);
        if (l + 1 < p.n_layers && lane == 0) {
            // L2 prefetch of the next layer's router rows and shared gate/up rows of this warp's jobs
            const DecLayer& Nx = p.L[l + 1];
            if (warp > 0)
                for (int job = blockIdx.x + nblocks * (warp - 1); job < E; job += nblocks * (WARPS - 1))
                    prefetch_l2(static_cast<const char*>(Nx.router_w) + size_t(job) * rrow, rrow);
            for (int job = gw; job < Is; job += Wtot) {
                prefetch_l2(static_cast<const char*>(Nx.sh_gate) + size_t(job) * grow, grow);
                prefetch_l2(static_cast<const char*>(Nx.sh_up) + size_t(job) * grow, grow);
            }
        }
        __syncthreads();
        mbar_wait(hbar, l & 1, err, to);
        const unsigned char* hr = hs;                      // routed h, slot s at hr + s * 4I
        const unsigned char* hsv = hs + 4 * nslot * I;     // shared h, token t at hsv + t * 4Is
        const int nr = has_rows ? min(rq, nrows - cq * rq) : 0;
        float2 acc[RQ_MAX][T];
#pragma unroll
        for (int r = 0; r < RQ_MAX; ++r)
#pragma unroll
            for (int t = 0; t < T; ++t) acc[r][t] = make_float2(0.f, 0.f);
        for (int u = cgrp; has_rows && u < jobsC; u += gpc) {
            const unsigned char* d = ring.wait(err, to);
            if (u < U) {
                const unsigned mask = s_um[u];
#pragma unroll
                for (int t = 0; t < T; ++t) {
                    if (mask >> t & 1u) {
                        const float wgt = s_uw[u * T + t];
                        const unsigned char* hv = hr + 4 * s_us[u * T + t] * I;
#pragma unroll
                        for (int r = 0; r < RQ_MAX; ++r) {
                            if (r < nr) {
                                float2 one[1] = {make_float2(0.f, 0.f)};
                                staged_dot<WT, DT_F32, 1>(d + r * drow, d + align16(RQ * drow) + r * dsc, I, hv, 0, lane, one);
                                acc[r][t] = ffma2(make_float2(wgt, wgt), one[0], acc[r][t]);
                            }
                        }
                    }
                }
            } else {
#pragma unroll
                for (int r = 0; r < RQ_MAX; ++r) {
                    if (r < nr) {
                        float2 dd[T];
#pragma unroll
                        for (int t = 0; t < T; ++t) dd[t] = make_float2(0.f, 0.f);
                        staged_dot<WT, DT_F32, T>(d + r * srow, d + align16(RQ * srow) + r * ssc, Is, hsv, 4 * Is, lane, dd);
#pragma unroll
                        for (int t = 0; t < T; ++t) acc[r][t] = ffma2(make_float2(s_sg[t], s_sg[t]), dd[t], acc[r][t]);
                    }
                }
            }
            ring.release();
            if (cj < jobsC) { ring.issue(segC(cj), lane); cj += gpc; }
        }
#pragma unroll
        for (int r = 0; r < RQ_MAX; ++r) {
            if (r < nr) {
#pragma unroll
                for (int t = 0; t < T; ++t) {
                    const float v = hsum(acc[r][t]);
                    if (lane == 0) s_part[(cgrp * RB + cq * rq + r) * T + t] = v;
                }
            }
        }
        __syncthreads();
        for (int i = threadIdx.x; i < nrows * T; i += THREADS) {
            const int row = i / T, t = i - (i / T) * T;
            float acc = 0.0f;
            for (int g2 = 0; g2 < gpc; ++g2) acc += s_part[(g2 * RB + row) * T + t];
            Ly.out[size_t(t) * H + r0 + row] = acc;
        }
        if (l + 1 < p.n_layers) grid_barrier(p.ctl, nblocks, bar_idx++, to);
    }
}

// Down rows per phase-C stage: as many as fit one stage (with their int4 scales), at most
// RQ_MAX; 0 if not even one row fits.
int decode_rows_per_stage(const redmoe_layer* sh) {
    const int wt = sh->expert_dtype;
    const int rb = int(row_bytes(wt, sh->inter > sh->shared_inter ? sh->inter : sh->shared_inter));
    const int sc = scale_bytes(wt, sh->inter > sh->shared_inter ? sh->inter : sh->shared_inter);
    for (int rq = RQ_MAX; rq >= 1; --rq)
        if (rq * rb <= SEG_MAX && align16(rq * rb) + rq * sc <= SB) return rq;
    return 0;
}

// Resident blocks per SM of a decode kernel at a dynamic shared-memory size, cached per
// (device, kernel, size) so that a launch makes no attribute calls after the first; -1
// on a CUDA error.
int blocks_per_sm(const void* kern, int smem) {
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
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, THREADS, smem) != cudaSuccess) return -1;
    per_sm = per_sm > 1 ? 1 : per_sm;
    cache.push_back({dev, kern, smem, per_sm});
    return per_sm;
}

template <int XT, int RT, int WT, int T, int NL>
redmoe_status launch_one(const redmoe_layer* sh, const DecLayer* layers, int n_layers, void* ws, cudaStream_t stream,
                         CacheBias cb) {
    DevInfo di;
    if (!get_dev_info(&di)) return REDMOE_ERR_CUDA;
    const int RB = (sh->hidden + di.sm_count - 1) / di.sm_count;
    const int RQ = decode_rows_per_stage(sh);
    if (RQ < 1 || RB > WARPS * RQ) return REDMOE_ERR_UNSUPPORTED;
    const Smem S = smem_layout(T, Stages<T>::NS, sh->hidden, sh->n_experts, sh->top_k, sh->inter, sh->shared_inter, XT, RB,
                               XWide<XT, T>::on);
    if (S.total > di.max_smem_optin) return REDMOE_ERR_UNSUPPORTED;
    auto kern = decode_kernel<XT, RT, WT, T, NL>;
    const int per_sm = blocks_per_sm(reinterpret_cast<const void*>(kern), S.total);
    if (per_sm < 0) return REDMOE_ERR_CUDA;
    if (per_sm == 0) return REDMOE_ERR_UNSUPPORTED;
    const int grid = di.sm_count * per_sm;

    DecParams<NL>* pp = new (std::nothrow) DecParams<NL>();
    if (!pp) return REDMOE_ERR_CUDA;
    DecParams<NL>& q = *pp;
    q.H = sh->hidden; q.E = sh->n_experts; q.k = sh->top_k; q.I = sh->inter; q.Is = sh->shared_inter;
    q.n_layers = n_layers;
    q.RB = RB;
    q.RQ = RQ;
    const DecodeWs L = decode_ws_layout(T, q.E, q.k, q.I, q.Is);
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
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(THREADS);
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

template <int XT, int RT, int WT, int T>
redmoe_status launch_t(const redmoe_layer* sh, const DecLayer* layers, int n_layers, void* ws, cudaStream_t stream,
                       int* launches, CacheBias cb) {
    redmoe_status st = REDMOE_OK;
    if (n_layers == 1) {
        st = launch_one<XT, RT, WT, T, 1>(sh, layers, 1, ws, stream, cb);
        if (st == REDMOE_OK && launches) *launches += 1;
        return st;
    }
    for (int l0 = 0; l0 < n_layers && st == REDMOE_OK; l0 += MAX_STACK) {
        const int n = n_layers - l0 < MAX_STACK ? n_layers - l0 : MAX_STACK;
        st = launch_one<XT, RT, WT, T, MAX_STACK>(sh, layers + l0, n, ws, stream, cb);
        if (st == REDMOE_OK && launches) *launches += 1;
    }
    return st;
}

template <int XT, int RT, int WT>
redmoe_status launch_dt(const redmoe_layer* sh, const DecLayer* layers, int n_layers, int T, void* ws,
                        cudaStream_t stream, int* launches, CacheBias cb) {
    switch (T) {
        case 1: return launch_t<XT, RT, WT, 1>(sh, layers, n_layers, ws, stream, launches, cb);
        case 2: return launch_t<XT, RT, WT, 2>(sh, layers, n_layers, ws, stream, launches, cb);
        case 3: return launch_t<XT, RT, WT, 3>(sh, layers, n_layers, ws, stream, launches, cb);
        case 4: return launch_t<XT, RT, WT, 4>(sh, layers, n_layers, ws, stream, launches, cb);
        default: return REDMOE_ERR_UNSUPPORTED;
    }
}

}  // namespace

DecodeWs decode_ws_layout(int T, int E, int k, int I, int Is) {
    DecodeWs w;
    size_t o = 256;  // control block
    w.logits = o; o = align256(o + 4ull * T * E);
    w.sgate = o; o = align256(o + 4ull * 2 * T);
    w.hsh = o; o = align256(o + 4ull * 2 * T * Is);
    w.hrt = o; o = align256(o + 4ull * T * k * I);
    w.total = o;
    return w;
}

// Shapes the decode kernel stages: every single weight segment must fit one 4 KiB stage.
bool decode_shape_ok(const redmoe_layer* sh) {
    const int H = sh->hidden, I = sh->inter, Is = sh->shared_inter, wt = sh->expert_dtype, rt = sh->router_dtype;
    if (wt == DT_INT2) return false;  // int2 experts: one-row kernel only
    if (row_bytes(rt, H) > SEG_MAX || row_bytes(wt, H) > SEG_MAX) return false;
    if (align16(int(row_bytes(wt, H))) + scale_bytes(wt, H) > SB) return false;
    if (decode_rows_per_stage(sh) < 1) return false;
    if (wt == DT_INT4 && (H % 256 || I % 256 || Is % 256)) return false;
    return true;
}

std::vector<DecLayer> dec_rows(const redmoe_layer* sh, const DecLayer* layers, int n_layers, int r0) {
    std::vector<DecLayer> v(layers, layers + n_layers);
    const size_t xb = sh->x_dtype == DT_F32 ? 4 : 2;
    for (DecLayer& d : v) {
        d.x = static_cast<const char*>(d.x) + size_t(r0) * sh->hidden * xb;
        d.out += size_t(r0) * sh->hidden;
        d.ids += size_t(r0) * sh->top_k;
        d.w += size_t(r0) * sh->top_k;
    }
    return v;
}

bool decode_split_ok(const redmoe_layer* sh, int T) {
    return (T == 3 || T == 4) && decodefr_shape_ok(sh, 2) && decode1_shape_ok(sh);
}

redmoe_status launch_decode(const redmoe_layer* sh, const DecLayer* layers, int n_layers, int T, void* ws,
                            cudaStream_t stream, int* launches, CacheBias cb) {
    if (T == 1 && decode1_shape_ok(sh)) return launch_decode1(sh, layers, n_layers, ws, stream, launches, cb);
    if (decodefr_shape_ok(sh, T)) return launch_decodefr(sh, layers, n_layers, T, ws, stream, launches, cb);
    if (decode_split_ok(sh, T)) {
        // three or four rows: rows 0-1 on the few-row kernel, then the rest on the one-row
        // (T = 3) or the few-row kernel (T = 4). Rows are independent through the layer,
        // and measured per bf16 call this beats one launch of the ring kernel below:
        // 24.7 + 48.9 = 73.6 against 80.8 us at T = 3, 2 x 48.9 = 97.8 against 107.4 us at T = 4.
        redmoe_status st = launch_decodefr(sh, layers, n_layers, 2, ws, stream, launches, cb);
        if (st != REDMOE_OK) return st;
        const std::vector<DecLayer> rest = dec_rows(sh, layers, n_layers, 2);
        return T == 3 ? launch_decode1(sh, rest.data(), n_layers, ws, stream, launches, cb)
                      : launch_decodefr(sh, rest.data(), n_layers, 2, ws, stream, launches, cb);
    }
    if (!decode_shape_ok(sh)) return REDMOE_ERR_UNSUPPORTED;
    const int xt = sh->x_dtype, rt = sh->router_dtype, wt = sh->expert_dtype;
    if (xt == DT_F32 && rt == DT_F32 && wt == DT_F32)
        return launch_dt<DT_F32, DT_F32, DT_F32>(sh, layers, n_layers, T, ws, stream, launches, cb);
    if (xt == DT_BF16 && rt == DT_BF16 && wt == DT_BF16)
        return launch_dt<DT_BF16, DT_BF16, DT_BF16>(sh, layers, n_layers, T, ws, stream, launches, cb);
    if (xt == DT_BF16 && rt == DT_BF16 && wt == DT_INT4)
        return launch_dt<DT_BF16, DT_BF16, DT_INT4>(sh, layers, n_layers, T, ws, stream, launches, cb);
    return REDMOE_ERR_UNSUPPORTED;
}

}  // namespace redmoe
