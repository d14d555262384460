// Decode path (1..4 token rows): one persistent cooperative kernel per call.
//
// A layer at decode size is a bandwidth problem: every routed expert row is read once
// from HBM and dotted with 1..4 activation rows. The kernel streams the layer in three
// phases separated by grid barriers, with every block of the grid resident:
//
//   A  router logits (E rows of Wr), the shared gate (row g) and the shared expert's
//      gate/up rows with SwiGLU (the shared expert needs no routing, so it overlaps
//      the router, like the "extra slot" of the DwarfStar MoE kernel in "Research
//      notes, October 2026", section 1); each block also starts an L2 prefetch of the
//      shared-expert down rows it will need in phase C.
//   B  every block computes the top-k of every token from the logits (a warp per
//      token, warp-shuffle selection), the renormalised weights, and the list of
//      distinct experts; it prefetches into L2 the routed down rows it will use in
//      phase C, then streams the routed gate/up rows (one gate row and one up row per
//      warp job) and writes h = silu(a) * u.
//   C  each warp owns output rows n: it sums, over every distinct expert and the
//      shared expert, weight * (Wd[n, :] . h), and writes out[t, n] once (the weighted
//      combine happens in registers, deterministically, with no atomics).
//
// Down rows are only 512 elements long (1 KiB in bf16, 256 B in int4): phase C spreads
// the (expert, 16-byte chunk) pairs of a row over the 32 lanes instead of giving each
// lane one row, the lesson of the narrow-row kernel in "Research notes, October 2026",
// section 4 ("Narrow-row IQ mul_mv", 512-column expert down rows).
//
// Activations are staged in shared memory in a chunk-interleaved layout: for a weight
// chunk c (16 bytes of weights = V elements) read by lane c % 32, the matching V
// activations sit in P 16-byte pieces at slots ((c / 32) * P + q) * 32 + c % 32, so the
// warp's activation reads are contiguous 512-byte rows (no bank conflicts) whatever V.
#include <new>

#include "common.cuh"
#include "internal.h"
#include "gemv.cuh"
#include "topk.cuh"

namespace redmoe {

namespace {

constexpr int THREADS = 256;
constexpr int WARPS = THREADS / 32;
constexpr int G = 8;         // 16-byte chunks per lane per row group
constexpr int NT = DECODE_MAX_T;
constexpr int CB = 8;        // (expert, chunk) items per lane in flight in phase C

struct Smem {
    int xr, xw, hr, hsh, ids, wts, ue, umask, uslot, uw, sg, nu, total;
};

__host__ __device__ inline Smem smem_layout(int T, int H, int k, int I, int Is, int xt, int rt, int wt) {
    Smem s;
    int o = 0;
    const int xr1 = staged_bytes(H, rt, xt);
    const int xw1 = staged_bytes(H, wt, xt);
    const bool same = (wv(rt) == wv(wt));
    s.xr = o; o += T * xr1;
    s.xw = same ? s.xr : o; o += same ? 0 : T * xw1;
    s.hr = o; o += T * k * staged_bytes(I, wt, DT_F32);
    s.hsh = o; o += T * staged_bytes(Is, wt, DT_F32);
    s.ids = o; o += 4 * T * k;
    s.wts = o; o += 4 * T * k;
    s.ue = o; o += 4 * T * k;
    s.umask = o; o += 4 * T * k;
    s.uslot = o; o += 4 * T * k * NT;
    s.uw = o; o += 4 * T * k * NT;
    s.sg = o; o += 4 * NT;
    s.nu = o; o += 16;
    s.total = (o + 127) & ~127;
    return s;
}

template <int NL>
struct DecParams {
    int T, H, E, k, I, Is, n_layers;
    Control* ctl;
    float* logits;   // [T, E]
    float* sgate;    // 2 x [T]        (double-buffered across layers)
    float* hsh;      // 2 x [T, Is]
    float* hrt;      // [T * k, I]     (slot t*k + j)
    uint64_t timeout_ns;
    DecLayer L[NL];
};

template <int XT, int RT, int WT, int NL>
__global__ void __launch_bounds__(THREADS, 1) decode_kernel(const __grid_constant__ DecParams<NL> p) {
    extern __shared__ __align__(128) unsigned char smem[];
    const int T = p.T, H = p.H, E = p.E, k = p.k, I = p.I, Is = p.Is;
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int nblocks = gridDim.x;
    const int gw = blockIdx.x * WARPS + warp;
    const int Wtot = nblocks * WARPS;
    const Smem S = smem_layout(T, H, k, I, Is, XT, RT, WT);
    uint4* xr = reinterpret_cast<uint4*>(smem + S.xr);
    uint4* xw = reinterpret_cast<uint4*>(smem + S.xw);
    uint4* hr = reinterpret_cast<uint4*>(smem + S.hr);
    uint4* hs = reinterpret_cast<uint4*>(smem + S.hsh);
    int* s_ids = reinterpret_cast<int*>(smem + S.ids);
    float* s_w = reinterpret_cast<float*>(smem + S.wts);
    int* s_ue = reinterpret_cast<int*>(smem + S.ue);
    unsigned* s_um = reinterpret_cast<unsigned*>(smem + S.umask);
    int* s_us = reinterpret_cast<int*>(smem + S.uslot);
    float* s_uw = reinterpret_cast<float*>(smem + S.uw);
    float* s_sg = reinterpret_cast<float*>(smem + S.sg);
    int* s_nu = reinterpret_cast<int*>(smem + S.nu);

    const int xr_stride = staged_bytes(H, RT, XT) / 16;
    const int xw_stride = staged_bytes(H, WT, XT) / 16;
    const int hr_stride = staged_bytes(I, WT, DT_F32) / 16;
    const int hs_stride = staged_bytes(Is, WT, DT_F32) / 16;
    const long xbytes = long(H) * vbytes(XT);
    const long gate_row = row_bytes(WT, H);   // bytes of one gate/up row
    const long down_row = row_bytes(WT, I);   // bytes of one routed down row
    const long sdown_row = row_bytes(WT, Is);
    const int rowsC = (H + Wtot - 1) / Wtot;  // phase-C rows per warp (strided by Wtot)

    for (int l = 0; l < p.n_layers; ++l) {
        const DecLayer& Ly = p.L[l];
        float* sgate = p.sgate + (l & 1) * T;
        float* hsh = p.hsh + size_t(l & 1) * T * Is;

        // ---------------------------------------------------------- phase A
        for (int t = 0; t < T; ++t) {
            const void* xt = static_cast<const char*>(Ly.x) + t * xbytes;
            stage_vec<RT, XT>(xr + t * xr_stride, xt, H, false);
            if (wv(RT) != wv(WT)) stage_vec<WT, XT>(xw + t * xw_stride, xt, H, false);
        }
        // L2 prefetch of the shared-expert down rows this block uses in phase C
        if (threadIdx.x == 0) {
            for (int r = 0; r < rowsC; ++r) {
                const int n0 = blockIdx.x * WARPS + r * Wtot;
                const int n1 = min(n0 + WARPS, H);
                if (n0 < H) {
                    prefetch_l2(static_cast<const char*>(Ly.sh_down) + n0 * sdown_row, uint32_t((n1 - n0) * sdown_row));
                    if (WT == DT_INT4)
                        prefetch_l2(Ly.sh_s_down + size_t(n0) * (Is / 32), uint32_t((n1 - n0) * (Is / 32) * 2));
                }
            }
        }
        __syncthreads();
        const int jobsA = E + 1 + Is;
        for (int job = gw; job < jobsA; job += Wtot) {
            float a[NT] = {0.f, 0.f, 0.f, 0.f};
            if (job <= E) {
                const void* row = (job < E) ? static_cast<const void*>(static_cast<const char*>(Ly.router_w) +
                                                                       size_t(job) * row_bytes(RT, H))
                                            : Ly.shared_gate_w;
                row_dots<RT, XT>(row, nullptr, H, xr, xr_stride, T, lane, a);
#pragma unroll
                for (int t = 0; t < NT; ++t) a[t] = warp_sum(a[t]);
                if (lane == 0) {
                    for (int t = 0; t < T; ++t) {
                        if (job < E)
                            p.logits[t * E + job] = a[t] + (Ly.router_bias ? Ly.router_bias[job] : 0.0f);
                        else
                            sgate[t] = 1.0f / (1.0f + expf(-a[t]));
                    }
                }
            } else {
                const int i = job - E - 1;
                float u[NT] = {0.f, 0.f, 0.f, 0.f};
                pair_dots<WT, XT>(static_cast<const char*>(Ly.sh_gate) + size_t(i) * gate_row,
                                  WT == DT_INT4 ? Ly.sh_s_gate + size_t(i) * (H / 32) : nullptr,
                                  static_cast<const char*>(Ly.sh_up) + size_t(i) * gate_row,
                                  WT == DT_INT4 ? Ly.sh_s_up + size_t(i) * (H / 32) : nullptr, H, xw,
                                  xw_stride, T, lane, a, u);
#pragma unroll
                for (int t = 0; t < NT; ++t) { a[t] = warp_sum(a[t]); u[t] = warp_sum(u[t]); }
                if (lane == 0)
                    for (int t = 0; t < T; ++t) hsh[t * Is + i] = silu_mul(a[t], u[t]);
            }
        }
        grid_barrier(p.ctl, nblocks, p.timeout_ns);

        // ---------------------------------------------------------- phase B
        if (warp < T) warp_topk(p.logits + warp * E, E, k, s_ids + warp * k, s_w + warp * k);
        __syncthreads();
        if (threadIdx.x == 0) {
            int nu = 0;
            for (int t = 0; t < T; ++t) {
                for (int j = 0; j < k; ++j) {
                    const int e = s_ids[t * k + j];
                    int u = 0;
                    while (u < nu && s_ue[u] != e) ++u;
                    if (u == nu) {
                        s_ue[u] = e;
                        s_um[u] = 0u;
                        for (int tt = 0; tt < NT; ++tt) { s_us[u * NT + tt] = -1; s_uw[u * NT + tt] = 0.0f; }
                        ++nu;
                    }
                    s_um[u] |= 1u << t;
                    s_us[u * NT + t] = t * k + j;
                    s_uw[u * NT + t] = s_w[t * k + j];
                }
            }
            *s_nu = nu;
        }
        if (blockIdx.x == 0) {
            for (int i = threadIdx.x; i < T * k; i += blockDim.x) {
                Ly.ids[i] = s_ids[i];
                Ly.w[i] = s_w[i];
            }
        }
        __syncthreads();
        const int U = *s_nu;
        // L2 prefetch of the routed down rows this block uses in phase C
        if (threadIdx.x < U) {
            const int e = s_ue[threadIdx.x];
            const char* base = static_cast<const char*>(Ly.w_down) + size_t(e) * H * down_row;
            for (int r = 0; r < rowsC; ++r) {
                const int n0 = blockIdx.x * WARPS + r * Wtot;
                const int n1 = min(n0 + WARPS, H);
                if (n0 < H) {
                    prefetch_l2(base + size_t(n0) * down_row, uint32_t((n1 - n0) * down_row));
                    if (WT == DT_INT4)
                        prefetch_l2(Ly.s_down + (size_t(e) * H + n0) * (I / 32), uint32_t((n1 - n0) * (I / 32) * 2));
                }
            }
        }
        const int jobsB = U * I;
        for (int job = gw; job < jobsB; job += Wtot) {
            const int u = job / I;
            const int i = job - u * I;
            const int e = s_ue[u];
            const unsigned mask = s_um[u];
            float a[NT] = {0.f, 0.f, 0.f, 0.f}, b[NT] = {0.f, 0.f, 0.f, 0.f};
            const size_t rowi = size_t(e) * I + i;
            pair_dots<WT, XT>(static_cast<const char*>(Ly.w_gate) + rowi * gate_row,
                              WT == DT_INT4 ? Ly.s_gate + rowi * (H / 32) : nullptr,
                              static_cast<const char*>(Ly.w_up) + rowi * gate_row,
                              WT == DT_INT4 ? Ly.s_up + rowi * (H / 32) : nullptr, H, xw, xw_stride, T, lane, a, b);
#pragma unroll
            for (int t = 0; t < NT; ++t) { a[t] = warp_sum(a[t]); b[t] = warp_sum(b[t]); }
            if (lane == 0)
                for (int t = 0; t < T; ++t)
                    if (mask >> t & 1u) p.hrt[size_t(s_us[u * NT + t]) * I + i] = silu_mul(a[t], b[t]);
        }
        grid_barrier(p.ctl, nblocks, p.timeout_ns);

        // ---------------------------------------------------------- phase C
        for (int s = 0; s < T * k; ++s) stage_vec<WT, DT_F32>(hr + s * hr_stride, p.hrt + size_t(s) * I, I, true);
        for (int t = 0; t < T; ++t) stage_vec<WT, DT_F32>(hs + t * hs_stride, hsh + size_t(t) * Is, Is, true);
        if (threadIdx.x < NT) s_sg[threadIdx.x] = threadIdx.x < T ? __ldcg(sgate + threadIdx.x) : 0.0f;
        __syncthreads();
        // prefetch the next layer's router rows and shared gate/up rows of this warp's phase-A jobs
        if (l + 1 < p.n_layers && lane == 0) {
            const DecLayer& Nx = p.L[l + 1];
            for (int job = gw; job < jobsA; job += Wtot) {
                if (job < E) {
                    prefetch_l2(static_cast<const char*>(Nx.router_w) + size_t(job) * row_bytes(RT, H),
                                uint32_t(row_bytes(RT, H)));
                } else if (job > E) {
                    const int i = job - E - 1;
                    prefetch_l2(static_cast<const char*>(Nx.sh_gate) + size_t(i) * gate_row, uint32_t(gate_row));
                    prefetch_l2(static_cast<const char*>(Nx.sh_up) + size_t(i) * gate_row, uint32_t(gate_row));
                }
            }
        }
        const int nchI = I / Wv<WT>::V;
        const int nchS = Is / Wv<WT>::V;
        const int itemsR = U * nchI;
        const int items = itemsR + nchS;   // routed (expert, chunk) pairs, then shared chunks
        for (int r = 0; r < rowsC; ++r) {
            const int n = gw + r * Wtot;
            if (n >= H) break;
            float acc[NT] = {0.f, 0.f, 0.f, 0.f};
            for (int base = 0; base < items; base += 32 * CB) {
                uint4 wc[CB];
                float sc[CB];
#pragma unroll
                for (int b = 0; b < CB; ++b) {
                    const int it = base + b * 32 + lane;
                    wc[b] = make_uint4(0u, 0u, 0u, 0u);
                    sc[b] = 0.0f;
                    if (it < itemsR) {
                        const int u = it / nchI;
                        const int c = it - u * nchI;
                        const size_t row = size_t(s_ue[u]) * H + n;
                        wc[b] = ld_stream(static_cast<const char*>(Ly.w_down) + row * down_row + size_t(c) * 16);
                        sc[b] = (WT == DT_INT4) ? bf16f(ld_stream_u16(Ly.s_down + row * (I / 32) + c)) : 1.0f;
                    } else if (it < items) {
                        const int c = it - itemsR;
                        wc[b] = ld_stream(static_cast<const char*>(Ly.sh_down) + size_t(n) * sdown_row + size_t(c) * 16);
                        sc[b] = (WT == DT_INT4) ? bf16f(ld_stream_u16(Ly.sh_s_down + size_t(n) * (Is / 32) + c)) : 1.0f;
                    }
                }
#pragma unroll
                for (int b = 0; b < CB; ++b) {
                    const int it = base + b * 32 + lane;
                    if (it < itemsR) {
                        const int u = it / nchI;
                        const int c = it - u * nchI;
                        const unsigned mask = s_um[u];
#pragma unroll
                        for (int t = 0; t < NT; ++t) {
                            if (t < T && (mask >> t & 1u)) {
                                const int slot = s_us[u * NT + t];
                                const float d = chunk_dot<WT, DT_F32>(wc[b], hr + slot * hr_stride, c >> 5, c & 31);
                                acc[t] = fmaf(s_uw[u * NT + t] * sc[b], d, acc[t]);
                            }
                        }
                    } else if (it < items) {
                        const int c = it - itemsR;
#pragma unroll
                        for (int t = 0; t < NT; ++t)
                            if (t < T)
                                acc[t] = fmaf(s_sg[t] * sc[b], chunk_dot<WT, DT_F32>(wc[b], hs + t * hs_stride, c >> 5, c & 31), acc[t]);
                    }
                }
            }
#pragma unroll
            for (int t = 0; t < NT; ++t) acc[t] = warp_sum(acc[t]);
            if (lane == 0)
                for (int t = 0; t < T; ++t) Ly.out[size_t(t) * H + n] = acc[t];
        }
        if (l + 1 < p.n_layers) grid_barrier(p.ctl, nblocks, p.timeout_ns);
    }
}

struct Cfg {
    int xt, rt, wt;
};

template <int XT, int RT, int WT, int NL>
redmoe_status launch_one(const redmoe_layer* sh, const DecLayer* layers, int n_layers, int T, void* ws,
                         cudaStream_t stream) {
    DevInfo di;
    if (!get_dev_info(&di)) return REDMOE_ERR_CUDA;
    const Smem S = smem_layout(T, sh->hidden, sh->top_k, sh->inter, sh->shared_inter, XT, RT, WT);
    if (S.total > di.max_smem_optin) return REDMOE_ERR_UNSUPPORTED;
    auto kern = decode_kernel<XT, RT, WT, NL>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, S.total) != cudaSuccess)
        return REDMOE_ERR_CUDA;
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, THREADS, S.total) != cudaSuccess || per_sm < 1)
        return REDMOE_ERR_UNSUPPORTED;
    per_sm = per_sm > 2 ? 2 : per_sm;
    const int grid = di.sm_count * per_sm;

    DecParams<NL>* pp = new (std::nothrow) DecParams<NL>();
    if (!pp) return REDMOE_ERR_CUDA;
    DecParams<NL>& q = *pp;
    q.T = T; q.H = sh->hidden; q.E = sh->n_experts; q.k = sh->top_k; q.I = sh->inter; q.Is = sh->shared_inter;
    q.n_layers = n_layers;
    const DecodeWs L = decode_ws_layout(T, q.E, q.k, q.I, q.Is);
    char* base = static_cast<char*>(ws);
    q.ctl = reinterpret_cast<Control*>(base);
    q.logits = reinterpret_cast<float*>(base + L.logits);
    q.sgate = reinterpret_cast<float*>(base + L.sgate);
    q.hsh = reinterpret_cast<float*>(base + L.hsh);
    q.hrt = reinterpret_cast<float*>(base + L.hrt);
    q.timeout_ns = BARRIER_TIMEOUT_NS;
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

template <int XT, int RT, int WT>
redmoe_status launch_dt(const redmoe_layer* sh, const DecLayer* layers, int n_layers, int T, void* ws,
                        cudaStream_t stream, int* launches) {
    redmoe_status st = REDMOE_OK;
    if (n_layers == 1) {
        st = launch_one<XT, RT, WT, 1>(sh, layers, 1, T, ws, stream);
        if (st == REDMOE_OK && launches) *launches += 1;
        return st;
    }
    for (int l0 = 0; l0 < n_layers && st == REDMOE_OK; l0 += MAX_STACK) {
        const int n = n_layers - l0 < MAX_STACK ? n_layers - l0 : MAX_STACK;
        st = launch_one<XT, RT, WT, MAX_STACK>(sh, layers + l0, n, T, ws, stream);
        if (st == REDMOE_OK && launches) *launches += 1;
    }
    return st;
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

redmoe_status launch_decode(const redmoe_layer* sh, const DecLayer* layers, int n_layers, int T, void* ws,
                            cudaStream_t stream, int* launches) {
    const int xt = sh->x_dtype, rt = sh->router_dtype, wt = sh->expert_dtype;
    if (xt == DT_F32 && rt == DT_F32 && wt == DT_F32)
        return launch_dt<DT_F32, DT_F32, DT_F32>(sh, layers, n_layers, T, ws, stream, launches);
    if (xt == DT_BF16 && rt == DT_BF16 && wt == DT_BF16)
        return launch_dt<DT_BF16, DT_BF16, DT_BF16>(sh, layers, n_layers, T, ws, stream, launches);
    if (xt == DT_BF16 && rt == DT_BF16 && wt == DT_INT4)
        return launch_dt<DT_BF16, DT_BF16, DT_INT4>(sh, layers, n_layers, T, ws, stream, launches);
    return REDMOE_ERR_UNSUPPORTED;
}

}  // namespace redmoe
