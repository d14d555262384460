/*
 * fp64 CPU oracle of one sparse mixture-of-experts FFN layer (Qwen3-Next-80B-A3B shape).
 *
 * TEST INFRASTRUCTURE ONLY. The parity tests, the smoke check and the benchmark's
 * CPU-baseline leg are the only callers. The GPU library never links, loads or calls
 * this file, and this file includes nothing of the GPU library: the two share no
 * code, header, table or constant.
 *
 * Sources.
 *  - Shape: hidden 2048, 512 routed experts, top-10 routed experts per token, one
 *    shared expert, expert intermediate 512 ("Architecture", section "Qwen3-Next
 *    shape"; the guide "DwarfStar Red Lite", section "What runs": each of the 48
 *    layers picks 10 of 512 experts).
 *  - Router, top-k and shared gate form one stage, and the shared expert is one more
 *    expert slot ("Research notes, October 2026", section 1 "DwarfStar today", Metal
 *    bullets).
 *  - A double-precision implementation of the same graph is the parity gate, and a
 *    router top-k divergence is a hard failure (guide "DwarfStar Red Lite", section
 *    "Correctness"; "Red Lite dev18", section "Engine parity").
 *  - Exact router ties happen and two implementations may break them differently
 *    ("Red Lite dev18", section "Scope boundary": experts 403 and 101 at 0.0077861).
 *
 * The pages never write the layer's formula. This oracle takes the plainest reading
 * consistent with the shape facts above (every such reading is listed in the design
 * notes):
 *
 *   l[e]  = sum_h x[h] Wr[e,h]  (+ b[e] when a per-expert logit offset is given)
 *   p[e]  = exp(l[e] - max l) / sum_e' exp(l[e'] - max l)       softmax over all E
 *   ids   = the k experts of largest logit, ordered by (logit desc, id asc)
 *   w[j]  = p[ids_j] / sum_j' p[ids_j']                          renormalised
 *   s     = 1 / (1 + exp(-sum_h x[h] g[h]))                      shared-expert gate
 *   y_e   = Wd_e ( silu(Wg_e x) * (Wu_e x) ),  silu(a) = a / (1 + exp(-a))
 *   out   = sum_j w[j] y_{ids_j} + s y_shared
 *
 * and the token->expert grouping used by batched (prefill) execution: counts[e],
 * offsets = exclusive prefix sum, and the stable permutation that lists the rows
 * (t, j) routed to expert e in increasing token order, entry value t*k + j.
 *
 * Every stored input is widened exactly to double before use: bf16 -> f64 bit-exact,
 * int4 group-32 -> double(scale) * (nibble - 8). Loops run in the plain order of the
 * definitions above (h = 0..H-1, i = 0..I-1, j = 0..k-1); the only parallelism is
 * OpenMP over independent tokens, which does not change any result.
 *
 * Weight storage (all row-major): Wr [E,H]; g [H]; per routed expert Wg, Wu [I,H] and
 * Wd [H,I]; shared expert Wsg, Wsu [Is,H] and Wsd [H,Is]. int4 rows of K elements are
 * K/2 bytes (element 2b in the low nibble of byte b, 2b+1 in the high nibble) with
 * K/32 bf16 scales.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

enum { ORC_F32 = 0, ORC_BF16 = 1, ORC_INT4G32 = 2, ORC_INT2G32 = 3 };

enum {
    ORC_OK = 0,
    ORC_ERR_ARG = -1,         /* bad sizes, dtype or null pointer                  */
    ORC_ERR_MISSING = -2,     /* an expert the routing needs was not supplied      */
    ORC_ERR_NOMEM = -3
};

typedef struct {
    int32_t H, E, k, I, Is;
    int32_t x_dtype, router_dtype, expert_dtype;
    const void *router_w;             /* [E,H]                                         */
    const float *router_bias;         /* [E] or NULL                                   */
    const void *shared_gate_w;        /* [H]                                           */
    const void *const *gate;          /* E pointers, each [I,H]; NULL = not supplied   */
    const void *const *up;            /* E pointers, each [I,H]                        */
    const void *const *down;          /* E pointers, each [H,I]                        */
    const uint16_t *const *gate_scale;/* int4: E pointers to [I,H/32]; else NULL       */
    const uint16_t *const *up_scale;
    const uint16_t *const *down_scale;/* int4: E pointers to [H,I/32]                  */
    const void *sh_gate, *sh_up, *sh_down;
    const uint16_t *sh_gate_scale, *sh_up_scale, *sh_down_scale;
} orc_layer;

/* ------------------------------------------------------------------ widening */
static double bf16_bits_to_double(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* Scale of the 32-element group holding element (n, c) of a packed N x K matrix. */
static double group_scale(const uint16_t *scale, long K, long n, long c)
{
    return bf16_bits_to_double(scale[n * (K / 32) + c / 32]);
}

/* Element (n, c) of an N x K matrix stored in `dtype`. */
static double w_at(const void *w, const uint16_t *scale, int dtype, long K, long n, long c)
{
    switch (dtype) {
    case ORC_F32:
        return (double)((const float *)w)[n * K + c];
    case ORC_BF16:
        return bf16_bits_to_double(((const uint16_t *)w)[n * K + c]);
    case ORC_INT2G32: {
        uint8_t byte = ((const uint8_t *)w)[n * (K / 4) + c / 4];
        int code = (byte >> (2 * (c % 4))) & 3;
        return group_scale(scale, K, n, c) * (double)(code - 2);
    }
    default: {
        uint8_t byte = ((const uint8_t *)w)[n * (K / 2) + c / 2];
        int nibble = (c & 1) ? (byte >> 4) : (byte & 15);
        return group_scale(scale, K, n, c) * (double)(nibble - 8);
    }
    }
}

static double act_at(const void *x, int dtype, long i)
{
    if (dtype == ORC_F32)
        return (double)((const float *)x)[i];
    return bf16_bits_to_double(((const uint16_t *)x)[i]);
}

static int dtype_ok(int d, int allow_packed)
{
    return d == ORC_F32 || d == ORC_BF16 || (allow_packed && (d == ORC_INT4G32 || d == ORC_INT2G32));
}

static int shape_ok(const orc_layer *L)
{
    if (!L || L->H <= 0 || L->E <= 0 || L->k <= 0 || L->k > L->E || L->I <= 0 || L->Is <= 0)
        return 0;
    if (!dtype_ok(L->x_dtype, 0) || !dtype_ok(L->router_dtype, 0) || !dtype_ok(L->expert_dtype, 1))
        return 0;
    if ((L->expert_dtype == ORC_INT4G32 || L->expert_dtype == ORC_INT2G32) && (L->H % 32 || L->I % 32 || L->Is % 32))
        return 0;
    return 1;
}

int orc_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Threads of later calls (timing only: results do not depend on it). */
void orc_set_num_threads(int32_t n)
{
#ifdef _OPENMP
    if (n > 0)
        omp_set_num_threads(n);
#else
    (void)n;
#endif
}

/* ------------------------------------------------------------ int4 group-32 */
int orc_dequant_int4(int32_t N, int32_t K, const uint8_t *packed, const uint16_t *scales, double *out)
{
    if (N < 0 || K <= 0 || K % 32 || !packed || !scales || !out)
        return ORC_ERR_ARG;
    for (long n = 0; n < N; ++n)
        for (long c = 0; c < K; ++c)
            out[n * K + c] = w_at(packed, scales, ORC_INT4G32, K, n, c);
    return ORC_OK;
}

/* int2 group-32: element c of row n is scale[n][c/32] * (code - 2), the 2-bit code in
 * bits 2*(c%4) .. 2*(c%4)+1 of byte c/4. */
int orc_dequant_int2(int32_t N, int32_t K, const uint8_t *packed, const uint16_t *scales, double *out)
{
    if (N < 0 || K <= 0 || K % 32 || !packed || !scales || !out)
        return ORC_ERR_ARG;
    for (long n = 0; n < N; ++n)
        for (long c = 0; c < K; ++c)
            out[n * K + c] = w_at(packed, scales, ORC_INT2G32, K, n, c);
    return ORC_OK;
}

/* ------------------------------------------------------------------- router */
/* Top-k of one logit row by repeated selection: the j-th pick is the largest logit
 * not yet picked, the lower id winning an exact tie. */
static void topk_select(const double *l, int E, int k, int32_t *ids, unsigned char *taken)
{
    memset(taken, 0, (size_t)E);
    for (int j = 0; j < k; ++j) {
        int best = -1;
        for (int e = 0; e < E; ++e) {
            if (taken[e])
                continue;
            if (best < 0 || l[e] > l[best])
                best = e;
        }
        taken[best] = 1;
        ids[j] = best;
    }
}

/* Router stage for T tokens: logits, softmax probabilities, top-k ids, renormalised
 * weights and the shared-expert gate. Any output pointer except ids/w/s may be NULL. */
int orc_router(const orc_layer *L, int32_t T, const void *x,
               double *logits, double *probs, int32_t *ids, double *w, double *s)
{
    if (!shape_ok(L) || T < 0 || (T > 0 && (!x || !ids || !w || !s)) || !L->router_w || !L->shared_gate_w)
        return ORC_ERR_ARG;
    const int H = L->H, E = L->E, k = L->k;
    int err = ORC_OK;
#pragma omp parallel
    {
        double *l = (double *)malloc(sizeof(double) * (size_t)E);
        double *p = (double *)malloc(sizeof(double) * (size_t)E);
        unsigned char *taken = (unsigned char *)malloc((size_t)E);
        if (!l || !p || !taken) {
#pragma omp atomic write
            err = ORC_ERR_NOMEM;
        }
        /* every thread reaches the work-sharing loop; a thread without buffers skips */
#pragma omp for schedule(static)
        for (int t = 0; t < T; ++t) {
            if (l && p && taken) {
                for (int e = 0; e < E; ++e) {
                    double acc = 0.0;
                    for (int h = 0; h < H; ++h)
                        acc += act_at(x, L->x_dtype, (long)t * H + h) *
                               w_at(L->router_w, NULL, L->router_dtype, H, e, h);
                    if (L->router_bias)
                        acc += (double)L->router_bias[e];
                    l[e] = acc;
                }
                double m = l[0];
                for (int e = 1; e < E; ++e)
                    if (l[e] > m)
                        m = l[e];
                double z = 0.0;
                for (int e = 0; e < E; ++e)
                    z += exp(l[e] - m);
                for (int e = 0; e < E; ++e)
                    p[e] = exp(l[e] - m) / z;

                int32_t *id = ids + (long)t * k;
                topk_select(l, E, k, id, taken);
                double ps = 0.0;
                for (int j = 0; j < k; ++j)
                    ps += p[id[j]];
                for (int j = 0; j < k; ++j)
                    w[(long)t * k + j] = p[id[j]] / ps;

                double gx = 0.0;
                for (int h = 0; h < H; ++h)
                    gx += act_at(x, L->x_dtype, (long)t * H + h) *
                          w_at(L->shared_gate_w, NULL, L->router_dtype, H, 0, h);
                s[t] = 1.0 / (1.0 + exp(-gx));

                if (logits)
                    memcpy(logits + (long)t * E, l, sizeof(double) * (size_t)E);
                if (probs)
                    memcpy(probs + (long)t * E, p, sizeof(double) * (size_t)E);
            }
        }
        free(l);
        free(p);
        free(taken);
    }
    return err;
}

/* Renormalised weights of an arbitrary k-subset of one token's experts:
 * w[j] = p[ids_j] / sum_j' p[ids_j'] with p the softmax over all E logits. */
int orc_renorm(int32_t E, int32_t k, const double *logits_row, const int32_t *ids, double *w)
{
    if (E <= 0 || k <= 0 || k > E || !logits_row || !ids || !w)
        return ORC_ERR_ARG;
    double m = logits_row[0];
    for (int e = 1; e < E; ++e)
        if (logits_row[e] > m)
            m = logits_row[e];
    double z = 0.0;
    for (int e = 0; e < E; ++e)
        z += exp(logits_row[e] - m);
    double ps = 0.0;
    for (int j = 0; j < k; ++j) {
        if (ids[j] < 0 || ids[j] >= E)
            return ORC_ERR_ARG;
        ps += exp(logits_row[ids[j]] - m) / z;
    }
    for (int j = 0; j < k; ++j)
        w[j] = (exp(logits_row[ids[j]] - m) / z) / ps;
    return ORC_OK;
}

/* ------------------------------------------------------------ expert SwiGLU */
/* One SwiGLU expert on one token: a = Wg x, u = Wu x, h = silu(a) * u, y = Wd h.
 * gate/up are [I,H], down is [H,I]. `hbuf` holds I doubles. */
static void swiglu_expert(int H, int I, int dtype, const double *x,
                          const void *wg, const uint16_t *sg, const void *wu, const uint16_t *su,
                          const void *wd, const uint16_t *sd, double *hbuf, double *y)
{
    for (int i = 0; i < I; ++i) {
        double a = 0.0, u = 0.0;
        for (int h = 0; h < H; ++h) {
            a += w_at(wg, sg, dtype, H, i, h) * x[h];
            u += w_at(wu, su, dtype, H, i, h) * x[h];
        }
        hbuf[i] = a / (1.0 + exp(-a)) * u;
    }
    for (int h = 0; h < H; ++h) {
        double acc = 0.0;
        for (int i = 0; i < I; ++i)
            acc += w_at(wd, sd, dtype, I, h, i) * hbuf[i];
        y[h] = acc;
    }
}

static int expert_supplied(const orc_layer *L, int e)
{
    if (!L->gate || !L->up || !L->down || !L->gate[e] || !L->up[e] || !L->down[e])
        return 0;
    if (L->expert_dtype == ORC_INT4G32 &&
        (!L->gate_scale || !L->up_scale || !L->down_scale ||
         !L->gate_scale[e] || !L->up_scale[e] || !L->down_scale[e]))
        return 0;
    return 1;
}

static int shared_supplied(const orc_layer *L)
{
    if (!L->sh_gate || !L->sh_up || !L->sh_down)
        return 0;
    if (L->expert_dtype == ORC_INT4G32 && (!L->sh_gate_scale || !L->sh_up_scale || !L->sh_down_scale))
        return 0;
    return 1;
}

/* Output of one expert for one token given as doubles; e = -1 selects the shared expert. */
int orc_expert_ffn(const orc_layer *L, int32_t e, const double *x, double *y)
{
    if (!shape_ok(L) || !x || !y || e < -1 || e >= L->E)
        return ORC_ERR_ARG;
    if (e < 0 ? !shared_supplied(L) : !expert_supplied(L, e))
        return ORC_ERR_MISSING;
    int I = e < 0 ? L->Is : L->I;
    double *hbuf = (double *)malloc(sizeof(double) * (size_t)I);
    if (!hbuf)
        return ORC_ERR_NOMEM;
    if (e < 0)
        swiglu_expert(L->H, I, L->expert_dtype, x, L->sh_gate, L->sh_gate_scale, L->sh_up,
                      L->sh_up_scale, L->sh_down, L->sh_down_scale, hbuf, y);
    else
        swiglu_expert(L->H, I, L->expert_dtype, x, L->gate[e], L->gate_scale ? L->gate_scale[e] : NULL,
                      L->up[e], L->up_scale ? L->up_scale[e] : NULL, L->down[e],
                      L->down_scale ? L->down_scale[e] : NULL, hbuf, y);
    free(hbuf);
    return ORC_OK;
}

/* Weighted combine for T tokens with the routing given:
 * out[t] = sum_j w[t,j] y_{ids[t,j]}(x_t) + s[t] y_shared(x_t). */
int orc_experts(const orc_layer *L, int32_t T, const void *x, const int32_t *ids,
                const double *w, const double *s, double *out)
{
    if (!shape_ok(L) || T < 0 || (T > 0 && (!x || !ids || !w || !s || !out)))
        return ORC_ERR_ARG;
    if (!shared_supplied(L))
        return ORC_ERR_MISSING;
    for (long i = 0; i < (long)T * L->k; ++i) {
        if (ids[i] < 0 || ids[i] >= L->E)
            return ORC_ERR_ARG;
        if (!expert_supplied(L, ids[i]))
            return ORC_ERR_MISSING;
    }
    const int H = L->H, k = L->k;
    const int Imax = L->I > L->Is ? L->I : L->Is;
    int err = ORC_OK;
#pragma omp parallel
    {
        double *xd = (double *)malloc(sizeof(double) * (size_t)H);
        double *y = (double *)malloc(sizeof(double) * (size_t)H);
        double *hbuf = (double *)malloc(sizeof(double) * (size_t)Imax);
        if (!xd || !y || !hbuf) {
#pragma omp atomic write
            err = ORC_ERR_NOMEM;
        }
#pragma omp for schedule(dynamic, 1)
        for (int t = 0; t < T; ++t) {
            if (xd && y && hbuf) {
                for (int h = 0; h < H; ++h)
                    xd[h] = act_at(x, L->x_dtype, (long)t * H + h);
                double *o = out + (long)t * H;
                for (int h = 0; h < H; ++h)
                    o[h] = 0.0;
                for (int j = 0; j < k; ++j) {
                    int e = ids[(long)t * k + j];
                    swiglu_expert(H, L->I, L->expert_dtype, xd, L->gate[e],
                                  L->gate_scale ? L->gate_scale[e] : NULL, L->up[e],
                                  L->up_scale ? L->up_scale[e] : NULL, L->down[e],
                                  L->down_scale ? L->down_scale[e] : NULL, hbuf, y);
                    double wj = w[(long)t * k + j];
                    for (int h = 0; h < H; ++h)
                        o[h] += wj * y[h];
                }
                swiglu_expert(H, L->Is, L->expert_dtype, xd, L->sh_gate, L->sh_gate_scale, L->sh_up,
                              L->sh_up_scale, L->sh_down, L->sh_down_scale, hbuf, y);
                for (int h = 0; h < H; ++h)
                    o[h] += s[t] * y[h];
            }
        }
        free(xd);
        free(y);
        free(hbuf);
    }
    return err;
}

/* Whole layer: router stage, then the routed experts and the shared expert. */
int orc_forward(const orc_layer *L, int32_t T, const void *x, double *out, int32_t *ids,
                double *w, double *s, double *logits)
{
    int rc = orc_router(L, T, x, logits, NULL, ids, w, s);
    if (rc != ORC_OK)
        return rc;
    return orc_experts(L, T, x, ids, w, s, out);
}

/* ------------------------------------------------------------- brute force */
/* Dense reference for tiny shapes: every expert's output is computed (in the
 * outer-product loop order, not the dot-product order used above), the selection is
 * a full sort of the probability vector by (p desc, id asc), and the weights are
 * p / sum p over the selection. Needs every expert supplied. */
static const double *g_sort_p;
static int cmp_prob_desc(const void *a, const void *b)
{
    int ia = *(const int *)a, ib = *(const int *)b;
    if (g_sort_p[ia] > g_sort_p[ib])
        return -1;
    if (g_sort_p[ia] < g_sort_p[ib])
        return 1;
    return ia < ib ? -1 : (ia > ib);
}

static void expert_outer(int H, int I, int dtype, const double *x, const void *wg, const uint16_t *sg,
                         const void *wu, const uint16_t *su, const void *wd, const uint16_t *sd,
                         double *a, double *u, double *y)
{
    for (int i = 0; i < I; ++i)
        a[i] = u[i] = 0.0;
    for (int h = 0; h < H; ++h)
        for (int i = 0; i < I; ++i) {
            a[i] += x[h] * w_at(wg, sg, dtype, H, i, h);
            u[i] += x[h] * w_at(wu, su, dtype, H, i, h);
        }
    for (int h = 0; h < H; ++h)
        y[h] = 0.0;
    for (int i = 0; i < I; ++i) {
        double hv = a[i] * u[i] / (1.0 + exp(-a[i]));
        for (int h = 0; h < H; ++h)
            y[h] += w_at(wd, sd, dtype, I, h, i) * hv;
    }
}

int orc_brute(const orc_layer *L, int32_t T, const void *x, double *out, int32_t *ids, double *w)
{
    if (!shape_ok(L) || T < 0 || (T > 0 && (!x || !out || !ids || !w)))
        return ORC_ERR_ARG;
    for (int e = 0; e < L->E; ++e)
        if (!expert_supplied(L, e))
            return ORC_ERR_MISSING;
    if (!shared_supplied(L))
        return ORC_ERR_MISSING;
    const int H = L->H, E = L->E, k = L->k;
    const int Imax = L->I > L->Is ? L->I : L->Is;
    double *xd = malloc(sizeof(double) * (size_t)H);
    double *Y = malloc(sizeof(double) * (size_t)E * H);
    double *ysh = malloc(sizeof(double) * (size_t)H);
    double *a = malloc(sizeof(double) * (size_t)Imax);
    double *u = malloc(sizeof(double) * (size_t)Imax);
    double *p = malloc(sizeof(double) * (size_t)E);
    int *order = malloc(sizeof(int) * (size_t)E);
    int rc = ORC_OK;
    if (!xd || !Y || !ysh || !a || !u || !p || !order) {
        rc = ORC_ERR_NOMEM;
        goto done;
    }
    for (int t = 0; t < T; ++t) {
        for (int h = 0; h < H; ++h)
            xd[h] = act_at(x, L->x_dtype, (long)t * H + h);
        for (int e = 0; e < E; ++e)
            expert_outer(H, L->I, L->expert_dtype, xd, L->gate[e], L->gate_scale ? L->gate_scale[e] : NULL,
                         L->up[e], L->up_scale ? L->up_scale[e] : NULL, L->down[e],
                         L->down_scale ? L->down_scale[e] : NULL, a, u, Y + (long)e * H);
        expert_outer(H, L->Is, L->expert_dtype, xd, L->sh_gate, L->sh_gate_scale, L->sh_up,
                     L->sh_up_scale, L->sh_down, L->sh_down_scale, a, u, ysh);
        /* probabilities: exp of the logits over their sum (logits shifted by their max) */
        double m = -INFINITY, gx = 0.0;
        for (int e = 0; e < E; ++e) {
            double acc = L->router_bias ? (double)L->router_bias[e] : 0.0;
            for (int h = 0; h < H; ++h)
                acc += w_at(L->router_w, NULL, L->router_dtype, H, e, h) * xd[h];
            p[e] = acc;
            if (acc > m)
                m = acc;
        }
        double z = 0.0;
        for (int e = 0; e < E; ++e) {
            p[e] = exp(p[e] - m);
            z += p[e];
        }
        for (int e = 0; e < E; ++e) {
            p[e] /= z;
            order[e] = e;
        }
        g_sort_p = p;
        qsort(order, (size_t)E, sizeof(int), cmp_prob_desc);
        double ps = 0.0;
        for (int j = 0; j < k; ++j)
            ps += p[order[j]];
        for (int h = 0; h < H; ++h)
            gx += w_at(L->shared_gate_w, NULL, L->router_dtype, H, 0, h) * xd[h];
        double sg = 1.0 / (1.0 + exp(-gx));
        for (int h = 0; h < H; ++h)
            out[(long)t * H + h] = sg * ysh[h];
        for (int j = 0; j < k; ++j) {
            int e = order[j];
            ids[(long)t * k + j] = e;
            w[(long)t * k + j] = p[e] / ps;
            for (int h = 0; h < H; ++h)
                out[(long)t * H + h] += w[(long)t * k + j] * Y[(long)e * H + h];
        }
    }
done:
    free(xd); free(Y); free(ysh); free(a); free(u); free(p); free(order);
    return rc;
}

/* ------------------------------------------------------- token->expert grouping */
/* Stable counting sort of the T*k (token, slot) rows by expert:
 * counts[e] = number of rows routed to e; offsets[0] = 0, offsets[e+1] = offsets[e] +
 * counts[e] (E+1 entries); perm[offsets[e] + r] = t*k + j for the r-th row routed to e
 * in increasing (t, j) order. */
int orc_route_build(int32_t T, int32_t k, int32_t E, const int32_t *ids,
                    int32_t *counts, int32_t *offsets, int32_t *perm)
{
    if (T < 0 || k <= 0 || E <= 0 || !counts || !offsets || (T > 0 && (!ids || !perm)))
        return ORC_ERR_ARG;
    for (long i = 0; i < (long)T * k; ++i)
        if (ids[i] < 0 || ids[i] >= E)
            return ORC_ERR_ARG;
    for (int e = 0; e < E; ++e)
        counts[e] = 0;
    for (long i = 0; i < (long)T * k; ++i)
        counts[ids[i]] += 1;
    offsets[0] = 0;
    for (int e = 0; e < E; ++e)
        offsets[e + 1] = offsets[e] + counts[e];
    int32_t *cursor = malloc(sizeof(int32_t) * (size_t)E);
    if (!cursor)
        return ORC_ERR_NOMEM;
    for (int e = 0; e < E; ++e)
        cursor[e] = offsets[e];
    for (long i = 0; i < (long)T * k; ++i)
        perm[cursor[ids[i]]++] = (int32_t)i;
    free(cursor);
    return ORC_OK;
}

/* ------------------------------------------------- cache-aware routing (opt-in) */
/* Routing with a bias towards experts the caller holds in a cache ("Research notes,
 * October 2026", section 4, row "Cache-aware routing bias": z + lambda * Delta * cached,
 * opt-in only because it changes outputs). The pages give only that expression; this
 * oracle takes its plainest reading:
 *   z[e]       the token's router logits (offset included), as from orc_router;
 *   cached[e]  1 if expert e is resident in the caller's cache, else 0;
 *   Delta      the token's logit range, max_e z[e] - min_e z[e], so that lambda is
 *              dimensionless (lambda = 1 lets a cached expert at the lowest logit tie
 *              the best uncached one);
 *   selection  the k largest z[e] + lambda * Delta * cached[e], ties to the lower id;
 *   weights    the softmax of the unbiased z over all E restricted to the selection and
 *              renormalised: the bias changes which experts run, not how the selected
 *              experts' outputs are mixed.
 * lambda = 0 is plain routing. `biased` (T x E, may be NULL) receives the biased
 * logits the selection ranks. */
int orc_cache_route(int32_t T, int32_t E, int32_t k, const double *logits, const uint8_t *cached,
                    double lambda, int32_t *ids, double *w, double *biased)
{
    if (T < 0 || E <= 0 || k <= 0 || k > E || lambda < 0.0 || (T > 0 && (!logits || !cached || !ids || !w)))
        return ORC_ERR_ARG;
    double *zb = malloc(sizeof(double) * (size_t)E);
    unsigned char *taken = malloc((size_t)E);
    if (!zb || !taken) {
        free(zb);
        free(taken);
        return ORC_ERR_NOMEM;
    }
    for (long t = 0; t < T; ++t) {
        const double *z = logits + t * E;
        double zmax = z[0], zmin = z[0];
        for (int e = 1; e < E; ++e) {
            if (z[e] > zmax)
                zmax = z[e];
            if (z[e] < zmin)
                zmin = z[e];
        }
        const double delta = zmax - zmin;
        for (int e = 0; e < E; ++e)
            zb[e] = z[e] + lambda * delta * (cached[e] ? 1.0 : 0.0);
        if (biased)
            memcpy(biased + t * E, zb, sizeof(double) * (size_t)E);
        int32_t *id = ids + t * k;
        topk_select(zb, E, k, id, taken);
        /* softmax over all E of the unbiased logits, then the selection renormalised */
        double zsum = 0.0;
        for (int e = 0; e < E; ++e)
            zsum += exp(z[e] - zmax);
        double ps = 0.0;
        for (int j = 0; j < k; ++j)
            ps += exp(z[id[j]] - zmax) / zsum;
        for (int j = 0; j < k; ++j)
            w[t * k + j] = (exp(z[id[j]] - zmax) / zsum) / ps;
    }
    free(zb);
    free(taken);
    return ORC_OK;
}
