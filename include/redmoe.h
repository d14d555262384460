/*
 * redmoe.h -- C ABI of libredmoe.so: one sparse mixture-of-experts FFN layer on an
 * NVIDIA B200 (sm_100a), written for the Qwen3-Next-80B-A3B MoE block.
 *
 * The layer (shape from the "Architecture" page, section "Qwen3-Next shape": hidden
 * 2048, 512 routed experts, top-10 per token, one shared expert, expert intermediate
 * 512; the guide "DwarfStar Red Lite", section "What runs": every layer picks 10 of
 * 512 experts) computes, for each token row x of [T, H]:
 *
 *   l[e] = x . Wr[e] (+ b[e])            router logits over E experts
 *   ids  = the k largest logits, ordered by (logit desc, expert id asc)
 *   w[j] = softmax(l)[ids_j] / sum_j' softmax(l)[ids_j']     renormalised weights
 *   s    = sigmoid(x . g)                shared-expert gate
 *   y_e  = Wd_e (silu(Wg_e x) * (Wu_e x)) SwiGLU expert, silu(a) = a sigmoid(a)
 *   out  = sum_j w[j] y_{ids_j} + s y_shared
 *
 * The pages do not print this formula; it is the plainest reading of the shape facts
 * (softmax gating with renormalised top-k weights, SwiGLU experts, a sigmoid-gated
 * shared expert). Router, top-k and shared gate form one stage and the shared expert
 * is one more expert slot, as in the DwarfStar Metal kernels ("Research notes, October
 * 2026", section 1 "DwarfStar today").
 *
 * Conventions for every entry point:
 *  - Every tensor pointer is DEVICE memory owned by the caller; the library allocates
 *    no memory and keeps no state between calls except a per-device cache of device
 *    attributes and the fixed scratch array of redmoe_forward_noalloc (static memory in
 *    the library image). Tensors are dense, row-major, contiguous.
 *  - `stream` is a cudaStream_t (NULL: the legacy default stream). Work is only
 *    enqueued; no call synchronises the host except redmoe_check_timeout().
 *  - Arguments are validated on the host before anything is enqueued. On any error
 *    status nothing has been enqueued and no output has been touched (except
 *    REDMOE_ERR_CUDA, returned when a launch itself fails).
 *  - Pointers to weights and activations must be 16-byte aligned; int4 scale tensors
 *    2-byte aligned; id/count arrays 4-byte aligned.
 *  - No entry point aborts or throws; all failures are status codes.
 */
#ifndef REDMOE_H
#define REDMOE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define REDMOE_ABI_VERSION 1

typedef enum {
    REDMOE_OK = 0,
    REDMOE_ERR_INVALID_ARG = 1,   /* null/misaligned pointer, bad size, bad enum value      */
    REDMOE_ERR_UNSUPPORTED = 2,   /* valid arguments the library has no kernel for         */
    REDMOE_ERR_WORKSPACE = 3,     /* workspace null or smaller than redmoe_workspace_bytes  */
    REDMOE_ERR_CUDA = 4,          /* a CUDA runtime call or kernel launch failed            */
    REDMOE_ERR_TIMEOUT = 5        /* a bounded in-kernel wait ran out (see check_timeout)   */
} redmoe_status;

/* Storage types. REDMOE_INT4G32 (expert weights only): a matrix [N, K] is stored as
 * packed bytes [N, K/2] (element 2b in the low nibble of byte b, 2b+1 in the high
 * nibble, nibble = code + 8, codes -8..7) plus bf16 scales [N, K/32], one per 32
 * consecutive elements of a row; element value = scale * (nibble - 8). This format is
 * defined by this library (the pages ship GGUF IQ types only).
 * REDMOE_INT2G32 (expert weights only), this library's lower-bit counterpart (the pages
 * ship 2-bit expert files, guide "DwarfStar Red Lite", "Measured performance"): [N, K]
 * is stored as packed bytes [N, K/4] (elements 4b .. 4b+3 in bits 0-1, 2-3, 4-5, 6-7 of
 * byte b, code = q + 2, codes 0..3) plus bf16 scales [N, K/32]; element value =
 * scale * (code - 2). Supported at one token row (T = 1) with hidden 2048 and expert
 * intermediate 512; other sizes return REDMOE_ERR_UNSUPPORTED. */
typedef enum { REDMOE_F32 = 0, REDMOE_BF16 = 1, REDMOE_INT4G32 = 2, REDMOE_INT2G32 = 3 } redmoe_dtype;

/* One MoE layer. All tensors device-resident, row-major; E = n_experts, H = hidden,
 * I = inter, Is = shared_inter. The routed expert stacks keep the expert as the
 * outer dimension, like the merged blk.N.ffn_{gate,up,down}_exps tensors of the
 * "Red Lite v0.3 streaming development" page ("Implemented in dev1"). */
typedef struct redmoe_layer {
    int32_t hidden;          /* H, multiple of 64 (bf16/int4) or 32 (f32)                     */
    int32_t n_experts;       /* E, 1..1024                                                    */
    int32_t top_k;           /* k, 1..min(E, 32)                                              */
    int32_t inter;           /* I, multiple of 64 (int4: 32; f32: 32)                         */
    int32_t shared_inter;    /* Is, same rule as I                                            */
    int32_t x_dtype;         /* redmoe_dtype of x: F32 or BF16                                */
    int32_t router_dtype;    /* of router_w and shared_gate_w: F32 or BF16                    */
    int32_t expert_dtype;    /* of all routed and shared expert weights                       */
    const void *router_w;        /* [E, H]                                                    */
    const float *router_bias;    /* [E] fp32 per-expert logit offset, or NULL                 */
    const void *shared_gate_w;   /* [H]                                                       */
    const void *w_gate;          /* [E, I, H]   (int4: u8 [E, I, H/2]; int2: u8 [E, I, H/4])  */
    const void *w_up;            /* [E, I, H]   (as w_gate)                                   */
    const void *w_down;          /* [E, H, I]   (int4: u8 [E, H, I/2]; int2: u8 [E, H, I/4])  */
    const void *s_gate;          /* int4/int2: bf16 [E, I, H/32], 16-byte aligned; else NULL  */
    const void *s_up;            /* int4/int2: bf16 [E, I, H/32]                              */
    const void *s_down;          /* int4/int2: bf16 [E, H, I/32]                              */
    const void *sh_gate;         /* [Is, H]     (packed like the routed experts)              */
    const void *sh_up;           /* [Is, H]                                                   */
    const void *sh_down;         /* [H, Is]                                                   */
    const void *sh_s_gate;       /* int4/int2: bf16 [Is, H/32]; otherwise NULL                */
    const void *sh_s_up;         /* int4/int2: bf16 [Is, H/32]                                */
    const void *sh_s_down;       /* int4/int2: bf16 [H, Is/32]                                */
} redmoe_layer;

/* Optional device outputs of the token->expert grouping (see redmoe_route_build). */
typedef struct redmoe_route_debug {
    int32_t *counts;    /* [E]      */
    int32_t *offsets;   /* [E + 1]  */
    int32_t *perm;      /* [T * k]  */
} redmoe_route_debug;

/* ABI version of the loaded library (REDMOE_ABI_VERSION it was built with). */
int32_t redmoe_abi_version(void);

/* Static, NUL-terminated description of a status code; never NULL. */
const char *redmoe_status_string(int32_t status);

/* Bytes of workspace redmoe_forward / redmoe_router / redmoe_route_build need for this
 * layer at T tokens (a multiple of 256). Returns 0 if L is NULL or invalid or T < 0.
 * The workspace is caller-owned device memory, 256-byte aligned. Its first 256 bytes
 * are a control block that must be zero before the first use (redmoe_workspace_init
 * or a memset); every call leaves it zero again, except one that ran into
 * REDMOE_ERR_TIMEOUT, after which it must be re-initialised. Calls that share one
 * workspace must be ordered on the GPU (same stream or synchronised streams). */
size_t redmoe_workspace_bytes(const redmoe_layer *L, int32_t T);

/* Zero the control block of a workspace on `stream` (an async memset of 256 bytes).
 * workspace == NULL zeroes the control block of the current device's allocation-free
 * scratch (see redmoe_forward_noalloc) instead; workspace_bytes is then ignored. */
redmoe_status redmoe_workspace_init(void *workspace, size_t workspace_bytes, void *stream);

/* The whole layer for T token rows.
 *   x        [T, H] in L->x_dtype
 *   out      [T, H] fp32, overwritten (not accumulated)
 *   topk_ids [T, k] int32, expert ids ordered by logit descending, ties to the lower id
 *   topk_w   [T, k] fp32, renormalised weights in the same order (sum to 1 per row)
 *   dbg      NULL, or device arrays that receive the token->expert grouping
 * T == 0 is a valid empty call: nothing is enqueued. Decode sizes (T <= 4) run one
 * persistent kernel; larger T runs the batched path: a tensor-core router GEMM, top-k,
 * the grouping, and tensor-core grouped GEMMs for the experts (gate/up with SwiGLU,
 * then down with a weighted fp32 scatter-add into out, whose summation order is not
 * fixed). The batched path needs bf16 x, router and experts, shared_inter == inter,
 * hidden % 256 == 0 and inter % 128 == 0; other layers at T > 4 return
 * REDMOE_ERR_UNSUPPORTED. */
redmoe_status redmoe_forward(const redmoe_layer *L, const void *x, int32_t T, float *out,
                             int32_t *topk_ids, float *topk_w, void *workspace,
                             size_t workspace_bytes, const redmoe_route_debug *dbg, void *stream);

/* redmoe_forward with the opt-in cache-aware routing bias of "Research notes, October
 * 2026", section 4 ("Cache-aware routing bias (z + lambda * Delta * cached)", opt-in
 * only because it changes outputs). For a caller that keeps only some experts in a
 * fast tier and wants tokens to prefer those. The pages give only the expression; this
 * library's reading of it, which the oracle shares:
 *   cached   [E] uint8 device array: nonzero if the expert is resident in the caller's
 *            cache;
 *   lambda   >= 0 (finite); 0 gives exactly the routing of redmoe_forward;
 *   Delta    the token's logit range, max_e z[e] - min_e z[e] (router offsets included),
 *            which makes lambda dimensionless: with lambda > 1 and at least k cached
 *            experts only cached experts are selected;
 *   ids      the k largest z[e] + lambda * Delta * cached[e], ties to the lower id,
 *            ordered by that biased logit;
 *   weights  the softmax of the unbiased logits over all experts, restricted to the
 *            selection and renormalised (the bias changes which experts run, not how
 *            their outputs are mixed).
 * Other arguments, sizes and errors as redmoe_forward (no grouping debug output). */
redmoe_status redmoe_forward_cached(const redmoe_layer *L, const void *x, int32_t T, float *out,
                                    int32_t *topk_ids, float *topk_w, const uint8_t *cached, float lambda,
                                    void *workspace, size_t workspace_bytes, void *stream);

/* ---------------------------------------------------------------------------------
 * Routed experts in host memory, served through a bounded device cache.
 *
 * The pages keep the dense and shared weights resident and stream routed experts into a
 * bounded expert cache whose per-expert hotness is halved every 16 tokens ("Research
 * notes, October 2026", section 1, SSD streaming bullets), with router-driven prefetch for
 * the next MoE layer ("Architecture", "Future native Red Metal path"). Here the slow tier
 * is pinned host memory that the GPU reads over the host link, and the cache is a set of
 * device slots. All arrays below are caller-owned DEVICE memory, 16-byte aligned. */
typedef struct redmoe_expert_cache {
    int32_t n_slots;          /* S: slots, at least top_k                                     */
    void *slot_gate;          /* [S, I, H] in the layer's expert dtype (int4/int2: packed)     */
    void *slot_up;            /* [S, I, H]                                                     */
    void *slot_down;          /* [S, H, I]                                                     */
    void *slot_s_gate;        /* int4/int2: bf16 [S, I, H/32] scales; bf16 experts: NULL       */
    void *slot_s_up;          /* int4/int2: bf16 [S, I, H/32]                                  */
    void *slot_s_down;        /* int4/int2: bf16 [S, H, I/32]                                  */
    int32_t *slot_of;         /* [E]: slot holding expert e, or -1                             */
    int32_t *expert_in;       /* [S]: expert held by slot s, or -1                             */
    float *hot;               /* [E]: hotness, +1 per routed token, halved every 16 tokens     */
    int32_t *stats;           /* [4]: tokens, hits, misses (filled by calls), prefetch fills   */
    int32_t *fill;            /* [257]: the last call's fill list (count, then expert/slot)    */
} redmoe_expert_cache;

/* Bytes of one cache slot for this layer: one routed expert's three matrices, with int4 /
 * int2 scales (0 if the layer is invalid). slot_* arrays hold n_slots such experts. */
size_t redmoe_expert_cache_slot_bytes(const redmoe_layer *L);

/* Empty the cache on `stream`: every slot free, hotness and counters zero. */
redmoe_status redmoe_expert_cache_init(const redmoe_layer *L, redmoe_expert_cache *cache, void *stream);

/* redmoe_forward with the activations and results in HOST memory: the call a host
 * program makes per step. x_host [T, H] (L->x_dtype) is copied into the workspace's
 * device staging area with one cudaMemcpyAsync (any host memory; pinned keeps it
 * asynchronous). At decode sizes (T <= 4), when out_host, ids_host and w_host are pinned
 * (page-locked) host memory, the kernel stores the results straight into them through
 * their device mapping, so no copy back is enqueued; otherwise (T > 4, or pageable
 * outputs) the results go to device staging and three cudaMemcpyAsync bring them back.
 * Either way the results are in host memory once `stream` has reached the end of the
 * call: synchronise it before reading them. Same layouts, alignment rules (16 bytes for
 * x and out, 4 for ids and w) and statuses as redmoe_forward; the workspace must hold
 * redmoe_workspace_bytes_host(L, T) bytes (the forward's workspace, then the staging).
 * The arithmetic is redmoe_forward's; the pages have no separate counterpart. */
size_t redmoe_workspace_bytes_host(const redmoe_layer *L, int32_t T);
redmoe_status redmoe_forward_host(const redmoe_layer *L, const void *x_host, int32_t T, float *out_host,
                                  int32_t *ids_host, float *w_host, void *workspace, size_t workspace_bytes,
                                  void *stream);

/* redmoe_forward_stack with every x and every result in HOST memory (each array holds
 * n_layers host pointers and lives in host memory). At T = 1 on the one-row kernel's
 * layers, with every buffer pinned, the whole stack is one launch with no copy enqueued:
 * the kernel reads each layer's x over the link at the layer's start and stores its
 * results straight into the pinned buffers. Otherwise the layers run one after the other
 * as redmoe_forward_host calls. Same rules and statuses as redmoe_forward_stack; the
 * workspace must hold redmoe_workspace_bytes_host(&layers[0], T) bytes. The results are
 * in host memory once `stream` has reached the end of the call. */
redmoe_status redmoe_forward_stack_host(const redmoe_layer *layers, int32_t n_layers,
                                        const void *const *xs, int32_t T, float *const *outs,
                                        int32_t *const *ids, float *const *ws, void *workspace,
                                        size_t workspace_bytes, void *stream);

/* redmoe_forward for one token row (T = 1) whose routed expert stacks (w_gate, w_up,
 * w_down and their scales) may live in pinned host memory that the device can read
 * (cudaHostAlloc / cudaHostRegister, e.g. torch pin_memory); router, shared gate and
 * shared expert stay in device memory. Four launches on `stream`, no host round trip:
 * the router; a one-block directory update (hotness += 1 for each selected expert and
 * halved when the token count crosses a multiple of 16; each selected expert that is not
 * resident takes a free slot, else the slot of the resident expert with the lowest
 * hotness that this call does not use, ties to the lower slot); the copy of the missing
 * experts from host memory into their slots; the one-row decode kernel reading expert e
 * from slot slot_of[e] with the router's selection. The result is the layer's result
 * (the cache changes where weights are read from, never the arithmetic). Needs the
 * one-row kernel's layers (bf16 x/router; bf16, int4 or int2 experts; hidden <= 2048,
 * intermediate 512; top_k <= 11, n_experts <= 512): REDMOE_ERR_UNSUPPORTED otherwise or
 * for T != 1. REDMOE_ERR_INVALID_ARG if a routed stack is memory the device cannot read,
 * or the cache is malformed. Workspace: redmoe_workspace_bytes(L, 1). */
redmoe_status redmoe_forward_host_experts(const redmoe_layer *L, const void *x, int32_t T, float *out,
                                          int32_t *topk_ids, float *topk_w, redmoe_expert_cache *cache,
                                          void *workspace, size_t workspace_bytes, void *stream);

/* Router-driven prefetch: bring the n experts `ids` (device int32, 0 <= n <= 128, each in
 * [0, E)) into the cache on `stream` without counting them as used (no hotness, no
 * token), e.g. the experts the next layer's router picks from the current hidden state,
 * on a second stream while this layer computes. Victims are chosen as above; experts
 * already resident stay. Workspace: at least the 256-byte control block. */
redmoe_status redmoe_expert_cache_prefetch(const redmoe_layer *L, redmoe_expert_cache *cache, const int32_t *ids,
                                           int32_t n, void *workspace, size_t workspace_bytes, void *stream);

/* The router stage alone: logits, top-k ids, renormalised weights, shared gate.
 *   topk_ids [T, k] int32, topk_w [T, k] fp32, shared_gate [T] fp32 = sigmoid(x . g),
 *   logits [T, E] fp32 (router_bias included) or NULL. */
redmoe_status redmoe_router(const redmoe_layer *L, const void *x, int32_t T, int32_t *topk_ids,
                            float *topk_w, float *shared_gate, float *logits, void *workspace,
                            size_t workspace_bytes, void *stream);

/* Token->expert grouping of a [T, k] id matrix (k distinct ids per row, each in
 * [0, E)): counts[e] = rows routed to e; offsets[0] = 0, offsets[e+1] = offsets[e] +
 * counts[e]; perm[offsets[e] + r] = t*k + j for the r-th row (t, j) routed to e in
 * increasing t. Bit-exact and deterministic. The batched path of redmoe_forward uses
 * the same kernel. Out-of-range ids are not detected on the device: they are skipped
 * and the outputs are then unspecified. The kernel needs no scratch memory: workspace
 * and workspace_bytes are not used (pass NULL and 0); they keep the signature uniform
 * with the other entry points. */
redmoe_status redmoe_route_build(const int32_t *topk_ids, int32_t T, int32_t k, int32_t E,
                                 int32_t *counts, int32_t *offsets, int32_t *perm,
                                 void *workspace, size_t workspace_bytes, void *stream);

/* n_layers independent layers of the same shape and dtypes, one after the other on
 * `stream` (layer l reads xs[l] and writes outs[l], ids[l], ws[l]; each array holds
 * n_layers device pointers and lives in HOST memory). Equivalent to n_layers calls of
 * redmoe_forward; the decode sizes (T <= 4) run them in one persistent launch, which
 * lets the L2 prefetch of layer l+1's router and shared-expert weights overlap layer l. */
redmoe_status redmoe_forward_stack(const redmoe_layer *layers, int32_t n_layers,
                                   const void *const *xs, int32_t T, float *const *outs,
                                   int32_t *const *ids, float *const *ws, void *workspace,
                                   size_t workspace_bytes, void *stream);

/* redmoe_forward for decode sizes (1 <= T <= 4) without a caller workspace, for callers
 * that cannot allocate device memory: code inside a strict CUDA stream capture (where an
 * allocation breaks the capture), latency-critical loops that must not touch the
 * allocator, or plug-ins whose host framework owns the whole device memory budget.
 * There is no counterpart on the pages; it is a deployment convenience of this library.
 *
 * The scratch memory is a fixed 1 MiB array inside the library image; every GPU that
 * loads the library holds it until the process exits. Arguments and outputs are those of
 * redmoe_forward. The first call on each device looks up the array's device address
 * (cudaGetSymbolAddress, with that device current): make that first call outside any
 * stream capture. Nothing is allocated or freed. Each call clears the scratch's two
 * grid-barrier counters with an async 8-byte memset before the kernel; the error word
 * is kept, so a bounded in-kernel wait that gave up stays visible: read it with
 * redmoe_check_timeout(NULL, stream) and clear it with redmoe_workspace_init(NULL, 0,
 * stream); until then later calls may give up their own waits early and their outputs are
 * unspecified. All calls on a device share the array, so calls that can overlap on the GPU
 * race and must not be made; order them on one stream. Returns REDMOE_ERR_WORKSPACE if
 * the layer at this T needs more than the 1 MiB scratch, REDMOE_ERR_UNSUPPORTED for
 * T > 4, otherwise as redmoe_forward. */
redmoe_status redmoe_forward_noalloc(const redmoe_layer *L, const void *x, int32_t T, float *out,
                                     int32_t *topk_ids, float *topk_w, void *stream);

/* Synchronise `stream`, then read the workspace's error word: REDMOE_ERR_TIMEOUT if an
 * in-kernel grid barrier gave up waiting (bounded at about one second) since the last
 * redmoe_workspace_init; REDMOE_ERR_INVALID_ARG if a kernel found device state it cannot
 * use (an expert cache without a slot for a selected expert, an id out of range); else
 * REDMOE_OK. REDMOE_ERR_CUDA if the stream reports an error.
 * workspace == NULL reads the error word of the current device's allocation-free
 * scratch (redmoe_forward_noalloc). */
redmoe_status redmoe_check_timeout(const void *workspace, void *stream);

/* Self-test of the bounded in-kernel waits (the pages have no counterpart; this checks
 * the library's own failure reporting on a given device). Launches one cooperative
 * kernel of one 32-thread block per SM whose blocks meet at a grid barrier of the same
 * kind the layer kernels use. Block `withhold` (0 <= withhold < SM count) never arrives;
 * withhold < 0 lets every block arrive. Waiting blocks give up after limit_ns
 * (1 ns .. 1 s), record the timeout in the error word of `workspace` and return, so the
 * device stays usable. workspace == NULL uses the allocation-free scratch of the current
 * device. Afterwards redmoe_check_timeout reports REDMOE_ERR_TIMEOUT (withhold >= 0) or
 * REDMOE_OK (withhold < 0, unless an earlier timeout is still recorded); clear it with
 * redmoe_workspace_init. Returns REDMOE_ERR_INVALID_ARG for a limit or block index out of
 * range, REDMOE_ERR_WORKSPACE for a misaligned or short workspace. */
redmoe_status redmoe_selftest_wait_limit(void *workspace, size_t workspace_bytes, int32_t withhold,
                                         uint64_t limit_ns, void *stream);

/* Debugging aid (no counterpart on the pages): enqueue on `stream` one kernel that fills
 * the shared memory of every SM with the 32-bit `pattern` (0x7fc00000 is a quiet NaN).
 * The layer kernels launched next on that stream then start on that pattern instead of
 * on whatever an earlier launch left, so a kernel that reads its shared memory before the
 * data has arrived produces visibly wrong results on every call, not only on the first
 * call of a process. Not needed for correct use. */
redmoe_status redmoe_fill_shared_memory(uint32_t pattern, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* REDMOE_H */
