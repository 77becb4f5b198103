/*
 * moe.h -- C ABI of libmoe: one routed mixture-of-experts FFN layer on
 * ggml-style block-quantized expert weights, for NVIDIA B200 (sm_100a).
 *
 * The layer (what an MoE serving engine runs per token; FreeToken wiki
 * explainer, opening section: only a subset of experts is active per token):
 *
 *   logits  L = x . W_r (+ b)                         fp32
 *   S_t     = top-k experts of L[t,:], descending, ties -> lower expert id
 *   g[t,j]  = softmax(L[t,:])[S_tj] / sum_{i in S_t} softmax(L[t,:])[i]
 *   Y[t,j]  = W_down,e ( silu(W_gate,e x_t) * (W_up,e x_t) ),  e = S_tj
 *   y_t     = sum_j g[t,j] Y[t,j]  (+ shared expert, weight 1)
 *
 * Weight formats: the ggml Standard-family types Q4_0 and Q8_0 named in the
 * FreeToken fork README, "Quant types" table.  32 weights per block with
 * one fp16 scale d: Q8_0 = {fp16 d; int8 q[32]} (34 B), value q*d;
 * Q4_0 = {fp16 d; uint8 qs[16]} (18 B), value (q-8)*d, byte j holding
 * element j in its low nibble and element j+16 in its high nibble.
 * Expert pool (FreeToken fork README, "Known limits"): one allocation per
 * matrix kind, experts back to back as slot * nrows * (ncols / 32) blocks,
 * no padding, ONE quant type for the whole pool.  Per slot:
 *   gate, up : [F rows][D/32 blocks]      down : [D rows][F/32 blocks]
 * so every row is contiguous along its reduction dimension.
 *
 * Conventions shared by every call:
 *  - Every call returns a moe_status; on anything but MOE_OK,
 *    moe_last_error() (thread-local) holds a one-line reason, and no kernel
 *    of the failing call was enqueued.  Every dispatch on a quant type or
 *    dtype has an erroring default (the FreeToken fork README, "What else
 *    changed", reports silent garbage from switches without one).
 *  - Calls only ENQUEUE work on the stream they are given and return; the
 *    stream is a cudaStream_t (NULL = the legacy default stream).
 *  - Device buffers are allocated and owned by the caller.  Calls allocate
 *    no device memory; scratch comes in through (workspace, ws_bytes), whose
 *    required size the matching *_workspace_size() reports.  A workspace must
 *    be zero-filled once before its first use; every call leaves it in a
 *    state the next call accepts.  Calls that share a workspace must be
 *    ordered (same stream, or synchronised).
 *  - Shapes: D % 32 == 0, F % 32 == 0 (blocks run along the reduction
 *    dimension), 1 <= k <= E <= MOE_MAX_EXPERTS, k <= MOE_MAX_TOPK, T >= 0.
 *    T == 0 is a no-op that succeeds.
 *  - Pointers named "device" must be device memory (or managed); "host"
 *    means host memory (pinned where stated).
 */
#ifndef MOE_H
#define MOE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define MOE_QK 32
#define MOE_Q4_0_BLOCK_BYTES 18
#define MOE_Q8_0_BLOCK_BYTES 34
#define MOE_MAX_EXPERTS 1024
#define MOE_MAX_TOPK 32

typedef enum {
    MOE_OK = 0,
    MOE_ERR_INVALID_ARG = 1,        /* null pointer, bad enum, bad flag */
    MOE_ERR_UNSUPPORTED_QTYPE = 2,  /* quant type not Q4_0 / Q8_0, or mixed */
    MOE_ERR_SHAPE = 3,              /* a size rule above is broken */
    MOE_ERR_CUDA = 4,               /* a CUDA runtime call failed */
    MOE_ERR_CAPACITY = 5,           /* more experts requested than cache slots */
    MOE_ERR_TIMEOUT = 6,            /* a bounded host wait ran out */
    MOE_ERR_WORKSPACE = 7           /* workspace missing or too small */
} moe_status;

/* ggml type ids */
typedef enum { MOE_Q4_0 = 2, MOE_Q8_0 = 8 } moe_qtype;

typedef enum { MOE_F32 = 0, MOE_BF16 = 1, MOE_F16 = 2 } moe_dtype;

/* Same type as cudaStream_t. */
typedef struct CUstream_st *moe_stream;

/* A device expert pool (see the layout above).  slot_of_expert maps expert
 * id -> slot (device int32[E]); NULL means slot = expert id.  Every expert
 * that a call reaches must map to a slot in [0, n_slots). */
typedef struct {
    int32_t qtype;                  /* moe_qtype */
    int32_t n_slots;
    const void *gate;               /* device, n_slots * F * (D/32) blocks */
    const void *up;                 /* device, n_slots * F * (D/32) blocks */
    const void *down;               /* device, n_slots * D * (F/32) blocks */
    const int32_t *slot_of_expert;  /* device int32[E] or NULL */
} moe_pool;

/* ---------------------------------------------------------------- misc */
const char *moe_last_error(void);
const char *moe_version(void);
/* Bytes of one 32-weight block of a quant type; 0 for an unknown type. */
int moe_block_bytes(int32_t qtype);

/* ------------------------------------------------------------- routing
 * moe_route: router logits, softmax, top-k and renormalised gates.
 *   x        device [T, D], x_dtype F32 or BF16 (row-major).  When w_router
 *            is NULL, x instead holds the logits [T, E] in F32 and D is
 *            ignored (routing from given logits).
 *   w_router device [D, E] fp32 row-major, or NULL (see x).
 *   bias     device [E] fp32 or NULL; added to the logits, so it moves both
 *            the selection and the softmax.
 *   renorm   1: g = p_S / sum(p_S) (the gates sum to 1); 0: g = p_S.
 *   ids      device int32 [T, k]: selected experts, descending logit, ties
 *            to the lower expert id.
 *   gates    device fp32 [T, k].
 *   logits   device fp32 [T, E] or NULL: the logits as computed (fp32
 *            accumulation), for tie diagnostics.
 * Logits are accumulated in fp32.  Non-finite logits give unspecified ids. */
size_t moe_route_workspace_size(int T, int D, int E, int k);
moe_status moe_route(const void *x, int32_t x_dtype, const float *w_router,
                     const float *bias, int T, int D, int E, int k, int renorm,
                     int32_t *ids, float *gates, float *logits,
                     void *workspace, size_t ws_bytes, moe_stream stream);

/* moe_route_noalloc: the same routing as moe_route for small batches, for
 * callers that cannot allocate device memory when they route (code running
 * inside an allocator's own callbacks, serving loops that freeze their
 * memory footprint after start-up, embedders whose runtime owns every
 * device allocation and lends no scratch buffer).  It takes no workspace:
 * its scratch is a fixed array inside the library, 2 MiB per GPU that loads
 * the library, held until the process exits.  The pages have no counterpart
 * to this entry point; it exists for such callers only.
 *   Arguments as moe_route, except: w_router must not be NULL, and
 *   T <= 16 and ceil(D/32) * T * E <= 524288 (else MOE_ERR_SHAPE, with the
 *   limit in the message).
 *   The first call on each device looks up the array's device address
 *   (cudaGetSymbolAddress) with that device current; make that first call
 *   before capturing any stream.  Every call on a device shares the array
 *   and leaves its contents behind (the completion counter is cleared at the
 *   start of each call); calls that overlap on the GPU race, so serialise
 *   them (one stream, or events between streams). */
moe_status moe_route_noalloc(const void *x, int32_t x_dtype, const float *w_router,
                             const float *bias, int T, int D, int E, int k, int renorm,
                             int32_t *ids, float *gates, float *logits, moe_stream stream);

/* --------------------------------------------------------- permutation
 * moe_permute: stable grouping of the T*k (token, slot) entries by expert.
 *   ids     device int32 [T, k], each in [0, E).
 *   counts  device int32 [E]      entries per expert.
 *   offsets device int32 [E + 1]  exclusive prefix sum, offsets[E] = T*k.
 *   perm    device int32 [T*k]    perm[pos] = t*k + j, sorted by
 *                                 (expert, t, j).
 *   inv     device int32 [T*k]    inv[t*k + j] = pos.
 * Deterministic (no atomics decide an order).  Ids outside [0, E) are
 * dropped (not counted; their perm/inv entries are left unwritten): the
 * kernel cannot report them, so validate ids upstream (moe_route only
 * writes ids in range). */
moe_status moe_permute(const int32_t *ids, int T, int k, int E, int32_t *counts,
                       int32_t *offsets, int32_t *perm, int32_t *inv,
                       moe_stream stream);

/* ---------------------------------------------------------- expert FFN
 * moe_expert_ffn: per permuted row pos (token t = perm[pos] / k, expert e =
 * the segment of offsets that holds pos):
 *   out_rows[pos, :] = W_down,e ( silu(W_gate,e x_t) * (W_up,e x_t) )
 * (no gate weight; moe_combine applies it).
 *   x           device [T, D], x_dtype F32 or BF16.
 *   perm,offsets from moe_permute.
 *   pool        expert weights (see moe_pool); pool->qtype fixes the format.
 *   expert_mask device uint8 [E] or NULL: when given, only rows of experts
 *               with a nonzero mask are computed and the others are left
 *               untouched (two-phase runs: resident experts first, then the
 *               experts whose copies just landed).
 *   out_rows    device fp32 [T*k, D], permuted order.
 * Each row is computed by the same kernels in the same order whatever the
 * mask or the other rows, so a row's bits do not depend on the phase split. */
size_t moe_expert_ffn_workspace_size(int T, int k, int D, int F);
moe_status moe_expert_ffn(const void *x, int32_t x_dtype, int T, int D, int F,
                          int E, int k, const int32_t *perm,
                          const int32_t *offsets, const moe_pool *pool,
                          const uint8_t *expert_mask, float *out_rows,
                          void *workspace, size_t ws_bytes, moe_stream stream);

/* ------------------------------------------------------------- combine
 * moe_combine: y[t, :] = sum_{j<k} gates[t,j] * rows[inv[t*k+j], :]
 *                        (+ shared_rows[t, :]),
 * summed in fp32 in j order, written as y_dtype (F32, BF16 or F16).
 *   rows        device fp32 [T*k, D] (moe_expert_ffn output).
 *   shared_rows device fp32 [T, D] or NULL. */
moe_status moe_combine(const float *rows, const int32_t *inv, const float *gates,
                       int T, int k, int D, const float *shared_rows, void *y,
                       int32_t y_dtype, moe_stream stream);

/* ------------------------------------------------------ fused forward
 * moe_layer_forward: the whole layer in one call (routing, permutation,
 * expert FFNs, gate-weighted combine, optional shared expert), with the
 * fused kernels: small T takes the dequant-fused grouped GEMV path, large T
 * the grouped tensor-core GEMM path.  Results equal the step-by-step calls
 * up to fp32 rounding order.
 * Fields of moe_layer_args:
 *   T, D, E, k, F        shapes (shared_F for the shared expert, 0 = none)
 *   renorm               as moe_route
 *   x, x_dtype           device [T, D] activations (F32 or BF16)
 *   w_router, bias       as moe_route; w_router NULL -> logits_in is used
 *   logits_in            device fp32 [T, E] or NULL
 *   pool                 routed experts
 *   shared               NULL or a pool with one slot (Q8_0 or Q4_0) of a
 *                        SwiGLU expert with F = shared_F, added with weight 1
 *   y, y_dtype           device [T, D] output (F32 or BF16)
 *   ids_out, gates_out   device [T, k] or NULL: routing decisions
 *   logits_out           device fp32 [T, E] or NULL
 *   trace                NULL, or per-kernel timing of this call (moe_trace) */

/* Per-kernel timing of one moe_layer_forward call.  The caller creates
 * `capacity` CUDA events (cudaEvent_t, timing enabled) and passes them in
 * `events`; the call records events[i] on the stream right before its i-th
 * kernel and one more after the last, so kernel i ran between events[i] and
 * events[i+1] (read with cudaEventElapsedTime after the stream is done).
 * On return `count` holds the number of events recorded and kinds[i] the
 * moe_kernel_kind of kernel i.  A capacity too small for the call's kernels
 * is MOE_ERR_INVALID_ARG.  Recording adds a few hundred ns per kernel. */
typedef enum {
    MOE_KERNEL_ROUTE = 1,          /* logits + top-k in one kernel (small T) */
    MOE_KERNEL_ROUTE_LOGITS = 2,   /* tiled router GEMM (large T) */
    MOE_KERNEL_ROUTE_SELECT = 3,   /* top-k + gates from logits */
    MOE_KERNEL_PERMUTE = 4,
    MOE_KERNEL_GATEUP = 5,         /* gate/up GEMM(V) + SwiGLU */
    MOE_KERNEL_DOWN = 6,           /* down GEMM(V) (+ fused combine) */
    MOE_KERNEL_COMBINE = 7,
    MOE_KERNEL_SHARED_GATEUP = 8,
    MOE_KERNEL_SHARED_DOWN = 9,
    MOE_KERNEL_CONVERT = 10,       /* activation cast for the tensor-core path */
    MOE_KERNEL_ZERO = 11,          /* accumulator clear */
    MOE_KERNEL_FFN_DECODE = 12     /* decode gate/up + down (+combine) pair; the
                                      two kernels overlap through programmatic
                                      dependent launch, so they are timed as one */
} moe_kernel_kind;

#define MOE_TRACE_MAX 24
typedef struct {
    void **events;
    int32_t capacity;
    int32_t count;
    int32_t kinds[MOE_TRACE_MAX];
} moe_trace;

typedef struct {
    int32_t T, D, E, k, F, shared_F;
    int32_t renorm;
    int32_t x_dtype;
    int32_t y_dtype;
    int32_t reserved;
    const void *x;
    const float *w_router;
    const float *bias;
    const float *logits_in;
    const moe_pool *pool;
    const moe_pool *shared;
    void *y;
    int32_t *ids_out;
    float *gates_out;
    float *logits_out;
    moe_trace *trace;
} moe_layer_args;

size_t moe_layer_workspace_size(const moe_layer_args *args);
moe_status moe_layer_forward(const moe_layer_args *args, void *workspace,
                             size_t ws_bytes, moe_stream stream);

/* --------------------------------------------------------- expert cache
 * A per-layer HBM cache of expert slots fed from a pinned host pool (VRAM as
 * a cache over the full expert set held in host RAM: FreeToken fork README,
 * "About" (global LRU expert caching); kongchang article, "From Static
 * Allocation to Dynamic Scheduling").  Each layer has n_slots device slots;
 * replacement is least-recently-used:
 *  - every requested expert is stamped with the request's step number;
 *  - a missing expert takes the empty slot of lowest index, else evicts the
 *    resident expert with the oldest stamp that is not requested in the
 *    same call, the lower expert id on equal stamps;
 *  - ids are served in the order given.
 * Misses are copied host-to-device with cudaMemcpyAsync on the cache's copy
 * stream, after the copy stream has waited for the compute stream (so a
 * victim slot is never overwritten while a kernel may still read it).
 *
 * moe_cache_desc (all pools in the layout above; sizes in bytes):
 *   n_layers, E, n_slots, qtype
 *   bytes_gate, bytes_up, bytes_down   one expert's bytes of each matrix
 *   host_gate/up/down   host arrays of n_layers pointers, each to pinned
 *                       [E] experts (expert e at e * bytes_*)
 *   dev_gate/up/down    device [n_layers][n_slots] slots
 *   dev_slot_map        device int32 [n_layers][E]; entries of experts that
 *                       are not resident hold -1
 *   copy_stream         stream for the host-to-device copies (not NULL)
 * The cache keeps pointers to the caller's buffers; they must outlive it. */
typedef struct moe_cache moe_cache;
typedef struct {
    int32_t n_layers, E, n_slots, qtype;
    size_t bytes_gate, bytes_up, bytes_down;
    const void *const *host_gate;
    const void *const *host_up;
    const void *const *host_down;
    void *dev_gate;
    void *dev_up;
    void *dev_down;
    int32_t *dev_slot_map;
    moe_stream copy_stream;
} moe_cache_desc;

moe_status moe_cache_init(const moe_cache_desc *desc, moe_cache **out);
void moe_cache_destroy(moe_cache *cache);
/* Serve one request of n distinct expert ids (host int32) for `layer`:
 * runs the LRU on the host, enqueues the copies of the misses on the copy
 * stream, records the layer's copy event, and enqueues on `compute` the
 * update of the layer's device slot map.  Optional host outputs per id:
 * slots[n], miss[n] (0/1), evicted[n] (expert evicted or -1).
 * MOE_ERR_CAPACITY if n > n_slots; MOE_ERR_INVALID_ARG on a bad or repeated
 * id.  The cache state is unchanged on error. */
moe_status moe_cache_request(moe_cache *cache, int layer, const int32_t *ids,
                             int n, int32_t *slots, int32_t *miss,
                             int32_t *evicted, int *n_miss, moe_stream compute);
/* Make `compute` wait for the copies of the layer's last request. */
moe_status moe_cache_sync(moe_cache *cache, int layer, moe_stream compute);
/* Optional: every kernel that reads the layer's slots for its last request
 * has been enqueued on `compute` (call it after the layer's FFN).  Records an
 * event there; the layer's next request then starts its miss copies as soon
 * as that work is done, instead of after everything enqueued on `compute`
 * up to the request, so copies for later layers overlap the FFN of earlier
 * ones.  Consumed by that next request (without a new call, the request
 * falls back to waiting for all of `compute`).  MOE_ERR_INVALID_ARG on a bad
 * cache or layer. */
moe_status moe_cache_release(moe_cache *cache, int layer, moe_stream compute);
/* The device pool view of one layer (slot-mapped). */
moe_status moe_cache_layer_pool(moe_cache *cache, int layer, moe_pool *out);
moe_status moe_cache_stats(moe_cache *cache, int64_t *hits, int64_t *misses,
                           int64_t *bytes_copied);

#ifdef __cplusplus
}
#endif
#endif /* MOE_H */
