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
 * Weight formats: the ggml Standard-family types Q4_0, Q4_1, Q5_0, Q5_1 and
 * Q8_0 named in the FreeToken fork README, "Quant types" table (the page
 * names the types; the byte layouts are ggml's published ones).  32 weights
 * per block, an fp16 scale d and, for the _1 types, an fp16 minimum m; all
 * fields little endian:
 *   Q8_0 = {fp16 d; int8 q[32]}                       (34 B) value q*d
 *   Q4_0 = {fp16 d; uint8 qs[16]}                     (18 B) value (q-8)*d
 *   Q4_1 = {fp16 d; fp16 m; uint8 qs[16]}             (20 B) value q*d + m
 *   Q5_0 = {fp16 d; uint8 qh[4]; uint8 qs[16]}        (22 B) value (q-16)*d
 *   Q5_1 = {fp16 d; fp16 m; uint8 qh[4]; uint8 qs[16]} (24 B) value q*d + m
 * qs byte j holds the low four bits of element j (low nibble) and of element
 * j+16 (high nibble); bit i of the 32-bit word qh is bit 4 of element i.
 * K-quants (the same table, K-quants row; ggml's published layouts), 256
 * weights per block:
 *   Q4_K = {fp16 d; fp16 dmin; uint8 scales[12]; uint8 qs[128]}  (144 B):
 *          eight 32-weight sub-blocks j with 6-bit scale sc_j and min m_j
 *          (j < 4: low six bits of scales[j], scales[j+4]; j >= 4: low and
 *          high nibble of scales[j+4] plus the top two bits of scales[j-4]
 *          and scales[j]); value d*sc_j*q - dmin*m_j; weight 64c+l is the
 *          low nibble of qs[32c+l], weight 64c+32+l its high nibble.
 *   Q6_K = {uint8 ql[128]; uint8 qh[64]; int8 scales[16]; fp16 d} (210 B):
 *          value d*scales[i/16]*(q_i - 32); weight 128h+32r+l has its low
 *          four bits in nibble r/2 of ql[64h+32(r%2)+l] and its high two in
 *          bits 2r, 2r+1 of qh[32h+l].
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
 *  - Shapes: D and F multiples of the block (32 weights; 256 for the
 *    K-quants: blocks run along the reduction dimension), 1 <= k <= E <=
 *    MOE_MAX_EXPERTS, k <= MOE_MAX_TOPK, T >= 0.
 *    T == 0 is a no-op that succeeds.
 *  - Errors found on the GPU (a bounded wait inside a kernel that ran out,
 *    an expert whose slot is outside [0, n_slots)) cannot be returned by the
 *    enqueuing call.  The kernels record the first such error in a status
 *    word: the first int32 of the workspace.  moe_workspace_status() reads
 *    it (and can clear it); a new workspace is zero-filled, so it starts at
 *    MOE_DEV_OK.  A kernel that records an error skips the work it concerns
 *    and returns; the outputs that work would have written are unspecified,
 *    every other output is exact.
 *  - Numerics: the decode kernels apply block scales (and minimums) to fp32
 *    partial sums of exact codes; the tensor-core kernels round each weight
 *    to fp16 (Q4_K: its sub-block scale and minimum first).  Activations (x)
 *    and the hidden rows h are rounded to fp16 inside the FFN kernels (bf16 has 8 significant bits, fp16 11, so a bf16
 *    x in fp16's normal range [2^-14, 65504] converts exactly).  Inputs
 *    with |x| > 65504 overflow to inf and values under 2^-14 lose bits;
 *    keep activations inside that range (post-normalisation hidden states
 *    are).  Routing stays fp32 throughout.
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
#define MOE_Q4_1_BLOCK_BYTES 20
#define MOE_Q5_0_BLOCK_BYTES 22
#define MOE_Q5_1_BLOCK_BYTES 24
#define MOE_Q8_0_BLOCK_BYTES 34
#define MOE_QK_K 256
#define MOE_Q4_K_BLOCK_BYTES 144
#define MOE_Q6_K_BLOCK_BYTES 210
#define MOE_MAX_EXPERTS 1024
#define MOE_MAX_TOPK 32

typedef enum {
    MOE_OK = 0,
    MOE_ERR_INVALID_ARG = 1,        /* null pointer, bad enum, bad flag */
    MOE_ERR_UNSUPPORTED_QTYPE = 2,  /* quant type not one of moe_qtype */
    MOE_ERR_SHAPE = 3,              /* a size rule above is broken */
    MOE_ERR_CUDA = 4,               /* a CUDA runtime call failed */
    MOE_ERR_CAPACITY = 5,           /* more experts requested than cache slots */
    MOE_ERR_TIMEOUT = 6,            /* a bounded host wait ran out */
    MOE_ERR_WORKSPACE = 7           /* workspace missing or too small */
} moe_status;

/* Codes of the device status word (see moe_workspace_status). */
typedef enum {
    MOE_DEV_OK = 0,
    MOE_DEV_TIMEOUT_FULL = 1,      /* a consumer waited too long for data */
    MOE_DEV_TIMEOUT_EMPTY = 2,     /* a producer waited too long for a free buffer */
    MOE_DEV_TIMEOUT_DRAIN = 3,     /* copies still in flight at exit waited too long */
    MOE_DEV_BAD_SLOT = 4,          /* an expert with tokens maps outside [0, n_slots) */
    MOE_DEV_TIMEOUT_MMA = 5        /* tensor-core work did not complete in time */
} moe_device_status;

/* ggml type ids */
typedef enum {
    MOE_Q4_0 = 2, MOE_Q4_1 = 3, MOE_Q5_0 = 6, MOE_Q5_1 = 7, MOE_Q8_0 = 8,
    MOE_Q4_K = 12, MOE_Q6_K = 14
} moe_qtype;

typedef enum { MOE_F32 = 0, MOE_BF16 = 1, MOE_F16 = 2 } moe_dtype;

/* Same type as cudaStream_t. */
typedef struct CUstream_st *moe_stream;

/* A device expert pool (see the layout above).  slot_of_expert maps expert
 * id -> slot (device int32[E]); NULL means slot = expert id.  Every expert
 * that a call reaches (tokens routed to it, and not masked out) must map to
 * a slot in [0, n_slots): the kernels check each one before forming any
 * address, skip an expert that does not, and record MOE_DEV_BAD_SLOT in the
 * workspace's status word (an expert cache marks non-resident experts -1). */
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
/* Bytes of one block of a quant type; 0 for an unknown type. */
int moe_block_bytes(int32_t qtype);
/* Weights of one block of a quant type (32, or 256 for the K-quants); 0 for
 * an unknown type. */
int moe_block_weights(int32_t qtype);

/* moe_selftest_wait_timeout: exercises the kernels' bounded-wait path.  One
 * warp waits, with the same wait routine the FFN kernels use, on a shared-
 * memory barrier that nothing arrives at, for budget_cycles SM clock cycles
 * (1 .. 4e9); the wait runs out, records MOE_DEV_TIMEOUT_FULL in the status
 * word of `workspace` (device, >= 64 bytes, as moe_workspace_status reads it)
 * and the kernel returns: no fault, no hang, the context stays usable.
 * Enqueues one kernel on `stream`; MOE_ERR_INVALID_ARG for a budget out of
 * range, MOE_ERR_WORKSPACE for a missing or short workspace. */
moe_status moe_selftest_wait_timeout(void *workspace, size_t ws_bytes, int64_t budget_cycles,
                                     moe_stream stream);

/* moe_workspace_status: the device status word of a workspace (its first
 * int32, written by the kernels of the calls that used it; see the
 * conventions above).  Waits for the work enqueued on `stream` so far, then
 * stores the word in *code (a moe_device_status) and, if clear != 0, resets
 * it to MOE_DEV_OK (the reset is enqueued on `stream` and waited for).
 * Returns MOE_OK when the word is MOE_DEV_OK, MOE_ERR_TIMEOUT for the
 * timeout codes, MOE_ERR_INVALID_ARG for MOE_DEV_BAD_SLOT (with a message),
 * MOE_ERR_CUDA if the copy fails.  Blocks the calling thread; not for use
 * inside stream capture. */
moe_status moe_workspace_status(void *workspace, int32_t *code, int clear, moe_stream stream);

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
 *   (cudaGetSymbolAddress) with that device current.  Under CUDA's lazy
 *   module loading (the default) that first call may also load the
 *   library's device code, and loading allocates device memory: make one
 *   call per device at start-up, before the point where allocation is
 *   forbidden and before capturing any stream.  Later calls allocate
 *   nothing.  The address stays valid for the life of the device's primary
 *   context: after cudaDeviceReset on that device this entry point must not
 *   be called again until the process has reloaded the library.  Every call
 *   on a device shares the array and leaves its contents behind (the
 *   completion counter is cleared at the start of each call); calls that
 *   overlap on the GPU race, so serialise them (one stream, or events
 *   between streams). */
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
 * Kernels, by shape (the same as moe_layer_forward's, except that the layer
 * runs Q6_K at T > 16 on the tensor cores from fp16 copies of the pools it
 * makes in its workspace, which is larger by the pools' size in fp16):
 *   1 <= T <= 16, D in {256, 512, 768, 1024, 2048}, F % 256 == 0, F <= 1024:
 *     the dequant-fused grouped GEMV (mma.sync, TMA-streamed weights);
 *   T > 16, D % 256 == 0, F % 256 == 0, E <= 720: the grouped GEMM on the
 *     tcgen05 tensor cores (weights dequantised to fp16 in shared memory);
 *   any other shape: a portable CUDA-core kernel (correct, not tuned).
 * Q6_K (210-byte blocks) takes the GEMV only at D = 2048, where its gate/up
 * rows are whole 16-byte units for the tensor copies (its down rows are
 * copied in 8-row groups, which always are), and the portable kernel at
 * every other shape here, T > 16 included (630-byte rows of 768 weights are
 * not tensor-copyable; the fused layer converts instead, as above).
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
 *   shared               NULL or a pool with one slot (any moe_qtype) of a
 *                        SwiGLU expert with F = shared_F, added with weight 1
 *   y, y_dtype           device [T, D] output (F32 or BF16)
 *   ids_out, gates_out   device [T, k] or NULL: routing decisions
 *   logits_out           device fp32 [T, E] or NULL
 *   trace                NULL, or per-kernel timing of this call (moe_trace)
 *   phases               0 = the whole layer; else an OR of MOE_PHASE_* bits
 *                        (below): the parts this call runs
 *   expert_mask          device uint8 [E] or NULL: the FFN part of this call
 *                        runs only experts with a nonzero entry (NULL: all)
 *   counts_out, offsets_out, perm_out, inv_out
 *                        device int32 [E], [E+1], [T*k], [T*k] or NULL: the
 *                        permutation as moe_permute defines it; when given,
 *                        the call keeps its permutation there instead of in
 *                        the workspace.
 *   act_bits             0 or 16: 16-bit activations into the expert FFNs (as
 *                        above); 8: the inputs of every expert matmul (x, and
 *                        h before the down projection) quantized to 8-bit
 *                        blocks of 32 -- the fork README's W4A8 / W8A8 MMVQ
 *                        mode: per block, in fp32, d = max|v| / 127,
 *                        q = round-half-away-from-zero(v * (1 / d)) (0 when
 *                        d = 0), and int8 tensor-core products scaled by the
 *                        weight and activation block scales; the gate weight
 *                        multiplies each expert's output.  Decode shapes
 *                        (1 <= T <= 16, the decode GEMV's D and F) with Q4_0
 *                        or Q8_0 experts only: MOE_ERR_SHAPE or
 *                        MOE_ERR_UNSUPPORTED_QTYPE otherwise.
 * Phases let an expert cache overlap its miss copies with the FFN of the
 * experts already resident (kongchang article, "From Static Allocation to
 * Dynamic Scheduling"; FreeToken wiki explainer on hiding transfer time):
 *   call 1  ROUTE | FFN | SHARED, expert_mask = resident experts
 *           (or ROUTE alone, when the ids must reach the host first)
 *   wait    moe_cache_sync(...)  (the misses' copies)
 *   call 2  FFN | COMBINE, expert_mask = the experts just copied
 * The calls of one layer step must get the same arguments (except phases
 * and expert_mask) and the same workspace, on one stream.  Each expert row
 * is computed by the same kernel in the same order whatever the split, so
 * the result is bit-identical to a single call. */
#define MOE_PHASE_ROUTE 1u    /* logits, top-k, gates, permutation */
#define MOE_PHASE_FFN 2u      /* routed experts' FFN (those expert_mask admits) */
#define MOE_PHASE_SHARED 4u   /* the shared expert's FFN */
#define MOE_PHASE_COMBINE 8u  /* gate-weighted combine into y */
#define MOE_PHASE_ALL 15u

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
    int32_t phases;
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
    const uint8_t *expert_mask;
    int32_t *counts_out;
    int32_t *offsets_out;
    int32_t *perm_out;
    int32_t *inv_out;
    int32_t act_bits;
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
 * Global mode (global = 1; FreeToken fork README, "About": global LRU
 * expert caching, and "Elastic Memory Management": run-time re-allocation
 * of the expert cache's VRAM; kongchang article, "Dynamic Cache Adjustment
 * Experiments"): one pool of max_slots device slots shared by every layer,
 * of which the first n_slots are in use (the capacity, changed at run time
 * by moe_cache_resize).  One step counter serves every layer; an entry is
 * (layer, expert), keyed layer * E + expert; a missing entry takes the
 * empty slot of lowest index below the capacity, else evicts the entry with
 * the oldest stamp in ANY layer that is not requested in the same call (the
 * lower key on equal stamps).  A miss copy waits for the release point of
 * the victim's layer.  A request may evict the experts of another layer, so
 * enqueue a layer's FFN (and its release point) before requesting the next
 * layer, and request a layer before each use of it (its slot map is written
 * by its own requests only).
 *
 * moe_cache_desc (all pools in the layout above; sizes in bytes):
 *   n_layers, E, n_slots, qtype
 *   bytes_gate, bytes_up, bytes_down   one expert's bytes of each matrix
 *   host_gate/up/down   host arrays of n_layers pointers, each to pinned
 *                       [E] experts (expert e at e * bytes_*)
 *   dev_gate/up/down    device [n_layers][n_slots] slots; global mode:
 *                       device [max_slots] slots
 *   dev_slot_map        device int32 [n_layers][E]; entries of experts that
 *                       are not resident hold -1
 *   copy_stream         stream for the host-to-device copies (not NULL)
 *   dev_masks           device uint8 [n_layers][2][E] or NULL: per layer, the
 *                       last request's hit mask (requested and already
 *                       resident) and miss mask (requested and copied by
 *                       that request), written with the slot map; they are
 *                       the expert_mask arguments of the two moe_layer_forward
 *                       calls that overlap the copies with the FFN of the
 *                       resident experts (see moe_layer_args)
 *   global, max_slots   0: per-layer mode (max_slots unused); 1: global
 *                       mode with max_slots >= n_slots pool slots
 *                       (max_slots <= n_layers * E)
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
    uint8_t *dev_masks;
    int32_t global;
    int32_t max_slots;
} moe_cache_desc;

moe_status moe_cache_init(const moe_cache_desc *desc, moe_cache **out);
void moe_cache_destroy(moe_cache *cache);
/* Serve one request of n distinct expert ids (host int32) for `layer`:
 * runs the LRU on the host, enqueues the copies of the misses on the copy
 * stream, records the layer's copy event, and enqueues on `compute` the
 * update of the layer's device slot map.  Optional host outputs per id:
 * slots[n], miss[n] (0/1), evicted[n] (expert evicted, or in global mode
 * its key layer * E + expert; -1 when none).
 * MOE_ERR_CAPACITY if n > the capacity; MOE_ERR_INVALID_ARG on a bad or
 * repeated id.  The cache state is unchanged on error. */
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
/* The device pool view of one layer (slot-mapped; in global mode the whole
 * shared pool, n_slots = max_slots). */
moe_status moe_cache_layer_pool(moe_cache *cache, int layer, moe_pool *out);
/* Global mode: change the capacity to n_slots (1 <= n_slots <= max_slots)
 * at run time, without touching the host pools.  Growing adds empty slots.
 * Shrinking evicts entries, oldest stamp first (lower key on ties), until
 * at most n_slots are resident, then moves every entry held in a slot >=
 * n_slots, in increasing slot order, to the empty slot of lowest index
 * below n_slots: device-to-device copies on the copy stream after all work
 * enqueued on `compute` so far; work enqueued on `compute` after the call
 * runs once they are done, and from then on the slots [n_slots, max_slots)
 * are unused (their memory may serve something else until the cache grows
 * again).  Layers' slot maps are rewritten by their next requests.
 * *n_evicted / *n_moved (may be NULL) receive the counts.
 * MOE_ERR_INVALID_ARG for a per-layer cache, MOE_ERR_SHAPE out of range. */
moe_status moe_cache_resize(moe_cache *cache, int n_slots, int *n_evicted, int *n_moved,
                            moe_stream compute);
/* Device addresses of one layer's hit and miss masks (dev_masks).  The
 * flow of one cached layer step, with the copies overlapping compute:
 *   moe_cache_request(c, l, ids, ...)
 *   moe_layer_forward(ROUTE | FFN | SHARED, expert_mask = hit)
 *   moe_cache_sync(c, l, compute)
 *   moe_layer_forward(FFN | COMBINE, expert_mask = miss)
 *   moe_cache_release(c, l, compute)
 * MOE_ERR_INVALID_ARG without dev_masks. */
moe_status moe_cache_layer_masks(moe_cache *cache, int layer, const uint8_t **hit,
                                 const uint8_t **miss);
/* Counters since moe_cache_init: hits, misses, bytes copied, and
 * exposed_ns, the time the compute stream spent waiting in moe_cache_sync
 * for miss copies (measured on the GPU between two events recorded around
 * the wait; copies that finished before the compute stream reached the
 * sync point add nothing).  Waits for the compute stream to pass the sync
 * points it has not yet passed.  Any output pointer may be NULL. */
moe_status moe_cache_stats(moe_cache *cache, int64_t *hits, int64_t *misses,
                           int64_t *bytes_copied, int64_t *exposed_ns);

/* --------------------------------------------- prefill layer streaming
 * Full-layer double-buffered streaming of expert weights (FreeToken fork
 * README, "About": full-layer double-buffered prefill streaming; kongchang
 * article, "Dual-Buffering to Solve the Prefill Bottleneck").  A long prompt
 * reaches nearly every expert of every layer, so whole layers move: two
 * device buffers, each one layer's [E] experts in the pool layout; layer l
 * uses buffer l % 2 while the copy stream fills the other with the next
 * layer.  One stack pass:
 *   moe_streamer_prefetch(s, 0); moe_streamer_prefetch(s, 1);
 *   for each layer l:
 *     moe_streamer_acquire(s, l, compute, &pool)   compute waits for l's copy
 *     moe_layer_forward(... pool ...)               on compute
 *     moe_streamer_release(s, l, compute)           l's kernels are enqueued
 *     moe_streamer_prefetch(s, l + 2)               waits for that release
 * moe_streamer_desc:
 *   n_layers, E, qtype; bytes_gate/up/down   one expert's bytes
 *   host_gate/up/down   host arrays of n_layers pointers to pinned [E] experts
 *   dev_gate/up/down    two device buffers of [E] experts each
 *   copy_stream         stream for the host-to-device copies (not NULL)
 * The streamer keeps pointers to the caller's buffers; they must outlive it. */
typedef struct moe_streamer moe_streamer;
typedef struct {
    int32_t n_layers, E, qtype, reserved;
    size_t bytes_gate, bytes_up, bytes_down;
    const void *const *host_gate;
    const void *const *host_up;
    const void *const *host_down;
    void *dev_gate[2];
    void *dev_up[2];
    void *dev_down[2];
    moe_stream copy_stream;
} moe_streamer_desc;

moe_status moe_streamer_init(const moe_streamer_desc *desc, moe_streamer **out);
void moe_streamer_destroy(moe_streamer *s);
/* Enqueue the copy of `layer` into buffer layer % 2 on the copy stream,
 * after the release point of the layer that used that buffer last (a no-op
 * if the buffer already holds `layer`). */
moe_status moe_streamer_prefetch(moe_streamer *s, int layer);
/* Make `compute` wait for `layer`'s copy (prefetching it first if needed)
 * and return the pool view of its buffer (n_slots = E, no slot map). */
moe_status moe_streamer_acquire(moe_streamer *s, int layer, moe_stream compute, moe_pool *out);
/* Every kernel that reads `layer`'s buffer is enqueued on `compute`. */
moe_status moe_streamer_release(moe_streamer *s, int layer, moe_stream compute);
/* Bytes copied, and the time `compute` has waited in acquire for copies
 * (events around each wait; waits for the pending ones). */
moe_status moe_streamer_stats(moe_streamer *s, int64_t *bytes_copied, int64_t *exposed_ns);

#ifdef __cplusplus
}
#endif
#endif /* MOE_H */
