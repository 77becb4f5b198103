// abi.cu -- the extern "C" entry points of libmoe declared in include/moe.h:
// argument checks (every dispatch has an erroring default), workspace
// carving and kernel dispatch.  No call allocates device memory.
#include "moe_internal.cuh"
#include "moe_paths.cuh"
#include "sm100.cuh"

#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <string>

namespace moe {

static thread_local std::string g_err;

void set_error(const char *fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof(buf), fmt, ap);
    va_end(ap);
    g_err = buf;
}

moe_status cuda_status(cudaError_t e, const char *what) {
    if (e == cudaSuccess) return MOE_OK;
    set_error("%s: %s", what, cudaGetErrorString(e));
    return MOE_ERR_CUDA;
}

int num_sms() {
    static int cached[64] = {0};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64) dev = 0;
    if (!cached[dev]) {
        int n = 0;
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
        cached[dev] = n > 0 ? n : 148;
    }
    return cached[dev];
}

static bool qtype_ok(int q) { return qt_known(q); }
static bool act_dtype_ok(int d) { return d == MOE_F32 || d == MOE_BF16; }

static moe_status check_shapes(const char *fn, int T, int D, int F, int E, int k) {
    if (T < 0 || D <= 0 || F <= 0 || E <= 0 || k <= 0) {
        set_error("%s: non-positive size (T=%d D=%d F=%d E=%d k=%d)", fn, T, D, F, E, k);
        return MOE_ERR_SHAPE;
    }
    if (D % QK || F % QK) {
        set_error("%s: D=%d and F=%d must be multiples of 32 (blocks run along the "
                  "reduction dimension)", fn, D, F);
        return MOE_ERR_SHAPE;
    }
    if (k > E || E > MOE_MAX_EXPERTS || k > MOE_MAX_TOPK) {
        set_error("%s: need 1 <= k <= E <= %d and k <= %d (k=%d E=%d)", fn, MOE_MAX_EXPERTS,
                  MOE_MAX_TOPK, k, E);
        return MOE_ERR_SHAPE;
    }
    return MOE_OK;
}

static moe_status check_pool(const char *fn, const moe_pool *p, int E) {
    if (!p) { set_error("%s: pool is NULL", fn); return MOE_ERR_INVALID_ARG; }
    if (!qtype_ok(p->qtype)) {
        set_error("%s: unsupported quant type %d (Q4_0=2, Q4_1=3, Q5_0=6, Q5_1=7, Q8_0=8)", fn,
                  (int)p->qtype);
        return MOE_ERR_UNSUPPORTED_QTYPE;
    }
    if (!p->gate || !p->up || !p->down || p->n_slots <= 0) {
        set_error("%s: pool has a NULL matrix or no slots", fn);
        return MOE_ERR_INVALID_ARG;
    }
    if (!p->slot_of_expert && p->n_slots < E) {
        set_error("%s: pool without a slot map holds %d slots for %d experts", fn, (int)p->n_slots, E);
        return MOE_ERR_SHAPE;
    }
    return MOE_OK;
}

// D and F must hold whole blocks of the pool's type (256 weights for the
// K-quants)
static moe_status check_block_shape(const char *fn, const moe_pool *p, int D, int F) {
    const int bw = qt_weights(p->qtype);
    if (D % bw || F % bw) {
        set_error("%s: D=%d and F=%d must be multiples of %d for quant type %d", fn, D, F, bw,
                  (int)p->qtype);
        return MOE_ERR_SHAPE;
    }
    return MOE_OK;
}

// The bounded-wait self test: one warp waits, with the kernels' wait
// routine and a short budget, on an mbarrier that nothing arrives at; the
// wait runs out, records MOE_DEV_TIMEOUT_FULL in the status word and the
// kernel returns (no fault, no hang: the context stays usable).
__global__ void selftest_wait_kernel(int *status, long long budget) {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_mbar_init();
    }
    __syncthreads();
    (void)__all_sync(0xffffffffu, mbar_wait_budget(&bar, 0, status, kErrTimeoutFull, budget));
}

}  // namespace moe

using namespace moe;

extern "C" {

const char *moe_last_error(void) { return g_err.c_str(); }

const char *moe_version(void) { return "libmoe 0.1 (sm_100a)"; }

int moe_block_bytes(int32_t qtype) {
    return qt_bytes(qtype);
}

int moe_block_weights(int32_t qtype) { return qt_weights(qtype); }

moe_status moe_selftest_wait_timeout(void *workspace, size_t ws_bytes, int64_t budget_cycles,
                                     moe_stream stream) {
    g_err.clear();
    if (!workspace || ws_bytes < 64) { set_error("moe_selftest_wait_timeout: workspace of at least 64 bytes needed"); return MOE_ERR_WORKSPACE; }
    if (budget_cycles <= 0 || budget_cycles > 4000000000LL) {
        set_error("moe_selftest_wait_timeout: budget_cycles must be in (0, 4e9]");
        return MOE_ERR_INVALID_ARG;
    }
    selftest_wait_kernel<<<1, 32, 0, (cudaStream_t)stream>>>((int *)workspace, (long long)budget_cycles);
    return cuda_status(cudaGetLastError(), "selftest_wait_kernel");
}

// ------------------------------------------------------ device status word
moe_status moe_workspace_status(void *workspace, int32_t *code, int clear, moe_stream stream) {
    g_err.clear();
    if (!workspace || !code) { set_error("moe_workspace_status: NULL workspace or code"); return MOE_ERR_INVALID_ARG; }
    cudaStream_t s = (cudaStream_t)stream;
    int32_t v = 0;
    moe_status st = cuda_status(cudaMemcpyAsync(&v, workspace, sizeof(v), cudaMemcpyDeviceToHost, s),
                                "moe_workspace_status: read");
    if (st == MOE_OK) st = cuda_status(cudaStreamSynchronize(s), "moe_workspace_status: wait");
    if (st != MOE_OK) return st;
    *code = v;
    if (clear && v != kErrNone) {
        st = cuda_status(cudaMemsetAsync(workspace, 0, sizeof(int32_t), s), "moe_workspace_status: clear");
        if (st == MOE_OK) st = cuda_status(cudaStreamSynchronize(s), "moe_workspace_status: wait");
        if (st != MOE_OK) return st;
    }
    switch (v) {
    case kErrNone: return MOE_OK;
    case kErrBadSlot:
        set_error("device status: an expert with tokens maps to a slot outside [0, n_slots); "
                  "its rows were skipped");
        return MOE_ERR_INVALID_ARG;
    case kErrTimeoutFull: case kErrTimeoutEmpty: case kErrTimeoutDrain: case kErrTimeoutMma:
        set_error("device status: a bounded wait inside a kernel ran out (code %d)", (int)v);
        return MOE_ERR_TIMEOUT;
    default:
        set_error("device status: unknown code %d", (int)v);
        return MOE_ERR_INVALID_ARG;
    }
}

// ----------------------------------------------------------------- route
size_t moe_route_workspace_size(int T, int D, int E, int k) {
    return route_ws_bytes(T < 0 ? 0 : T, D, E, k);
}

moe_status moe_route(const void *x, int32_t x_dtype, const float *w_router, const float *bias,
                     int T, int D, int E, int k, int renorm, int32_t *ids, float *gates,
                     float *logits, void *workspace, size_t ws_bytes, moe_stream stream) {
    g_err.clear();
    if (w_router == nullptr) D = QK;   // logits given: D unused
    moe_status st = check_shapes("moe_route", T, D, QK, E, k);
    if (st != MOE_OK) return st;
    if (!act_dtype_ok(x_dtype) || (w_router == nullptr && x_dtype != MOE_F32)) {
        set_error("moe_route: x dtype %d not allowed (F32/BF16 activations, F32 logits)", x_dtype);
        return MOE_ERR_INVALID_ARG;
    }
    if (renorm != 0 && renorm != 1) { set_error("moe_route: renorm must be 0 or 1"); return MOE_ERR_INVALID_ARG; }
    if (T == 0) return MOE_OK;
    if (!x || !ids || !gates) { set_error("moe_route: NULL x, ids or gates"); return MOE_ERR_INVALID_ARG; }
    if (!workspace || ws_bytes < route_ws_bytes(T, D, E, k)) {
        set_error("moe_route: workspace needs %zu bytes, got %zu", route_ws_bytes(T, D, E, k), ws_bytes);
        return MOE_ERR_WORKSPACE;
    }
    bool permuted = false;
    // the route workspace starts with 64 words: word 0 is the status word,
    // word 1 the split-K completion ticket
    int *err = (int *)workspace;
    return launch_route_permute(x, x_dtype, w_router, bias, T, D, E, k, renorm, ids, gates,
                                logits, nullptr, nullptr, nullptr, nullptr, err, workspace,
                                ws_bytes, (cudaStream_t)stream, nullptr, &permuted);
}

// --------------------------------------------------------------- permute
moe_status moe_permute(const int32_t *ids, int T, int k, int E, int32_t *counts, int32_t *offsets,
                       int32_t *perm, int32_t *inv, moe_stream stream) {
    g_err.clear();
    moe_status st = check_shapes("moe_permute", T, QK, QK, E, k);
    if (st != MOE_OK) return st;
    if (!counts || !offsets) { set_error("moe_permute: NULL counts or offsets"); return MOE_ERR_INVALID_ARG; }
    if (T > 0 && (!ids || !perm || !inv)) { set_error("moe_permute: NULL ids, perm or inv"); return MOE_ERR_INVALID_ARG; }
    if ((long long)T * k > 0x7fffffffLL) { set_error("moe_permute: T*k overflows int32"); return MOE_ERR_SHAPE; }
    return launch_permute(ids, T, k, E, counts, offsets, perm, inv, (cudaStream_t)stream);
}

// ------------------------------------------------------------ expert FFN
// Workspace pieces of moe_expert_ffn: the status word, then the decode
// path's fp16 hidden rows, or the tensor-core path's fp16 activations and
// hidden rows, or the portable path's fp32 hidden rows.  Neither E nor the
// quant type is an argument of the size query, so it covers every path the
// shape admits (the portable one always).
size_t moe_expert_ffn_workspace_size(int T, int k, int D, int F) {
    T = T < 0 ? 0 : T;
    Carver c(nullptr, 0);
    c.take<int>(16);
    Carver g = c;
    g.take<float>((size_t)T * k * F);
    size_t need = g.off;
    if (decode_path_ok(T, D, F, 0, MOE_Q4_0, 0)) {
        Carver d = c;
        d.take<__half>(decode_hs_halves(T, k, F, 0));
        need = d.off > need ? d.off : need;
    }
    if (T > 16 && D % 256 == 0 && F % 256 == 0) {
        Carver p = c;
        p.take<__half>(prefill_x16_halves(T, D));
        p.take<__half>(prefill_h_halves(T, k, F, 0));
        need = p.off > need ? p.off : need;
    }
    return need;
}

moe_status moe_expert_ffn(const void *x, int32_t x_dtype, int T, int D, int F, int E, int k,
                          const int32_t *perm, const int32_t *offsets, const moe_pool *pool,
                          const uint8_t *expert_mask, float *out_rows, void *workspace,
                          size_t ws_bytes, moe_stream stream) {
    g_err.clear();
    moe_status st = check_shapes("moe_expert_ffn", T, D, F, E, k);
    if (st != MOE_OK) return st;
    if ((st = check_pool("moe_expert_ffn", pool, E)) != MOE_OK) return st;
    if ((st = check_block_shape("moe_expert_ffn", pool, D, F)) != MOE_OK) return st;
    if (!act_dtype_ok(x_dtype)) { set_error("moe_expert_ffn: x dtype %d not F32/BF16", x_dtype); return MOE_ERR_INVALID_ARG; }
    if (T == 0) return MOE_OK;
    if (!x || !perm || !offsets || !out_rows) { set_error("moe_expert_ffn: NULL x, perm, offsets or out_rows"); return MOE_ERR_INVALID_ARG; }
    size_t need = moe_expert_ffn_workspace_size(T, k, D, F);
    if (!workspace || ws_bytes < need) {
        set_error("moe_expert_ffn: workspace needs %zu bytes, got %zu", need, ws_bytes);
        return MOE_ERR_WORKSPACE;
    }
    Carver c(workspace, ws_bytes);
    int *status = c.take<int>(16);
    if (decode_path_ok(T, D, F, 0, pool->qtype, 0)) {
        __half *Hs = c.take<__half>(decode_hs_halves(T, k, F, 0));
        return launch_ffn_decode(x, x_dtype, T, D, F, E, k, perm, nullptr, offsets, nullptr, *pool,
                                 expert_mask, true, nullptr, 0, false, Hs, nullptr, MOE_F32,
                                 out_rows, status, (cudaStream_t)stream, nullptr);
    }
    if (prefill_path_ok(T, D, F, 0, E, pool->qtype, 0)) {
        __half *x16 = c.take<__half>(prefill_x16_halves(T, D));
        __half *H16 = c.take<__half>(prefill_h_halves(T, k, F, 0));
        return launch_ffn_prefill(x, x_dtype, T, D, F, E, k, perm, offsets, *pool, expert_mask,
                                  true, nullptr, 0, x16, H16, out_rows, status,
                                  (cudaStream_t)stream, nullptr);
    }
    float *H = c.take<float>((size_t)T * k * F);
    return launch_ffn_generic(x, x_dtype, T, D, F, E, k, perm, offsets, *pool, expert_mask, H,
                              out_rows, status, (cudaStream_t)stream);
}

// --------------------------------------------------------------- combine
moe_status moe_combine(const float *rows, const int32_t *inv, const float *gates, int T, int k, int D,
                       const float *shared_rows, void *y, int32_t y_dtype, moe_stream stream) {
    g_err.clear();
    if (T < 0 || k <= 0 || D <= 0 || k > MOE_MAX_TOPK) { set_error("moe_combine: bad sizes"); return MOE_ERR_SHAPE; }
    if (y_dtype != MOE_F32 && y_dtype != MOE_BF16 && y_dtype != MOE_F16) {
        set_error("moe_combine: unsupported output dtype %d", y_dtype);
        return MOE_ERR_INVALID_ARG;
    }
    if (T == 0) return MOE_OK;
    if (!rows || !inv || !gates || !y) { set_error("moe_combine: NULL argument"); return MOE_ERR_INVALID_ARG; }
    return launch_combine(rows, inv, gates, T, k, D, shared_rows, y, y_dtype, (cudaStream_t)stream);
}

// ---------------------------------------------------------- fused forward
size_t moe_layer_workspace_size(const moe_layer_args *a) {
    if (!a) return 0;
    return layer_ws_bytes(*a);
}

moe_status moe_layer_forward(const moe_layer_args *a, void *workspace, size_t ws_bytes,
                             moe_stream stream) {
    g_err.clear();
    if (!a) { set_error("moe_layer_forward: args is NULL"); return MOE_ERR_INVALID_ARG; }
    const int D_eff = a->D;
    moe_status st = check_shapes("moe_layer_forward", a->T, D_eff, a->F, a->E, a->k);
    if (st != MOE_OK) return st;
    if ((st = check_pool("moe_layer_forward", a->pool, a->E)) != MOE_OK) return st;
    if ((st = check_block_shape("moe_layer_forward", a->pool, a->D, a->F)) != MOE_OK) return st;
    if (a->shared) {
        if ((st = check_pool("moe_layer_forward (shared)", a->shared, 1)) != MOE_OK) return st;
        if (a->shared_F <= 0 || a->shared_F % QK) {
            set_error("moe_layer_forward: shared_F=%d must be a positive multiple of 32", a->shared_F);
            return MOE_ERR_SHAPE;
        }
        if ((st = check_block_shape("moe_layer_forward (shared)", a->shared, a->D, a->shared_F)) != MOE_OK)
            return st;
    }
    if (!act_dtype_ok(a->x_dtype)) { set_error("moe_layer_forward: x dtype %d not F32/BF16", a->x_dtype); return MOE_ERR_INVALID_ARG; }
    if (a->y_dtype != MOE_F32 && a->y_dtype != MOE_BF16) {
        set_error("moe_layer_forward: y dtype %d not F32/BF16", a->y_dtype);
        return MOE_ERR_INVALID_ARG;
    }
    if (a->renorm != 0 && a->renorm != 1) { set_error("moe_layer_forward: renorm must be 0 or 1"); return MOE_ERR_INVALID_ARG; }
    if ((unsigned)a->phases & ~MOE_PHASE_ALL) {
        set_error("moe_layer_forward: phases %d has bits outside MOE_PHASE_ALL", (int)a->phases);
        return MOE_ERR_INVALID_ARG;
    }
    if (a->act_bits != 0 && a->act_bits != 8 && a->act_bits != 16) {
        set_error("moe_layer_forward: act_bits %d is not 0, 8 or 16", (int)a->act_bits);
        return MOE_ERR_INVALID_ARG;
    }
    if (a->act_bits == 8) {
        const int sqt = a->shared ? a->shared->qtype : MOE_Q8_0;
        if (a->pool->qtype != MOE_Q4_0 && a->pool->qtype != MOE_Q8_0) {
            set_error("moe_layer_forward: 8-bit activations need Q4_0 or Q8_0 experts (got %d)",
                      (int)a->pool->qtype);
            return MOE_ERR_UNSUPPORTED_QTYPE;
        }
        if (sqt != MOE_Q4_0 && sqt != MOE_Q8_0) {
            set_error("moe_layer_forward: 8-bit activations need a Q4_0 or Q8_0 shared expert (got %d)", sqt);
            return MOE_ERR_UNSUPPORTED_QTYPE;
        }
        if (a->T > 0 && !decode_a8_ok(a->T, a->D, a->F, a->shared ? a->shared_F : 0, a->pool->qtype, sqt)) {
            set_error("moe_layer_forward: 8-bit activations run on decode shapes only (1 <= T <= 16, "
                      "D in {256, 512, 768, 1024, 2048}, F and shared_F multiples of 256 up to 1024; "
                      "T=%d D=%d F=%d)", a->T, a->D, a->F);
            return MOE_ERR_SHAPE;
        }
    }
    if (a->T == 0) return MOE_OK;
    const unsigned ph = a->phases ? (unsigned)a->phases : MOE_PHASE_ALL;
    const bool need_x = (ph & (MOE_PHASE_FFN | MOE_PHASE_SHARED)) || ((ph & MOE_PHASE_ROUTE) && a->w_router);
    if ((need_x && !a->x) || ((ph & MOE_PHASE_COMBINE) && !a->y) ||
        ((ph & MOE_PHASE_ROUTE) && !a->w_router && !a->logits_in)) {
        set_error("moe_layer_forward: NULL x, y, or both w_router and logits_in, for phases %u", ph);
        return MOE_ERR_INVALID_ARG;
    }
    size_t need = layer_ws_bytes(*a);
    if (!workspace || ws_bytes < need) {
        set_error("moe_layer_forward: workspace needs %zu bytes, got %zu", need, ws_bytes);
        return MOE_ERR_WORKSPACE;
    }
    return layer_forward(*a, workspace, ws_bytes, (cudaStream_t)stream);
}

}  // extern "C"
