// layer.cu -- the whole layer in one call: route -> permute -> expert FFNs
// (+ shared expert) -> gate-weighted combine, or any subset of those parts
// (phases) for callers that split a layer step around an expert cache's
// copies.  The workspace holds every intermediate; its layout is fixed by
// carve() so that the size query and the call agree, and so that the calls
// of one split step find each other's results in it.
#include "moe_paths.cuh"

namespace moe {

struct LayerWs {
    int *status;         // device status word (first bytes of the workspace)
    void *route_ws;
    size_t route_bytes;
    int32_t *ids;
    float *gates;
    int32_t *counts, *offsets, *perm, *inv;
    int32_t *perm_scratch;   // per-CTA expert counts of the many-CTA permutation
    float *H;            // [T*k, F] fp32
    float *rows;         // [T*k, D] fp32
    float *shH;          // [T, shared_F]
    float *sh_rows;      // [T, D]
    __half *Hs;          // decode path: g*h in fp16 fragment order
    __half *x16, *H16;   // prefill path: fp16 activations and hidden rows
    __half *w16;         // prefill path: fp16 copies of the pools (Q6_K)
    int8_t *hq;          // 8-bit activations: h codes and their (scale, code sum)
    float2 *hs;
};

static LayerWs carve(const moe_layer_args &a, Carver &c) {
    LayerWs w{};
    const size_t Tk = (size_t)a.T * a.k;
    w.status = c.take<int>(16);
    w.route_bytes = route_ws_bytes(a.T, a.w_router ? a.D : QK, a.E, a.k);
    w.route_ws = c.take<char>(w.route_bytes);
    w.ids = c.take<int32_t>(Tk);
    w.gates = c.take<float>(Tk);
    w.counts = c.take<int32_t>(a.E);
    w.offsets = c.take<int32_t>(a.E + 1);
    w.perm = c.take<int32_t>(Tk);
    w.inv = c.take<int32_t>(Tk);
    w.perm_scratch = c.take<int32_t>(permute_scratch_ints(a.E));
    const int qt = a.pool ? a.pool->qtype : 0, sqt = a.shared ? a.shared->qtype : 0;
    if (a.act_bits == 8) {
        const int sF = a.shared ? a.shared_F : 0;
        w.hq = c.take<int8_t>(decode_a8_hq_bytes(a.T, a.k, a.F, sF));
        w.hs = c.take<float2>(decode_a8_hs_bytes(a.T, a.k, a.F, sF) / sizeof(float2));
        w.rows = c.take<float>(decode_rows_floats(a.T, a.k, a.D));
        return w;
    }
    if (decode_path_ok(a.T, a.D, a.F, a.shared ? a.shared_F : 0, qt, sqt)) {
        w.Hs = c.take<__half>(decode_hs_halves(a.T, a.k, a.F, a.shared ? a.shared_F : 0));
        w.rows = c.take<float>(decode_rows_floats(a.T, a.k, a.D));
        return w;
    }
    if (prefill_path_ok(a.T, a.D, a.F, a.shared ? a.shared_F : 0, a.E, qt, sqt, true)) {
        const int sF = a.shared ? a.shared_F : 0;
        if (prefill_needs_f16(qt, sqt, sF))
            w.w16 = c.take<__half>(prefill_f16_halves(a.pool ? a.pool->n_slots : a.E, a.D, a.F, sF));
        w.x16 = c.take<__half>(prefill_x16_halves(a.T, a.D));
        w.H16 = c.take<__half>(prefill_h_halves(a.T, a.k, a.F, sF));
        w.rows = c.take<float>(prefill_y_floats(a.T, a.k, a.D, sF));
        return w;
    }
    w.H = c.take<float>(Tk * a.F);
    w.rows = c.take<float>(Tk * a.D);
    if (a.shared) {
        w.shH = c.take<float>((size_t)a.T * a.shared_F);
        w.sh_rows = c.take<float>((size_t)a.T * a.D);
    }
    return w;
}

size_t layer_ws_bytes(const moe_layer_args &a) {
    Carver c(nullptr, 0);
    carve(a, c);
    return c.off;
}

static moe_status end_trace(Tracer *tr, moe_status st) {
    if (tr) {
        tr->end();
        if (st == MOE_OK && tr->err != cudaSuccess) {
            cudaGetLastError();   // the failed record is reported here, not left sticky
            return cuda_status(tr->err, "moe_layer_forward: trace event record");
        }
    }
    return st;
}

moe_status layer_forward(const moe_layer_args &a, void *ws, size_t ws_bytes, cudaStream_t s) {
    Carver c(ws, ws_bytes);
    LayerWs w = carve(a, c);
    Tracer trace;
    Tracer *tr = nullptr;
    if (a.trace) {
        if (!a.trace->events || a.trace->capacity < 12) {
            set_error("moe_layer_forward: trace needs at least 12 events");
            return MOE_ERR_INVALID_ARG;
        }
        a.trace->count = 0;
        trace.t = a.trace;
        trace.s = s;
        tr = &trace;
    }
    const unsigned ph = a.phases ? (unsigned)a.phases : MOE_PHASE_ALL;
    const bool do_route = ph & MOE_PHASE_ROUTE, do_ffn = ph & MOE_PHASE_FFN;
    const bool do_shared = (ph & MOE_PHASE_SHARED) && a.shared;
    const bool do_comb = ph & MOE_PHASE_COMBINE;
    int32_t *ids = a.ids_out ? a.ids_out : w.ids;
    float *gates = a.gates_out ? a.gates_out : w.gates;
    int32_t *counts = a.counts_out ? a.counts_out : w.counts;
    int32_t *offsets = a.offsets_out ? a.offsets_out : w.offsets;
    int32_t *perm = a.perm_out ? a.perm_out : w.perm;
    int32_t *inv = a.inv_out ? a.inv_out : w.inv;
    moe_status st;
    if (do_route) {
        bool permuted = false;
        if (a.w_router)
            st = launch_route_permute(a.x, a.x_dtype, a.w_router, a.bias, a.T, a.D, a.E, a.k,
                                      a.renorm, ids, gates, a.logits_out, counts, offsets, perm,
                                      inv, w.status, w.route_ws, w.route_bytes, s, tr, &permuted);
        else
            st = launch_route_permute(a.logits_in, MOE_F32, nullptr, a.bias, a.T, QK, a.E, a.k,
                                      a.renorm, ids, gates, a.logits_out, counts, offsets, perm,
                                      inv, w.status, w.route_ws, w.route_bytes, s, tr, &permuted);
        if (st != MOE_OK) return st;
        if (!permuted &&
            (st = launch_permute(ids, a.T, a.k, a.E, counts, offsets, perm, inv, s, tr,
                                 w.perm_scratch)) != MOE_OK)
            return st;
    }
    const int sF = a.shared ? a.shared_F : 0;
    if (w.hq) {
        if (!do_ffn && !do_shared && !do_comb) return end_trace(tr, MOE_OK);
        st = launch_ffn_decode_a8(a.x, a.x_dtype, a.T, a.D, a.F, a.E, a.k, perm, inv, offsets,
                                  gates, *a.pool, a.expert_mask, do_ffn,
                                  do_shared ? a.shared : nullptr, sF, a.shared != nullptr, w.hq,
                                  w.hs, do_comb ? a.y : nullptr, a.y_dtype, w.rows, w.status, s, tr);
        return end_trace(tr, st);
    }
    if (w.Hs) {
        if (!do_ffn && !do_shared && !do_comb) return end_trace(tr, MOE_OK);
        st = launch_ffn_decode(a.x, a.x_dtype, a.T, a.D, a.F, a.E, a.k, perm, inv, offsets, gates,
                               *a.pool, a.expert_mask, do_ffn, do_shared ? a.shared : nullptr, sF,
                               a.shared != nullptr, w.Hs, do_comb ? a.y : nullptr, a.y_dtype,
                               w.rows, w.status, s, tr);
        return end_trace(tr, st);
    }
    if (w.H16) {
        if ((do_ffn || do_shared) &&
            (st = launch_ffn_prefill(a.x, a.x_dtype, a.T, a.D, a.F, a.E, a.k, perm, offsets,
                                     *a.pool, a.expert_mask, do_ffn,
                                     do_shared ? a.shared : nullptr, sF, w.x16, w.H16, w.rows,
                                     w.status, s, tr, w.w16)) != MOE_OK)
            return st;
        st = MOE_OK;
        if (do_comb)
            st = launch_combine(w.rows, inv, gates, a.T, a.k, a.D,
                                a.shared ? w.rows + (size_t)a.T * a.k * a.D : nullptr, a.y,
                                a.y_dtype, s, tr);
        return end_trace(tr, st);
    }
    if (do_ffn &&
        (st = launch_ffn_generic(a.x, a.x_dtype, a.T, a.D, a.F, a.E, a.k, perm, offsets, *a.pool,
                                 a.expert_mask, w.H, w.rows, w.status, s, tr)) != MOE_OK)
        return st;
    if (do_shared &&
        (st = launch_ffn_generic(a.x, a.x_dtype, a.T, a.D, a.shared_F, 1, 1, nullptr, nullptr,
                                 *a.shared, nullptr, w.shH, w.sh_rows, w.status, s, tr, true)) !=
            MOE_OK)
        return st;
    st = MOE_OK;
    if (do_comb)
        st = launch_combine(w.rows, inv, gates, a.T, a.k, a.D, a.shared ? w.sh_rows : nullptr,
                            a.y, a.y_dtype, s, tr);
    return end_trace(tr, st);
}

}  // namespace moe
