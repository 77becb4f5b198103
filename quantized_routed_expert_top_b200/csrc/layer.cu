// layer.cu -- the whole layer in one call: route -> permute -> expert FFNs
// (+ shared expert) -> gate-weighted combine.  The workspace holds every
// intermediate; its layout is fixed by carve() so that the size query and
// the call agree.
#include "moe_paths.cuh"

namespace moe {

struct LayerWs {
    int *status;         // device status words (first bytes of the workspace)
    void *route_ws;
    size_t route_bytes;
    int32_t *ids;
    float *gates;
    int32_t *counts, *offsets, *perm, *inv;
    float *H;            // [T*k, F] fp32
    float *rows;         // [T*k, D] fp32
    float *shH;          // [T, shared_F]
    float *sh_rows;      // [T, D]
    __half *Hs;          // decode path: g*h in fp16 fragment order
    __half *x16, *H16;   // prefill path: fp16 activations and hidden rows
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
    if (decode_path_ok(a.T, a.D, a.F, a.shared ? a.shared_F : 0)) {
        w.Hs = c.take<__half>(decode_hs_halves(a.T, a.k, a.F, a.shared ? a.shared_F : 0));
        w.rows = c.take<float>(decode_rows_floats(a.T, a.k, a.D));
        return w;
    }
    if (prefill_path_ok(a.T, a.D, a.F, a.shared ? a.shared_F : 0, a.E)) {
        const int sF = a.shared ? a.shared_F : 0;
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
    int32_t *ids = a.ids_out ? a.ids_out : w.ids;
    float *gates = a.gates_out ? a.gates_out : w.gates;
    moe_status st;
    bool permuted = false;
    if (a.w_router)
        st = launch_route_permute(a.x, a.x_dtype, a.w_router, a.bias, a.T, a.D, a.E, a.k, a.renorm,
                                  ids, gates, a.logits_out, w.counts, w.offsets, w.perm, w.inv,
                                  w.status, w.route_ws, w.route_bytes, s, tr, &permuted);
    else
        st = launch_route_permute(a.logits_in, MOE_F32, nullptr, a.bias, a.T, QK, a.E, a.k,
                                  a.renorm, ids, gates, a.logits_out, w.counts, w.offsets, w.perm,
                                  w.inv, w.status, w.route_ws, w.route_bytes, s, tr, &permuted);
    if (st != MOE_OK) return st;
    if (!permuted &&
        (st = launch_permute(ids, a.T, a.k, a.E, w.counts, w.offsets, w.perm, w.inv, s, tr)) != MOE_OK)
        return st;
    if (w.Hs) {
        st = launch_ffn_decode(a.x, a.x_dtype, a.T, a.D, a.F, a.E, a.k, w.perm, w.inv, w.offsets,
                               gates, *a.pool, nullptr, a.shared, a.shared ? a.shared_F : 0, w.Hs,
                               a.y, a.y_dtype, w.rows, w.status, s, tr);
        if (tr) {
            tr->end();
            if (st == MOE_OK && tr->err != cudaSuccess) {
                cudaGetLastError();
                return cuda_status(tr->err, "moe_layer_forward: trace event record");
            }
        }
        return st;
    }
    if (w.H16) {
        const int sF = a.shared ? a.shared_F : 0;
        if ((st = launch_ffn_prefill(a.x, a.x_dtype, a.T, a.D, a.F, a.E, a.k, w.perm, w.offsets,
                                     *a.pool, a.shared, sF, w.x16, w.H16, w.rows, w.status, s,
                                     tr)) != MOE_OK)
            return st;
        st = launch_combine(w.rows, w.inv, gates, a.T, a.k, a.D,
                            a.shared ? w.rows + (size_t)a.T * a.k * a.D : nullptr, a.y, a.y_dtype,
                            s, tr);
        if (tr) {
            tr->end();
            if (st == MOE_OK && tr->err != cudaSuccess) {
                cudaGetLastError();
                return cuda_status(tr->err, "moe_layer_forward: trace event record");
            }
        }
        return st;
    }
    if ((st = launch_ffn_generic(a.x, a.x_dtype, a.T, a.D, a.F, a.E, a.k, w.perm, w.offsets,
                                 *a.pool, nullptr, w.H, w.rows, s, tr)) != MOE_OK)
        return st;
    if (a.shared) {
        if ((st = launch_ffn_generic(a.x, a.x_dtype, a.T, a.D, a.shared_F, 1, 1, nullptr, nullptr,
                                     *a.shared, nullptr, w.shH, w.sh_rows, s, tr, true)) != MOE_OK)
            return st;
    }
    st = launch_combine(w.rows, w.inv, gates, a.T, a.k, a.D, a.shared ? w.sh_rows : nullptr, a.y,
                        a.y_dtype, s, tr);
    if (tr) {
        tr->end();
        if (st == MOE_OK && tr->err != cudaSuccess) {
            cudaGetLastError();   // the failed record is reported here, not left sticky
            return cuda_status(tr->err, "moe_layer_forward: trace event record");
        }
    }
    return st;
}

}  // namespace moe
