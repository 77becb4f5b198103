// stream.cu -- full-layer double-buffered streaming of expert weights for
// prefill (FreeToken fork README, "About": full-layer double-buffered
// prefill streaming; kongchang article, "Dual-Buffering to Solve the Prefill
// Bottleneck": while the GPU computes the current layer, the next layer's
// expert data is already being transferred over PCIe in the background).
//
// A long prompt routes tokens to nearly every expert of every layer, so the
// whole layer is copied: two device buffers of one layer's experts each;
// layer l runs from buffer l % 2 while the copy stream fills buffer
// (l + 1) % 2 with layer l + 1.  Ordering, all on the GPU through events:
//  - the copy of layer l waits for the release point of the layer that last
//    used the same buffer (l - 2), so no kernel still reads it;
//  - the compute stream waits for layer l's copy only when it needs the
//    weights (moe_streamer_acquire), so that wait is the exposed copy time.
#include "moe_internal.cuh"

#include <vector>

struct moe_streamer {
    moe_streamer_desc d;
    cudaEvent_t copied[2] = {nullptr, nullptr};     // buffer b holds its layer
    cudaEvent_t released[2] = {nullptr, nullptr};   // buffer b's last user is done
    bool rel_valid[2] = {false, false};
    int holds[2] = {-1, -1};                        // layer copied (or being copied) into b
    std::vector<std::pair<cudaEvent_t, cudaEvent_t>> waits;   // around acquire waits
    std::vector<cudaEvent_t> spare;
    int64_t bytes = 0, exposed_ns = 0;
};

namespace moe {
static moe_status harvest(moe_streamer *s, bool all) {
    size_t keep = 0;
    for (auto &pr : s->waits) {
        cudaError_t q = all ? cudaEventSynchronize(pr.second) : cudaEventQuery(pr.second);
        if (q != cudaSuccess) {
            if (all) return cuda_status(q, "moe_streamer_stats: wait");
            s->waits[keep++] = pr;
            continue;
        }
        float ms = 0.f;
        if (cudaEventElapsedTime(&ms, pr.first, pr.second) == cudaSuccess)
            s->exposed_ns += (int64_t)((double)ms * 1e6);
        s->spare.push_back(pr.first);
        s->spare.push_back(pr.second);
    }
    s->waits.resize(keep);
    cudaGetLastError();          // a not-ready query is no error of a later call
    return MOE_OK;
}

static cudaEvent_t spare_event(moe_streamer *s) {
    if (!s->spare.empty()) {
        cudaEvent_t e = s->spare.back();
        s->spare.pop_back();
        return e;
    }
    cudaEvent_t e = nullptr;
    return cudaEventCreate(&e) == cudaSuccess ? e : nullptr;
}
}  // namespace moe

using namespace moe;

extern "C" {

moe_status moe_streamer_init(const moe_streamer_desc *desc, moe_streamer **out) {
    if (!desc || !out) { set_error("moe_streamer_init: NULL argument"); return MOE_ERR_INVALID_ARG; }
    *out = nullptr;
    const moe_streamer_desc &d = *desc;
    if (d.n_layers <= 0 || d.E <= 0 || d.E > MOE_MAX_EXPERTS) {
        set_error("moe_streamer_init: need n_layers > 0 and 0 < E <= %d", MOE_MAX_EXPERTS);
        return MOE_ERR_SHAPE;
    }
    if (!qt_known(d.qtype)) {
        set_error("moe_streamer_init: unsupported quant type %d", (int)d.qtype);
        return MOE_ERR_UNSUPPORTED_QTYPE;
    }
    if (!d.host_gate || !d.host_up || !d.host_down || !d.copy_stream || !d.bytes_gate ||
        !d.bytes_up || !d.bytes_down) {
        set_error("moe_streamer_init: NULL host pools or copy stream, or zero expert size");
        return MOE_ERR_INVALID_ARG;
    }
    for (int b = 0; b < 2; b++)
        if (!d.dev_gate[b] || !d.dev_up[b] || !d.dev_down[b]) {
            set_error("moe_streamer_init: NULL device buffer %d", b);
            return MOE_ERR_INVALID_ARG;
        }
    for (int l = 0; l < d.n_layers; l++)
        if (!d.host_gate[l] || !d.host_up[l] || !d.host_down[l]) {
            set_error("moe_streamer_init: NULL host pool of layer %d", l);
            return MOE_ERR_INVALID_ARG;
        }
    moe_streamer *s = new (std::nothrow) moe_streamer();
    if (!s) { set_error("moe_streamer_init: out of host memory"); return MOE_ERR_INVALID_ARG; }
    s->d = d;
    moe_status st = MOE_OK;
    for (int b = 0; b < 2 && st == MOE_OK; b++) {
        st = cuda_status(cudaEventCreateWithFlags(&s->copied[b], cudaEventDisableTiming), "cudaEventCreate");
        if (st == MOE_OK)
            st = cuda_status(cudaEventCreateWithFlags(&s->released[b], cudaEventDisableTiming), "cudaEventCreate");
    }
    if (st != MOE_OK) { moe_streamer_destroy(s); return st; }
    *out = s;
    return MOE_OK;
}

void moe_streamer_destroy(moe_streamer *s) {
    if (!s) return;
    for (int b = 0; b < 2; b++) {
        if (s->copied[b]) cudaEventDestroy(s->copied[b]);
        if (s->released[b]) cudaEventDestroy(s->released[b]);
    }
    for (auto &pr : s->waits) { cudaEventDestroy(pr.first); cudaEventDestroy(pr.second); }
    for (auto e : s->spare) cudaEventDestroy(e);
    delete s;
}

moe_status moe_streamer_prefetch(moe_streamer *s, int layer) {
    if (!s || layer < 0 || layer >= s->d.n_layers) { set_error("moe_streamer_prefetch: bad streamer or layer"); return MOE_ERR_INVALID_ARG; }
    const moe_streamer_desc &d = s->d;
    const int b = layer & 1;
    cudaStream_t xs = (cudaStream_t)d.copy_stream;
    if (s->holds[b] == layer) return MOE_OK;          // already there (or on its way)
    moe_status st = MOE_OK;
    if (s->rel_valid[b])
        st = cuda_status(cudaStreamWaitEvent(xs, s->released[b], 0), "cudaStreamWaitEvent");
    const size_t E = (size_t)d.E;
    struct { void *dst; const void *src; size_t n; } cp[3] = {
        {d.dev_gate[b], d.host_gate[layer], E * d.bytes_gate},
        {d.dev_up[b], d.host_up[layer], E * d.bytes_up},
        {d.dev_down[b], d.host_down[layer], E * d.bytes_down},
    };
    for (auto &q : cp)
        if (st == MOE_OK)
            st = cuda_status(cudaMemcpyAsync(q.dst, q.src, q.n, cudaMemcpyHostToDevice, xs),
                             "moe_streamer_prefetch: cudaMemcpyAsync");
    if (st == MOE_OK) st = cuda_status(cudaEventRecord(s->copied[b], xs), "cudaEventRecord");
    if (st != MOE_OK) { s->holds[b] = -1; return st; }
    s->holds[b] = layer;
    s->rel_valid[b] = false;
    s->bytes += (int64_t)(E * (d.bytes_gate + d.bytes_up + d.bytes_down));
    return MOE_OK;
}

moe_status moe_streamer_acquire(moe_streamer *s, int layer, moe_stream compute, moe_pool *out) {
    if (!s || !out || layer < 0 || layer >= s->d.n_layers) { set_error("moe_streamer_acquire: bad argument"); return MOE_ERR_INVALID_ARG; }
    const moe_streamer_desc &d = s->d;
    const int b = layer & 1;
    moe_status st = MOE_OK;
    if (s->holds[b] != layer) st = moe_streamer_prefetch(s, layer);
    if (st != MOE_OK) return st;
    cudaStream_t cs = (cudaStream_t)compute;
    harvest(s, false);
    cudaEvent_t e0 = spare_event(s), e1 = spare_event(s);
    if (e0 && e1 && cudaEventRecord(e0, cs) == cudaSuccess) {
        st = cuda_status(cudaStreamWaitEvent(cs, s->copied[b], 0), "cudaStreamWaitEvent");
        if (st == MOE_OK) st = cuda_status(cudaEventRecord(e1, cs), "cudaEventRecord");
        if (st != MOE_OK) return st;
        s->waits.emplace_back(e0, e1);
    } else {
        if (e0) s->spare.push_back(e0);
        if (e1) s->spare.push_back(e1);
        cudaGetLastError();
        st = cuda_status(cudaStreamWaitEvent(cs, s->copied[b], 0), "cudaStreamWaitEvent");
        if (st != MOE_OK) return st;
    }
    out->qtype = d.qtype;
    out->n_slots = d.E;
    out->gate = d.dev_gate[b];
    out->up = d.dev_up[b];
    out->down = d.dev_down[b];
    out->slot_of_expert = nullptr;
    return MOE_OK;
}

moe_status moe_streamer_release(moe_streamer *s, int layer, moe_stream compute) {
    if (!s || layer < 0 || layer >= s->d.n_layers) { set_error("moe_streamer_release: bad streamer or layer"); return MOE_ERR_INVALID_ARG; }
    const int b = layer & 1;
    if (s->holds[b] != layer) { set_error("moe_streamer_release: layer %d does not hold its buffer", layer); return MOE_ERR_INVALID_ARG; }
    moe_status st = cuda_status(cudaEventRecord(s->released[b], (cudaStream_t)compute), "cudaEventRecord");
    s->rel_valid[b] = st == MOE_OK;
    return st;
}

moe_status moe_streamer_stats(moe_streamer *s, int64_t *bytes_copied, int64_t *exposed_ns) {
    if (!s) { set_error("moe_streamer_stats: NULL streamer"); return MOE_ERR_INVALID_ARG; }
    if (bytes_copied) *bytes_copied = s->bytes;
    if (exposed_ns) {
        moe_status st = harvest(s, true);
        if (st != MOE_OK) return st;
        *exposed_ns = s->exposed_ns;
    }
    return MOE_OK;
}

}  // extern "C"
