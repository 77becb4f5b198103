// cache.cu -- per-layer HBM expert cache fed from a pinned host pool.
//
// The full expert set stays in pinned host memory; each layer owns n_slots
// device slots used as an LRU cache (FreeToken fork README, "About": global
// LRU expert caching; wiki explainer: LRU caching follows token-level
// routing locality; kongchang article: VRAM as a cache, system RAM as the
// source of truth).  Replacement rules:
//  - each request is one step; every requested expert is stamped with it;
//  - ids are served in the order given; resident ids are hits;
//  - a miss takes the empty slot of lowest index, else evicts the resident
//    expert with the oldest stamp among those NOT requested in this step
//    (lower expert id on equal stamps).
// Missed experts are copied host->device with cudaMemcpyAsync on the copy
// stream, which first waits for an event recorded on the compute stream (a
// victim slot may still be read by earlier kernels): the layer's release
// event when the caller recorded one after the layer's last FFN
// (moe_cache_release; the slots of a layer are read by that layer's kernels
// only, so copies for later layers then overlap the FFN of earlier ones),
// else an event over everything enqueued on the compute stream so far.  The copy-done event of
// the layer lets the compute stream wait (moe_cache_sync) only when the
// missing experts are needed, so the FFN of resident experts overlaps the
// copies.  The layer's device slot map is refreshed from a pinned staging
// buffer (two per layer, alternating; each reuse waits, with a time limit,
// for the copy that last read it).
// Exposed copy time: moe_cache_sync brackets the compute stream's wait with
// two timing events; the time between them is how long the compute stream
// stood still for copies (zero when the copies had already landed).  The
// pairs are read back lazily (at the next sync once complete, or in
// moe_cache_stats).
#include "moe_internal.cuh"

#include <chrono>
#include <cstring>
#include <new>
#include <thread>
#include <vector>

struct moe_cache {
    moe_cache_desc d;
    struct Layer {
        std::vector<int32_t> slot_expert;   // [n_slots] -1 empty
        std::vector<int32_t> expert_slot;   // [E] -1 not resident
        std::vector<int64_t> stamp;         // [E]
        int64_t step = 0;
        bool pending = false;
        bool released = false;              // release_ev marks the last use of the slots
        cudaEvent_t copied = nullptr;
        cudaEvent_t release_ev = nullptr;
        cudaEvent_t map_done[2] = {nullptr, nullptr};
        int map_buf = 0;
    };
    std::vector<Layer> layers;
    // global mode: one pool of max_slots slots shared by every layer, the
    // first `cap` in use; entries keyed layer * E + expert; one step counter
    bool global = false;
    struct Glob {
        int cap = 0;
        int64_t step = 0;
        std::vector<int32_t> slot_key;      // [max_slots] -1 empty
        std::vector<int32_t> key_slot;      // [n_layers * E] -1 not resident
        std::vector<int64_t> stamp;         // [n_layers * E]
    } g;
    // pinned staging per (layer, buffer): the slot map (int32[E]), then the
    // request's hit and miss masks (uint8[E] each)
    uint8_t *pinned_stage = nullptr;
    size_t stage_stride = 0;
    int32_t *stage_map(int l, int b) { return (int32_t *)(pinned_stage + ((size_t)l * 2 + b) * stage_stride); }
    uint8_t *stage_masks(int l, int b) { return (uint8_t *)(stage_map(l, b) + d.E); }
    cudaEvent_t compute_ready = nullptr;
    int64_t hits = 0, misses = 0, bytes = 0;
    int fail_copy_at = -1;                // test hook: fail the n-th copy
    int copies_issued = 0;
    // exposed copy time: (before, after) event pairs around each wait
    std::vector<std::pair<cudaEvent_t, cudaEvent_t>> wait_pairs;
    std::vector<cudaEvent_t> free_events;
    int64_t exposed_ns = 0;
};

namespace moe {
static cudaEvent_t take_event(moe_cache *c) {
    if (!c->free_events.empty()) {
        cudaEvent_t e = c->free_events.back();
        c->free_events.pop_back();
        return e;
    }
    cudaEvent_t e = nullptr;
    if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
    return e;
}

// Add the completed wait pairs to exposed_ns (all of them if `all`, waiting
// for each; else only those already complete).
static moe_status harvest_waits(moe_cache *c, bool all);

static moe_status wait_event_bounded(cudaEvent_t ev, double seconds) {
    auto t0 = std::chrono::steady_clock::now();
    for (;;) {
        cudaError_t e = cudaEventQuery(ev);
        if (e == cudaSuccess) return MOE_OK;
        if (e != cudaErrorNotReady) return cuda_status(e, "cudaEventQuery");
        double dt = std::chrono::duration<double>(std::chrono::steady_clock::now() - t0).count();
        if (dt > seconds) {
            set_error("expert cache: wait for a slot-map copy exceeded %.1f s", seconds);
            return MOE_ERR_TIMEOUT;
        }
        std::this_thread::yield();
    }
}
static moe_status harvest_waits(moe_cache *c, bool all) {
    size_t keep = 0;
    moe_status st = MOE_OK;
    for (size_t i = 0; i < c->wait_pairs.size(); i++) {
        auto pr = c->wait_pairs[i];
        if (st == MOE_OK && all) st = wait_event_bounded(pr.second, 60.0);
        const bool done = st == MOE_OK && cudaEventQuery(pr.second) == cudaSuccess;
        if (!done) {
            c->wait_pairs[keep++] = pr;
            continue;
        }
        float ms = 0.f;
        if (cudaEventElapsedTime(&ms, pr.first, pr.second) == cudaSuccess)
            c->exposed_ns += (int64_t)((double)ms * 1e6);
        c->free_events.push_back(pr.first);
        c->free_events.push_back(pr.second);
    }
    c->wait_pairs.resize(keep);
    cudaGetLastError();     // a not-ready query is not an error of any later call
    return st;
}

}  // namespace moe

using namespace moe;

extern "C" {

moe_status moe_cache_init(const moe_cache_desc *desc, moe_cache **out) {
    if (!desc || !out) { set_error("moe_cache_init: NULL argument"); return MOE_ERR_INVALID_ARG; }
    *out = nullptr;
    const moe_cache_desc &d = *desc;
    if (d.global != 0 && d.global != 1) { set_error("moe_cache_init: global must be 0 or 1"); return MOE_ERR_INVALID_ARG; }
    if (d.n_layers <= 0 || d.E <= 0 || d.E > MOE_MAX_EXPERTS || d.n_slots <= 0 ||
        (!d.global && d.n_slots > d.E)) {
        set_error("moe_cache_init: need n_layers > 0, 0 < n_slots <= E <= %d", MOE_MAX_EXPERTS);
        return MOE_ERR_SHAPE;
    }
    if (d.global && (d.max_slots < d.n_slots || (int64_t)d.max_slots > (int64_t)d.n_layers * d.E)) {
        set_error("moe_cache_init: global cache needs n_slots <= max_slots <= n_layers * E");
        return MOE_ERR_SHAPE;
    }
    if (!qt_known(d.qtype)) {
        set_error("moe_cache_init: unsupported quant type %d", (int)d.qtype);
        return MOE_ERR_UNSUPPORTED_QTYPE;
    }
    if (!d.host_gate || !d.host_up || !d.host_down || !d.dev_gate || !d.dev_up || !d.dev_down ||
        !d.dev_slot_map || !d.copy_stream || !d.bytes_gate || !d.bytes_up || !d.bytes_down) {
        set_error("moe_cache_init: NULL pool pointer, copy stream or zero expert size");
        return MOE_ERR_INVALID_ARG;
    }
    for (int l = 0; l < d.n_layers; l++)
        if (!d.host_gate[l] || !d.host_up[l] || !d.host_down[l]) {
            set_error("moe_cache_init: NULL host pool of layer %d", l);
            return MOE_ERR_INVALID_ARG;
        }
    moe_cache *c = new (std::nothrow) moe_cache();
    if (!c) { set_error("moe_cache_init: out of host memory"); return MOE_ERR_INVALID_ARG; }
    c->d = d;
    c->layers.resize(d.n_layers);
    c->global = d.global != 0;
    if (c->global) {
        c->g.cap = d.n_slots;
        c->g.slot_key.assign(d.max_slots, -1);
        c->g.key_slot.assign((size_t)d.n_layers * d.E, -1);
        c->g.stamp.assign((size_t)d.n_layers * d.E, 0);
    }
    moe_status st = MOE_OK;
    c->stage_stride = round_up(sizeof(int32_t) * d.E + 2 * (size_t)d.E, 64);
    cudaError_t e = cudaHostAlloc((void **)&c->pinned_stage, c->stage_stride * d.n_layers * 2,
                                  cudaHostAllocDefault);
    if (e != cudaSuccess) st = cuda_status(e, "moe_cache_init: pinned slot maps");
    if (st == MOE_OK) st = cuda_status(cudaEventCreateWithFlags(&c->compute_ready, cudaEventDisableTiming), "cudaEventCreate");
    for (int l = 0; l < d.n_layers && st == MOE_OK; l++) {
        auto &L = c->layers[l];
        L.slot_expert.assign(d.n_slots, -1);
        L.expert_slot.assign(d.E, -1);
        L.stamp.assign(d.E, 0);
        st = cuda_status(cudaEventCreateWithFlags(&L.copied, cudaEventDisableTiming), "cudaEventCreate");
        if (st == MOE_OK)
            st = cuda_status(cudaEventCreateWithFlags(&L.release_ev, cudaEventDisableTiming), "cudaEventCreate");
        for (int b = 0; b < 2 && st == MOE_OK; b++)
            st = cuda_status(cudaEventCreateWithFlags(&L.map_done[b], cudaEventDisableTiming), "cudaEventCreate");
        if (st == MOE_OK)
            for (int b = 0; b < 2; b++) {
                for (int i = 0; i < d.E; i++) c->stage_map(l, b)[i] = -1;
                memset(c->stage_masks(l, b), 0, 2 * (size_t)d.E);
            }
    }
    // all slot maps start empty (-1), all masks zero
    for (int l = 0; l < d.n_layers && st == MOE_OK; l++) {
        st = cuda_status(cudaMemcpy(d.dev_slot_map + (size_t)l * d.E, c->stage_map(l, 0),
                                    sizeof(int32_t) * d.E, cudaMemcpyHostToDevice),
                         "moe_cache_init: slot map");
        if (st == MOE_OK && d.dev_masks)
            st = cuda_status(cudaMemcpy(d.dev_masks + (size_t)l * 2 * d.E, c->stage_masks(l, 0),
                                        2 * (size_t)d.E, cudaMemcpyHostToDevice),
                             "moe_cache_init: masks");
    }
    if (st != MOE_OK) { moe_cache_destroy(c); return st; }
    *out = c;
    return MOE_OK;
}

void moe_cache_destroy(moe_cache *c) {
    if (!c) return;
    for (auto &L : c->layers) {
        if (L.copied) cudaEventDestroy(L.copied);
        if (L.release_ev) cudaEventDestroy(L.release_ev);
        for (auto &ev : L.map_done) if (ev) cudaEventDestroy(ev);
    }
    if (c->compute_ready) cudaEventDestroy(c->compute_ready);
    for (auto &pr : c->wait_pairs) {
        cudaEventDestroy(pr.first);
        cudaEventDestroy(pr.second);
    }
    for (auto ev : c->free_events) cudaEventDestroy(ev);
    if (c->pinned_stage) cudaFreeHost(c->pinned_stage);
    delete c;
}

// Test hook (not in the public header): make the n-th expert copy (0-based,
// counted over the cache's lifetime) fail as if cudaMemcpyAsync had failed.
void moe_cache_debug_fail_copy(moe_cache *c, int nth) {
    if (c) { c->fail_copy_at = nth; c->copies_issued = 0; }
}

moe_status moe_cache_request(moe_cache *c, int layer, const int32_t *ids, int n, int32_t *slots,
                             int32_t *miss, int32_t *evicted, int *n_miss, moe_stream compute) {
    if (!c || (!ids && n > 0)) { set_error("moe_cache_request: NULL argument"); return MOE_ERR_INVALID_ARG; }
    const moe_cache_desc &d = c->d;
    if (layer < 0 || layer >= d.n_layers) { set_error("moe_cache_request: layer %d out of range", layer); return MOE_ERR_INVALID_ARG; }
    if (n < 0) { set_error("moe_cache_request: n < 0"); return MOE_ERR_INVALID_ARG; }
    const int capacity = c->global ? c->g.cap : d.n_slots;
    if (n > capacity) {
        set_error("moe_cache_request: %d experts requested but the cache has %d slots", n, capacity);
        return MOE_ERR_CAPACITY;
    }
    auto &L = c->layers[layer];
    std::vector<char> wanted(d.E, 0);
    for (int i = 0; i < n; i++) {
        if (ids[i] < 0 || ids[i] >= d.E) { set_error("moe_cache_request: expert id %d out of range", ids[i]); return MOE_ERR_INVALID_ARG; }
        if (wanted[ids[i]]) { set_error("moe_cache_request: expert id %d repeated", ids[i]); return MOE_ERR_INVALID_ARG; }
        wanted[ids[i]] = 1;
    }
    cudaStream_t cs = (cudaStream_t)compute;
    cudaStream_t xs = (cudaStream_t)d.copy_stream;
    // staging buffer for this request's slot map: wait until its last copy ran
    const int buf = L.map_buf;
    moe_status st = wait_event_bounded(L.map_done[buf], 10.0);
    if (st != MOE_OK) return st;

    // LRU decisions (committed below; on a copy failure the touched slots are
    // invalidated so the resident set stays truthful).  Per-layer mode: the
    // layer's own slots, keys = expert ids.  Global mode: the shared pool,
    // keys = layer * E + expert, victims from any layer.
    std::vector<int> miss_idx;
    std::vector<int32_t> out_slot(n), out_ev(n, -1);
    std::vector<char> victim_layer(d.n_layers, 0);     // layers whose slots the copies overwrite
    const bool gm = c->global;
    const int64_t step = gm ? c->g.step + 1 : L.step + 1;
    std::vector<int32_t> se = gm ? c->g.slot_key : L.slot_expert;
    std::vector<int32_t> es = gm ? c->g.key_slot : L.expert_slot;
    std::vector<int64_t> stamp = gm ? c->g.stamp : L.stamp;
    const int key0 = gm ? layer * d.E : 0;              // key of expert 0 of this layer
    const int nkeys = gm ? d.n_layers * d.E : d.E;
    for (int i = 0; i < n; i++) {
        const int key = key0 + ids[i];
        if (es[key] >= 0) {
            out_slot[i] = es[key];
        } else {
            int s = -1;
            for (int q = 0; q < capacity; q++) if (se[q] < 0) { s = q; break; }
            if (s < 0) {
                int victim = -1;
                for (int v = 0; v < nkeys; v++) {
                    if (es[v] < 0 || (v >= key0 && v < key0 + d.E && wanted[v - key0])) continue;
                    if (victim < 0 || stamp[v] < stamp[victim]) victim = v;
                }
                s = es[victim];
                es[victim] = -1;
                out_ev[i] = victim;
                victim_layer[gm ? victim / d.E : layer] = 1;
            }
            se[s] = key;
            es[key] = s;
            out_slot[i] = s;
            miss_idx.push_back(i);
        }
        stamp[key] = step;
    }

    // copies of the misses on the copy stream, after the last use of the
    // slots they overwrite: the release point of each victim's layer when it
    // has one, else everything enqueued on the compute stream so far (empty
    // slots were never read, or were vacated by a resize that waited)
    moe_status cst = MOE_OK;
    if (!miss_idx.empty()) {
        bool need_all = !gm && !L.released;
        for (int l = 0; l < d.n_layers && cst == MOE_OK; l++) {
            if (!victim_layer[l] && !(l == layer && !gm)) continue;
            if (c->layers[l].released)
                cst = cuda_status(cudaStreamWaitEvent(xs, c->layers[l].release_ev, 0), "cudaStreamWaitEvent");
            else
                need_all = true;
        }
        if (cst == MOE_OK && need_all) {
            cst = cuda_status(cudaEventRecord(c->compute_ready, cs), "cudaEventRecord");
            if (cst == MOE_OK) cst = cuda_status(cudaStreamWaitEvent(xs, c->compute_ready, 0), "cudaStreamWaitEvent");
        }
        for (size_t m = 0; m < miss_idx.size() && cst == MOE_OK; m++) {
            const int i = miss_idx[m];
            const int e = ids[i];
            const size_t slot = gm ? (size_t)out_slot[i] : (size_t)layer * d.n_slots + out_slot[i];
            struct { void *dst; const void *src; size_t n; } cp[3] = {
                {(char *)d.dev_gate + slot * d.bytes_gate, (const char *)d.host_gate[layer] + (size_t)e * d.bytes_gate, d.bytes_gate},
                {(char *)d.dev_up + slot * d.bytes_up, (const char *)d.host_up[layer] + (size_t)e * d.bytes_up, d.bytes_up},
                {(char *)d.dev_down + slot * d.bytes_down, (const char *)d.host_down[layer] + (size_t)e * d.bytes_down, d.bytes_down},
            };
            for (auto &q : cp) {
                if (c->fail_copy_at >= 0 && c->copies_issued == c->fail_copy_at) {
                    c->copies_issued++;
                    set_error("moe_cache_request: injected copy failure");
                    cst = MOE_ERR_CUDA;
                    break;
                }
                c->copies_issued++;
                cst = cuda_status(cudaMemcpyAsync(q.dst, q.src, q.n, cudaMemcpyHostToDevice, xs),
                                  "moe_cache_request: cudaMemcpyAsync");
                if (cst != MOE_OK) break;
            }
        }
        if (cst == MOE_OK) cst = cuda_status(cudaEventRecord(L.copied, xs), "cudaEventRecord");
    }
    if (cst != MOE_OK) {
        // invalidate every slot this request wrote into: the resident set is
        // the old one minus the victims, and no missed expert is resident
        for (int i : miss_idx) {
            const int s = out_slot[i];
            se[s] = -1;
            es[key0 + ids[i]] = -1;
        }
        // keep the old recency of experts that were not served
        stamp = gm ? c->g.stamp : L.stamp;
    }
    if (gm) {
        c->g.slot_key.swap(se);
        c->g.key_slot.swap(es);
        c->g.stamp.swap(stamp);
        c->g.step = step;
    } else {
        L.slot_expert.swap(se);
        L.expert_slot.swap(es);
        L.stamp.swap(stamp);
        L.step = step;
    }
    L.pending = L.pending || (!miss_idx.empty() && cst == MOE_OK);
    L.released = false;                   // the release point covered the previous request only

    // device slot map of the layer (and the request's hit / miss masks)
    int32_t *hm = c->stage_map(layer, buf);
    for (int e = 0; e < d.E; e++) hm[e] = gm ? c->g.key_slot[key0 + e] : L.expert_slot[e];
    moe_status mst = cuda_status(cudaMemcpyAsync(d.dev_slot_map + (size_t)layer * d.E, hm,
                                                 sizeof(int32_t) * d.E, cudaMemcpyHostToDevice, cs),
                                 "moe_cache_request: slot map copy");
    if (mst == MOE_OK && d.dev_masks) {
        uint8_t *hit = c->stage_masks(layer, buf), *mis = hit + d.E;
        memset(hit, 0, 2 * (size_t)d.E);
        std::vector<char> missed(n, 0);
        if (cst == MOE_OK) for (int i : miss_idx) missed[i] = 1;
        for (int i = 0; i < n; i++) {
            if (missed[i]) mis[ids[i]] = 1;
            else if (hm[ids[i]] >= 0) hit[ids[i]] = 1;
        }
        mst = cuda_status(cudaMemcpyAsync(d.dev_masks + (size_t)layer * 2 * d.E, hit, 2 * (size_t)d.E,
                                          cudaMemcpyHostToDevice, cs),
                          "moe_cache_request: mask copy");
    }
    if (mst == MOE_OK) mst = cuda_status(cudaEventRecord(L.map_done[buf], cs), "cudaEventRecord");
    L.map_buf ^= 1;
    if (cst != MOE_OK) return cst;
    if (mst != MOE_OK) return mst;

    const int nm = (int)miss_idx.size();
    c->hits += n - nm;
    c->misses += nm;
    c->bytes += (int64_t)nm * (int64_t)(d.bytes_gate + d.bytes_up + d.bytes_down);
    if (n_miss) *n_miss = nm;
    for (int i = 0; i < n; i++) {
        if (slots) slots[i] = out_slot[i];
        if (evicted) evicted[i] = out_ev[i];
        if (miss) miss[i] = 0;
    }
    if (miss) for (int i : miss_idx) miss[i] = 1;
    return MOE_OK;
}

moe_status moe_cache_sync(moe_cache *c, int layer, moe_stream compute) {
    if (!c || layer < 0 || layer >= c->d.n_layers) { set_error("moe_cache_sync: bad cache or layer"); return MOE_ERR_INVALID_ARG; }
    auto &L = c->layers[layer];
    if (!L.pending) return MOE_OK;
    L.pending = false;
    cudaStream_t cs = (cudaStream_t)compute;
    harvest_waits(c, false);
    cudaEvent_t e0 = take_event(c), e1 = take_event(c);
    if (e0 && e1 && cudaEventRecord(e0, cs) == cudaSuccess) {
        moe_status st = cuda_status(cudaStreamWaitEvent(cs, L.copied, 0), "cudaStreamWaitEvent");
        if (st != MOE_OK) return st;
        st = cuda_status(cudaEventRecord(e1, cs), "cudaEventRecord");
        if (st != MOE_OK) return st;
        c->wait_pairs.emplace_back(e0, e1);
        return MOE_OK;
    }
    // no timing events: wait without measuring
    if (e0) c->free_events.push_back(e0);
    if (e1) c->free_events.push_back(e1);
    cudaGetLastError();
    return cuda_status(cudaStreamWaitEvent(cs, L.copied, 0), "cudaStreamWaitEvent");
}

moe_status moe_cache_release(moe_cache *c, int layer, moe_stream compute) {
    if (!c || layer < 0 || layer >= c->d.n_layers) { set_error("moe_cache_release: bad cache or layer"); return MOE_ERR_INVALID_ARG; }
    auto &L = c->layers[layer];
    moe_status st = cuda_status(cudaEventRecord(L.release_ev, (cudaStream_t)compute), "cudaEventRecord");
    L.released = st == MOE_OK;
    return st;
}

moe_status moe_cache_layer_masks(moe_cache *c, int layer, const uint8_t **hit,
                                 const uint8_t **miss) {
    if (!c || layer < 0 || layer >= c->d.n_layers || !c->d.dev_masks) {
        set_error("moe_cache_layer_masks: bad cache or layer, or the cache has no dev_masks");
        return MOE_ERR_INVALID_ARG;
    }
    const uint8_t *base = c->d.dev_masks + (size_t)layer * 2 * c->d.E;
    if (hit) *hit = base;
    if (miss) *miss = base + c->d.E;
    return MOE_OK;
}

moe_status moe_cache_layer_pool(moe_cache *c, int layer, moe_pool *out) {
    if (!c || !out || layer < 0 || layer >= c->d.n_layers) { set_error("moe_cache_layer_pool: bad argument"); return MOE_ERR_INVALID_ARG; }
    const moe_cache_desc &d = c->d;
    const size_t base = c->global ? 0 : (size_t)layer * d.n_slots;
    out->qtype = d.qtype;
    out->n_slots = c->global ? d.max_slots : d.n_slots;
    out->gate = (const char *)d.dev_gate + base * d.bytes_gate;
    out->up = (const char *)d.dev_up + base * d.bytes_up;
    out->down = (const char *)d.dev_down + base * d.bytes_down;
    out->slot_of_expert = d.dev_slot_map + (size_t)layer * d.E;
    return MOE_OK;
}

moe_status moe_cache_resize(moe_cache *c, int n_slots, int *n_evicted, int *n_moved,
                            moe_stream compute) {
    if (n_evicted) *n_evicted = 0;
    if (n_moved) *n_moved = 0;
    if (!c || !c->global) { set_error("moe_cache_resize: needs a global cache"); return MOE_ERR_INVALID_ARG; }
    const moe_cache_desc &d = c->d;
    if (n_slots < 1 || n_slots > d.max_slots) {
        set_error("moe_cache_resize: %d slots outside [1, %d]", n_slots, d.max_slots);
        return MOE_ERR_SHAPE;
    }
    auto &G = c->g;
    if (n_slots >= G.cap) {                 // growing only adds empty slots
        G.cap = n_slots;
        return MOE_OK;
    }
    cudaStream_t cs = (cudaStream_t)compute, xs = (cudaStream_t)d.copy_stream;
    // the moves below overwrite slots that kernels enqueued so far may still
    // read (entries just evicted): the copy stream waits for all of them
    moe_status st = cuda_status(cudaEventRecord(c->compute_ready, cs), "cudaEventRecord");
    if (st == MOE_OK) st = cuda_status(cudaStreamWaitEvent(xs, c->compute_ready, 0), "cudaStreamWaitEvent");
    if (st != MOE_OK) return st;
    int resident = 0;
    for (int s = 0; s < G.cap; s++) if (G.slot_key[s] >= 0) resident++;
    const int nk = d.n_layers * d.E;
    int ne = 0, nm = 0;
    while (resident > n_slots) {            // oldest stamp first, lower key on ties
        int victim = -1;
        for (int k = 0; k < nk; k++) {
            if (G.key_slot[k] < 0) continue;
            if (victim < 0 || G.stamp[k] < G.stamp[victim]) victim = k;
        }
        G.slot_key[G.key_slot[victim]] = -1;
        G.key_slot[victim] = -1;
        resident--;
        ne++;
    }
    for (int s = n_slots; s < G.cap && st == MOE_OK; s++) {   // compact into the first n_slots
        const int key = G.slot_key[s];
        if (key < 0) continue;
        int t = 0;
        while (G.slot_key[t] >= 0) t++;
        const void *src[3] = {(char *)d.dev_gate + (size_t)s * d.bytes_gate, (char *)d.dev_up + (size_t)s * d.bytes_up,
                              (char *)d.dev_down + (size_t)s * d.bytes_down};
        void *dst[3] = {(char *)d.dev_gate + (size_t)t * d.bytes_gate, (char *)d.dev_up + (size_t)t * d.bytes_up,
                        (char *)d.dev_down + (size_t)t * d.bytes_down};
        const size_t nb[3] = {d.bytes_gate, d.bytes_up, d.bytes_down};
        for (int q = 0; q < 3 && st == MOE_OK; q++)
            st = cuda_status(cudaMemcpyAsync(dst[q], src[q], nb[q], cudaMemcpyDeviceToDevice, xs),
                             "moe_cache_resize: move");
        G.slot_key[t] = key;
        G.slot_key[s] = -1;
        G.key_slot[key] = t;
        nm++;
    }
    // work enqueued on the compute stream after this call sees the moves done
    if (st == MOE_OK) st = cuda_status(cudaEventRecord(c->compute_ready, xs), "cudaEventRecord");
    if (st == MOE_OK) st = cuda_status(cudaStreamWaitEvent(cs, c->compute_ready, 0), "cudaStreamWaitEvent");
    G.cap = n_slots;
    if (n_evicted) *n_evicted = ne;
    if (n_moved) *n_moved = nm;
    return st;
}

moe_status moe_cache_stats(moe_cache *c, int64_t *hits, int64_t *misses, int64_t *bytes_copied,
                           int64_t *exposed_ns) {
    if (!c) { set_error("moe_cache_stats: NULL cache"); return MOE_ERR_INVALID_ARG; }
    if (hits) *hits = c->hits;
    if (misses) *misses = c->misses;
    if (bytes_copied) *bytes_copied = c->bytes;
    if (exposed_ns) {
        moe_status st = harvest_waits(c, true);
        if (st != MOE_OK) return st;
        *exposed_ns = c->exposed_ns;
    }
    return MOE_OK;
}

}  // extern "C"
