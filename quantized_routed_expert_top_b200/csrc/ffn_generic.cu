// ffn_generic.cu -- portable SIMT expert FFN for every shape and block type.
//
// Per permuted row pos (token t = perm[pos] / k, expert e = its segment):
//   H[pos, r]  = silu(x_t . W_gate,e[r]) * (x_t . W_up,e[r])      (fp32)
//   out[pos, d] = H[pos, :] . W_down,e[d]                           (fp32)
// One warp per weight row, lanes over 32-weight units (a block of the
// 32-weight types, a sub-block of the K-quants); each weight row is read once
// per group of kTokGroup tokens of the segment.  This path favours
// simplicity over speed: the tuned decode (GEMV) and prefill (tensor-core)
// paths live in their own files and are checked against the same oracle.
//
// Experts without tokens are skipped: every CTA compacts the list of active
// experts (count > 0 and, when a mask is given, mask != 0) in shared memory
// and walks (active expert, row tile) work items with a grid stride.  An
// active expert whose slot lies outside [0, n_slots) is left out and
// recorded as kErrBadSlot in the status word; no address is formed from it.
// perm == NULL means the identity grouping of T rows for a single expert
// (used for the always-on shared expert).
#include "moe_internal.cuh"
#include "sm100.cuh"

namespace moe {

constexpr int kGenWarps = 8;
constexpr int kTokGroup = 4;

// Build the active-expert list in shared memory; returns how many.
__device__ int build_active(const int32_t *offsets, const uint8_t *mask, const int32_t *slot_map,
                            int n_slots, int E, int *err, int *act) {
    __shared__ int n_act;
    if (threadIdx.x == 0) n_act = 0;
    __syncthreads();
    // order does not matter for correctness (work items are independent),
    // but keep it ascending for reproducible scheduling: one warp scans
    if (threadIdx.x < 32) {
        int base = 0;
        for (int e0 = 0; e0 < E; e0 += 32) {
            int e = e0 + threadIdx.x;
            bool on = false;
            if (e < E) {
                int c = (offsets ? __ldg(offsets + e + 1) - __ldg(offsets + e) : 1);
                on = c > 0 && (!mask || __ldg(mask + e));
                if (on) {
                    const int sl = slot_of(slot_map, e);
                    if (sl < 0 || sl >= n_slots) {
                        if (err) atomicCAS(err, 0, kErrBadSlot);
                        on = false;
                    }
                }
            }
            unsigned b = __ballot_sync(0xffffffffu, on);
            if (on) act[base + __popc(b & ((1u << threadIdx.x) - 1u))] = e;
            base += __popc(b);
        }
        if (threadIdx.x == 0) n_act = base;
    }
    __syncthreads();
    return n_act;
}

template <int QT, typename XT>
__global__ void __launch_bounds__(kGenWarps * 32)
ffn_gateup_generic_kernel(const XT *__restrict__ x, int T, int D, int F, int E, int k,
                          const int32_t *__restrict__ perm, const int32_t *__restrict__ offsets,
                          const uint8_t *__restrict__ gate, const uint8_t *__restrict__ up,
                          const int32_t *__restrict__ slot_map, int n_slots,
                          const uint8_t *__restrict__ mask, float *__restrict__ H, int *err) {
    extern __shared__ int act[];
    const int n_act = build_active(offsets, mask, slot_map, n_slots, E, err, act);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int nb = D / QK;
    const size_t row_bytes = qt_row_bytes(QT, D);
    const int tiles = (F + kGenWarps - 1) / kGenWarps;
    for (int w = blockIdx.x; w < n_act * tiles; w += gridDim.x) {
        const int e = act[w / tiles];
        const int r = (w % tiles) * kGenWarps + warp;
        if (r >= F) continue;
        const int seg0 = offsets ? __ldg(offsets + e) : 0;
        const int seg1 = offsets ? __ldg(offsets + e + 1) : T;
        const size_t slot = (size_t)slot_of(slot_map, e);
        const uint8_t *grow = gate + (slot * F + r) * row_bytes;
        const uint8_t *urow = up + (slot * F + r) * row_bytes;
        for (int p0 = seg0; p0 < seg1; p0 += kTokGroup) {
            int tok[kTokGroup];
#pragma unroll
            for (int q = 0; q < kTokGroup; q++) {
                int p = p0 + q;
                tok[q] = (p < seg1) ? (perm ? __ldg(perm + p) / k : p) : -1;
            }
            float ag[kTokGroup] = {}, au[kTokGroup] = {};
            for (int b = lane; b < nb; b += 32) {
                float wg[QK], wu[QK];
                decode_unit_global<QT>(grow, b, wg);
                decode_unit_global<QT>(urow, b, wu);
#pragma unroll
                for (int q = 0; q < kTokGroup; q++) {
                    if (tok[q] < 0) continue;
                    const size_t xo = (size_t)tok[q] * D + (size_t)b * QK;
#pragma unroll
                    for (int i = 0; i < QK; i++) {
                        float xv = load_act(x, xo + i);
                        ag[q] = fmaf(xv, wg[i], ag[q]);
                        au[q] = fmaf(xv, wu[i], au[q]);
                    }
                }
            }
#pragma unroll
            for (int q = 0; q < kTokGroup; q++) {
                float g = warp_sum(ag[q]);
                float u = warp_sum(au[q]);
                if (lane == 0 && tok[q] >= 0) H[(size_t)(p0 + q) * F + r] = silu(g) * u;
            }
        }
    }
}

template <int QT>
__global__ void __launch_bounds__(kGenWarps * 32)
ffn_down_generic_kernel(const float *__restrict__ H, int T, int D, int F, int E, int k,
                        const int32_t *__restrict__ offsets,
                        const uint8_t *__restrict__ down, const int32_t *__restrict__ slot_map,
                        int n_slots, const uint8_t *__restrict__ mask, float *__restrict__ out,
                        int *err) {
    extern __shared__ int act[];
    const int n_act = build_active(offsets, mask, slot_map, n_slots, E, err, act);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int nb = F / QK;
    const size_t row_bytes = qt_row_bytes(QT, F);
    const int tiles = (D + kGenWarps - 1) / kGenWarps;
    for (int w = blockIdx.x; w < n_act * tiles; w += gridDim.x) {
        const int e = act[w / tiles];
        const int d = (w % tiles) * kGenWarps + warp;
        if (d >= D) continue;
        const int seg0 = offsets ? __ldg(offsets + e) : 0;
        const int seg1 = offsets ? __ldg(offsets + e + 1) : T;
        const size_t slot = (size_t)slot_of(slot_map, e);
        const uint8_t *drow = down + (slot * D + d) * row_bytes;
        for (int p0 = seg0; p0 < seg1; p0 += kTokGroup) {
            float acc[kTokGroup] = {};
            for (int b = lane; b < nb; b += 32) {
                float wd[QK];
                decode_unit_global<QT>(drow, b, wd);
#pragma unroll
                for (int q = 0; q < kTokGroup; q++) {
                    if (p0 + q >= seg1) continue;
                    const float *h = H + (size_t)(p0 + q) * F + (size_t)b * QK;
#pragma unroll
                    for (int i = 0; i < QK; i++) acc[q] = fmaf(h[i], wd[i], acc[q]);
                }
            }
#pragma unroll
            for (int q = 0; q < kTokGroup; q++) {
                float v = warp_sum(acc[q]);
                if (lane == 0 && p0 + q < seg1) out[(size_t)(p0 + q) * D + d] = v;
            }
        }
    }
}

template <int QT>
static moe_status run_generic(const void *x, int x_dtype, int T, int D, int F, int E, int k,
                              const int32_t *perm, const int32_t *offsets, const moe_pool &pool,
                              const uint8_t *mask, float *H, float *out, int *err,
                              cudaStream_t s, Tracer *tr, bool shared) {
    const int grid = num_sms() * 4;
    const size_t sm = (size_t)E * sizeof(int);
    mark(tr, shared ? MOE_KERNEL_SHARED_GATEUP : MOE_KERNEL_GATEUP);
    if (x_dtype == MOE_BF16)
        ffn_gateup_generic_kernel<QT, __nv_bfloat16><<<grid, kGenWarps * 32, sm, s>>>(
            (const __nv_bfloat16 *)x, T, D, F, E, k, perm, offsets, (const uint8_t *)pool.gate,
            (const uint8_t *)pool.up, pool.slot_of_expert, pool.n_slots, mask, H, err);
    else
        ffn_gateup_generic_kernel<QT, float><<<grid, kGenWarps * 32, sm, s>>>(
            (const float *)x, T, D, F, E, k, perm, offsets, (const uint8_t *)pool.gate,
            (const uint8_t *)pool.up, pool.slot_of_expert, pool.n_slots, mask, H, err);
    moe_status st = cuda_status(cudaGetLastError(), "ffn_gateup_generic_kernel");
    if (st != MOE_OK) return st;
    mark(tr, shared ? MOE_KERNEL_SHARED_DOWN : MOE_KERNEL_DOWN);
    ffn_down_generic_kernel<QT><<<grid, kGenWarps * 32, sm, s>>>(
        H, T, D, F, E, k, offsets, (const uint8_t *)pool.down, pool.slot_of_expert, pool.n_slots,
        mask, out, err);
    return cuda_status(cudaGetLastError(), "ffn_down_generic_kernel");
}

moe_status launch_ffn_generic(const void *x, int x_dtype, int T, int D, int F, int E, int k,
                              const int32_t *perm, const int32_t *offsets, const moe_pool &pool,
                              const uint8_t *mask, float *H, float *out_rows, int *err,
                              cudaStream_t s, Tracer *tr, bool shared) {
#define MOE_RUN(QT)                                                                           \
    case QT:                                                                                  \
        return run_generic<QT>(x, x_dtype, T, D, F, E, k, perm, offsets, pool, mask, H,       \
                               out_rows, err, s, tr, shared);
    switch (pool.qtype) {
        MOE_RUN(MOE_Q4_0)
        MOE_RUN(MOE_Q4_1)
        MOE_RUN(MOE_Q5_0)
        MOE_RUN(MOE_Q5_1)
        MOE_RUN(MOE_Q8_0)
        MOE_RUN(MOE_Q4_K)
        MOE_RUN(MOE_Q6_K)
#undef MOE_RUN
    default:
        set_error("expert FFN: unsupported quant type %d", (int)pool.qtype);
        return MOE_ERR_UNSUPPORTED_QTYPE;
    }
}

}  // namespace moe
