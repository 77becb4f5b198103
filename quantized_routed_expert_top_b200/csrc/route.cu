// route.cu -- router logits, softmax, top-k and renormalised gates.
//
// L = x . W_r (+ b) in fp32; the top-k experts per token are taken in
// descending logit order with ties to the lower expert id; the gates are the
// softmax probabilities of the selected experts renormalised over the
// selection (equivalently a softmax over the selected logits).
//
// Two logit paths:
//  * small T (decode): split-K GEMV.  W_r is only D*E*4 bytes (1 MiB at
//    D=2048, E=128) but at T=1 one CTA cannot stream it fast, so the D rows
//    are split over many CTAs; each writes fp32 partial sums to the
//    workspace, and the CTA that finishes last (atomic ticket) adds the
//    partials in split order (deterministic), adds the bias and runs the
//    warp-per-token selection.  One launch.
//  * large T (prefill): a register-tiled SIMT GEMM writes the logits, then a
//    warp-per-token selection kernel.
// Logits stay fp32 end to end (no TF32): the tie rule compares logits at a
// 1e-5 resolution.
#include "moe_internal.cuh"
#include "permute.cuh"
#include "sm100.cuh"

#include <cooperative_groups.h>
#include <algorithm>
#include <cfloat>
#include <climits>
#include <mutex>

namespace moe {

constexpr int kSplitMaxT = 16;      // tokens handled by the split-K path
constexpr int kSplitRows = 32;      // D rows per split CTA

// --------------------------------------------------------------- selection
// Orderable key of a logit: a larger value gives a larger unsigned key; -0
// and +0 share one key, so equal logits tie and the lower id wins.
__device__ __forceinline__ unsigned order_key(float v) {
    const unsigned b = __float_as_uint(v == 0.0f ? 0.0f : v);
    return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

// One warp selects the top-k of a logit row L[0..E) (any memory space) and
// writes ids/gates for that token (and the ids to ids_copy when given).
// E <= 1024 (32 values per lane), k <= 32.  Each lane keeps its best
// remaining candidate; a round is two warp reductions (largest key, then
// the lowest id holding it) and only the winning lane rescans its values.
__device__ void warp_select(const float *L, int E, int k, int renorm,
                            int32_t *ids_out, float *gates_out, int32_t *ids_copy = nullptr) {
    const int lane = threadIdx.x & 31;
    const int per_lane = (E + 31) >> 5;
    unsigned taken = 0u;
    float bv = -INFINITY;
    int bi = INT_MAX;
    auto local_best = [&]() {
        bv = -INFINITY;
        bi = INT_MAX;
        for (int i = 0; i < per_lane; i++) {
            const int e = lane + 32 * i;
            if (e < E && !((taken >> i) & 1u)) {
                const float v = L[e];
                if (v > bv || (v == bv && e < bi)) { bv = v; bi = e; }
            }
        }
    };
    local_best();
    float my_v = -INFINITY;
    int my_i = INT_MAX;
    for (int j = 0; j < k; j++) {
        const unsigned key = (bi == INT_MAX) ? 0u : order_key(bv);
        const unsigned kmax = __reduce_max_sync(0xffffffffu, key);
        const unsigned cand = (bi != INT_MAX && key == kmax) ? (unsigned)bi : 0xffffffffu;
        const unsigned win = __reduce_min_sync(0xffffffffu, cand);
        const int wi = (win == 0xffffffffu) ? INT_MAX : (int)win;
        const float wv = __shfl_sync(0xffffffffu, bv, wi == INT_MAX ? 0 : (wi & 31));
        if (lane == j) { my_v = (wi == INT_MAX) ? -INFINITY : wv; my_i = wi; }
        if (wi != INT_MAX && (wi & 31) == lane) {
            taken |= 1u << (wi >> 5);
            local_best();
        }
    }
    // gates: lane j < k holds selection j; the first selection is the max
    const float m = __shfl_sync(0xffffffffu, my_v, 0);
    float ex = (lane < k) ? expf(my_v - m) : 0.0f;
    float denom;
    if (renorm) {
        denom = warp_sum(ex);
    } else {
        float z = 0.0f;
        for (int i = 0; i < per_lane; i++) {
            int e = lane + 32 * i;
            if (e < E) z += expf(L[e] - m);
        }
        denom = warp_sum(z);
    }
    if (lane < k) {
        ids_out[lane] = my_i;
        gates_out[lane] = ex / denom;
        if (ids_copy) ids_copy[lane] = my_i;
    }
}

// All threads of a block select the top-k of one token's logits L[0..E)
// (shared memory): each element's rank is the number of elements that beat
// it (larger logit, or equal logit and lower id); ranks below k are the
// selection, in order.  One pass of compares instead of k dependent warp
// reductions.  NaN logits are never selected.  key: shared uint32[E];
// sel_v / sel_i: shared [32].  Writes ids/gates (and ids_copy) for the
// token; ends with the block synchronised.
__device__ void block_select(const float *L, unsigned *key, float *sel_v, int *sel_i, int E, int k,
                             int renorm, int32_t *ids_out, float *gates_out, int32_t *ids_copy) {
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        const float v = L[e];
        key[e] = (v != v) ? 0u : order_key(v);
    }
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        const unsigned kv = key[e];
        if (kv == 0u) continue;                       // NaN
        int r = 0;
#pragma unroll 4
        for (int e2 = 0; e2 < E; e2++) {
            const unsigned kw = key[e2];
            r += (kw > kv) | ((kw == kv) & (e2 < e));
        }
        if (r < k) {
            sel_i[r] = e;
            sel_v[r] = L[e];
        }
    }
    __syncthreads();
    if (threadIdx.x < 32) {
        const int lane = threadIdx.x;
        const float my_v = (lane < k) ? sel_v[lane] : -INFINITY;
        const int my_i = (lane < k) ? sel_i[lane] : INT_MAX;
        // gates exactly as warp_select computes them
        const float m = __shfl_sync(0xffffffffu, my_v, 0);
        float ex = (lane < k) ? expf(my_v - m) : 0.0f;
        float denom;
        if (renorm) {
            denom = warp_sum(ex);
        } else {
            float z = 0.0f;
            for (int e = lane; e < E; e += 32) z += expf(L[e] - m);
            denom = warp_sum(z);
        }
        if (lane < k) {
            ids_out[lane] = my_i;
            gates_out[lane] = ex / denom;
            if (ids_copy) ids_copy[lane] = my_i;
        }
    }
    __syncthreads();
}

// ------------------------------------------------- small T: split-K + select
template <typename XT>
__global__ void __launch_bounds__(1024)
route_splitk_kernel(const XT *__restrict__ x, const float *__restrict__ W,
                    const float *__restrict__ bias, int T, int D, int E, int k,
                    int renorm, int nsplit, float *__restrict__ partial,
                    unsigned *__restrict__ ticket, int32_t *__restrict__ ids,
                    float *__restrict__ gates, float *__restrict__ logits_out) {
    extern __shared__ float smem[];
    float *xs = smem;                         // [T][kSplitRows]
    __shared__ int s_last;
    const int s = blockIdx.x;
    const int i0 = s * kSplitRows;
    const int rows = min(kSplitRows, D - i0);
    for (int idx = threadIdx.x; idx < T * kSplitRows; idx += blockDim.x) {
        int t = idx / kSplitRows, r = idx % kSplitRows;
        xs[idx] = (r < rows) ? load_act(x, (size_t)t * D + i0 + r) : 0.0f;
    }
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        float acc[kSplitMaxT];
#pragma unroll
        for (int t = 0; t < kSplitMaxT; t++) acc[t] = 0.0f;
        for (int r = 0; r < rows; r++) {
            float w = __ldg(W + (size_t)(i0 + r) * E + e);
#pragma unroll
            for (int t = 0; t < kSplitMaxT; t++)
                if (t < T) acc[t] = fmaf(xs[t * kSplitRows + r], w, acc[t]);
        }
#pragma unroll
        for (int t = 0; t < kSplitMaxT; t++)
            if (t < T) partial[((size_t)s * T + t) * E + e] = acc[t];
    }
    // last CTA to finish reduces the partials and selects
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) s_last = (atomicAdd(ticket, 1u) == (unsigned)(nsplit - 1));
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    float *Ls = smem;                          // reuse: [T][E]
    for (int idx = threadIdx.x; idx < T * E; idx += blockDim.x) {
        int t = idx / E, e = idx % E;
        float v = 0.0f;
        for (int q = 0; q < nsplit; q++) v += __ldcg(partial + ((size_t)q * T + t) * E + e);
        if (bias) v += __ldg(bias + e);
        Ls[idx] = v;
        if (logits_out) logits_out[idx] = v;
    }
    __syncthreads();
    const int warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
    for (int t = warp; t < T; t += nwarps)
        warp_select(Ls + (size_t)t * E, E, k, renorm, ids + (size_t)t * k, gates + (size_t)t * k);
    if (threadIdx.x == 0) *ticket = 0u;        // ready for the next call
}

// ------------------------------------------------------ large T: tiled GEMM
constexpr int kTM = 64, kTN = 64, kTK = 16;  // 256 threads, 4x4 outputs each

template <typename XT>
__global__ void __launch_bounds__(256)
route_logits_tiled_kernel(const XT *__restrict__ x, const float *__restrict__ W,
                          const float *__restrict__ bias, int T, int D, int E,
                          float *__restrict__ logits) {
    __shared__ float As[kTK][kTM + 4];
    __shared__ float Bs[kTK][kTN + 4];
    const int t0 = blockIdx.x * kTM, e0 = blockIdx.y * kTN;
    const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
    float acc[4][4] = {};
    for (int k0 = 0; k0 < D; k0 += kTK) {
        for (int idx = threadIdx.x; idx < kTM * kTK; idx += 256) {
            int m = idx / kTK, kk = idx % kTK;
            int t = t0 + m;
            As[kk][m] = (t < T) ? load_act(x, (size_t)t * D + k0 + kk) : 0.0f;
        }
        for (int idx = threadIdx.x; idx < kTK * kTN; idx += 256) {
            int kk = idx / kTN, n = idx % kTN;
            int e = e0 + n;
            Bs[kk][n] = (e < E) ? __ldg(W + (size_t)(k0 + kk) * E + e) : 0.0f;
        }
        __syncthreads();
#pragma unroll
        for (int kk = 0; kk < kTK; kk++) {
            float a[4], b[4];
#pragma unroll
            for (int i = 0; i < 4; i++) a[i] = As[kk][ty * 4 + i];
#pragma unroll
            for (int j = 0; j < 4; j++) b[j] = Bs[kk][tx * 4 + j];
#pragma unroll
            for (int i = 0; i < 4; i++)
#pragma unroll
                for (int j = 0; j < 4; j++) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
        }
        __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 4; i++) {
        int t = t0 + ty * 4 + i;
        if (t >= T) continue;
#pragma unroll
        for (int j = 0; j < 4; j++) {
            int e = e0 + tx * 4 + j;
            if (e < E) logits[(size_t)t * E + e] = acc[i][j] + (bias ? __ldg(bias + e) : 0.0f);
        }
    }
}

// Large-T router logits, register-tiled SIMT GEMM: a CTA computes 64 tokens
// x 128 experts, a thread 4 tokens x 8 experts (two runs of 4, so its
// 16-byte shared loads of W_r are conflict-free), with the next 32-row
// K-tile loaded into registers while the current one is used.  With
// nsplit > 1 the K range is cut into nsplit equal segments (blockIdx.z): a
// segment's partial is one thread's fmaf chain over its k in ascending
// order, written without the bias to part[z]; route_reduce_select_kernel
// adds the partials in segment order, then the bias.  (More CTAs per SM:
// at T = 8192 one segment gives 128 CTAs of 8 warps for 148 SMs.)
// E % 4 == 0.
constexpr int kSM = 64, kSN = 128, kSK = 32;
constexpr int kLgSplit = 4;          // K segments when T is large
__host__ __device__ inline int logits_nsplit(int T, int D) {
    return (T >= 512 && D % (kLgSplit * kSK) == 0) ? kLgSplit : 1;
}

template <typename XT>
__global__ void __launch_bounds__(256)
route_logits_sgemm_kernel(const XT *__restrict__ x, const float *__restrict__ W,
                          const float *__restrict__ bias, int T, int D, int E,
                          float *__restrict__ logits, int kseg, int xvec) {
    extern __shared__ __align__(16) float smem_lg[];
    float *As = smem_lg;                                   // [2][kSK][kSM + 1]
    float *Bs = As + 2 * kSK * (kSM + 1);                  // [2][kSK][kSN + 4]
    const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
    const int t0 = blockIdx.x * kSM, e0 = blockIdx.y * kSN;
    const int kbeg = blockIdx.z * kseg, kend = kbeg + kseg;
    if (gridDim.z > 1) {                  // partial of segment z, no bias
        logits += (size_t)blockIdx.z * T * E;
        bias = nullptr;
    }
    // global -> register staging: A = 8 consecutive k of one token, B = 4
    // float4 of W_r rows
    const int am = tid >> 2, ak = (tid & 3) * 8;
    const int bc = (tid & 31) * 4, br = tid >> 5;
    float ra[8];
    float4 rb[4];
    auto load = [&](int k0) {
        const int t = t0 + am;
        const size_t xo = (size_t)t * D + k0 + ak;
        if (t >= T) {
#pragma unroll
            for (int i = 0; i < 8; i++) ra[i] = 0.f;
        } else if (xvec) {                 // 8 activations in 16 (bf16) or 32 (fp32) bytes
            if constexpr (sizeof(XT) == 2) {
                const uint4 w = __ldg(reinterpret_cast<const uint4 *>(x + xo));
                const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                for (int i = 0; i < 4; i++) {
                    ra[2 * i] = __uint_as_float(u[i] << 16);
                    ra[2 * i + 1] = __uint_as_float(u[i] & 0xFFFF0000u);
                }
            } else {
                const float4 w0 = __ldg(reinterpret_cast<const float4 *>(x + xo));
                const float4 w1 = __ldg(reinterpret_cast<const float4 *>(x + xo) + 1);
                ra[0] = w0.x; ra[1] = w0.y; ra[2] = w0.z; ra[3] = w0.w;
                ra[4] = w1.x; ra[5] = w1.y; ra[6] = w1.z; ra[7] = w1.w;
            }
        } else {
#pragma unroll
            for (int i = 0; i < 8; i++) ra[i] = load_act(x, xo + i);
        }
#pragma unroll
        for (int i = 0; i < 4; i++) {
            const int e = e0 + bc;
            rb[i] = (e < E) ? __ldg(reinterpret_cast<const float4 *>(W + (size_t)(k0 + br + 8 * i) * E + e))
                            : make_float4(0.f, 0.f, 0.f, 0.f);
        }
    };
    auto store = [&](int buf) {
        float *a = As + buf * kSK * (kSM + 1);
        float *b = Bs + buf * kSK * (kSN + 4);
#pragma unroll
        for (int i = 0; i < 8; i++) a[(ak + i) * (kSM + 1) + am] = ra[i];
#pragma unroll
        for (int i = 0; i < 4; i++) *reinterpret_cast<float4 *>(b + (br + 8 * i) * (kSN + 4) + bc) = rb[i];
    };
    float acc[4][8];
#pragma unroll
    for (int i = 0; i < 4; i++)
#pragma unroll
        for (int j = 0; j < 8; j++) acc[i][j] = 0.f;
    load(kbeg);
    store(0);
    __syncthreads();
    int buf = 0;
    for (int k0 = kbeg; k0 < kend; k0 += kSK) {
        if (k0 + kSK < kend) load(k0 + kSK);
        const float *a = As + buf * kSK * (kSM + 1);
        const float *b = Bs + buf * kSK * (kSN + 4);
#pragma unroll
        for (int kk = 0; kk < kSK; kk++) {
            float av[4];
#pragma unroll
            for (int i = 0; i < 4; i++) av[i] = a[kk * (kSM + 1) + ty * 4 + i];
            const float4 b0 = *reinterpret_cast<const float4 *>(b + kk * (kSN + 4) + tx * 4);
            const float4 b1 = *reinterpret_cast<const float4 *>(b + kk * (kSN + 4) + 64 + tx * 4);
            const float bv[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
            for (int i = 0; i < 4; i++)
#pragma unroll
                for (int j = 0; j < 8; j++) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
        }
        if (k0 + kSK < kend) {
            store(buf ^ 1);
            __syncthreads();
            buf ^= 1;
        }
    }
#pragma unroll
    for (int i = 0; i < 4; i++) {
        const int t = t0 + ty * 4 + i;
        if (t >= T) continue;
#pragma unroll
        for (int j = 0; j < 8; j++) {
            const int e = e0 + (j < 4 ? tx * 4 + j : 64 + tx * 4 + j - 4);
            if (e < E) logits[(size_t)t * E + e] = acc[i][j] + (bias ? __ldg(bias + e) : 0.0f);
        }
    }
}

__global__ void __launch_bounds__(256)
route_select_kernel(const float *__restrict__ logits, const float *__restrict__ bias_if_raw,
                    int T, int E, int k, int renorm, int32_t *__restrict__ ids,
                    float *__restrict__ gates, float *__restrict__ logits_copy) {
    const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    if (warp >= T) return;
    const float *L = logits + (size_t)warp * E;
    if (bias_if_raw || logits_copy) {
        // routing from given logits with a bias or a requested copy: stage
        // the biased row in the copy buffer and select from there
        const int lane = threadIdx.x & 31;
        float *C = logits_copy + (size_t)warp * E;
        for (int e = lane; e < E; e += 32) C[e] = L[e] + (bias_if_raw ? __ldg(bias_if_raw + e) : 0.0f);
        __syncwarp();
        L = C;
    }
    warp_select(L, E, k, renorm, ids + (size_t)warp * k, gates + (size_t)warp * k);
}

// Sum of the nsplit logit partials in segment order, plus the bias, into L
// (one warp per token), then the selection on that row.
__global__ void __launch_bounds__(256)
route_reduce_select_kernel(const float *__restrict__ part, int nsplit, const float *__restrict__ bias,
                           int T, int E, int k, int renorm, int32_t *__restrict__ ids,
                           float *__restrict__ gates, float *__restrict__ L) {
    const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    if (warp >= T) return;
    const int lane = threadIdx.x & 31;
    float *row = L + (size_t)warp * E;
    for (int e = lane; e < E; e += 32) {
        float v = __ldg(part + (size_t)warp * E + e);
        for (int z = 1; z < nsplit; z++) v += __ldg(part + ((size_t)z * T + warp) * E + e);
        row[e] = v + (bias ? __ldg(bias + e) : 0.0f);
    }
    __syncwarp();
    warp_select(row, E, k, renorm, ids + (size_t)warp * k, gates + (size_t)warp * k);
}

// ------------------------------------ small T: one cluster, DSMEM reduction
// Latency-bound: at T <= 16 the router reads W_r (D*E*4 bytes, 1 MiB at
// D=2048, E=128) once and does T FMAs per weight, so what matters is how
// many dependent memory round trips the critical path holds.  One cluster
// of CS CTAs:
//  1. CTA r takes rows [r*rpc, (r+1)*rpc) of W_r.  Thread (row group rg,
//     expert quad q) issues all its 16-byte row loads at once, then does
//     the FMAs for every token; the row groups are summed in a fixed order
//     in shared memory: CTA partial P_r[t][e].
//  2. cluster barrier; CTA r finalises tokens t = r, r + CS, ...: the CS
//     partials of the token are added in rank order through distributed
//     shared memory (deterministic), plus the bias (prefetched at start),
//     and the whole CTA selects by ranks.  The selected ids are also stored
//     straight into CTA 0's shared memory.
//  3. cluster barrier; CTA 0 runs the stable permutation over all ids.
constexpr int kClusterCTAs = 16;
constexpr int kRouteThreads = 256;
constexpr int kRouteBatch = 16;      // 16-byte W_r loads in flight per thread

namespace cg = cooperative_groups;

struct RouteGeo {
    int rpc, Q, RG;                    // rows per CTA, expert quads, row groups
};
// the row-group sums; later (CTA 0) the permutation histograms [8][E]
__host__ __device__ inline size_t route_red_floats(const RouteGeo &g, int TT, int E) {
    const size_t a = (size_t)g.RG * TT * E, b = (size_t)8 * E;
    return a > b ? a : b;
}
__host__ __device__ inline RouteGeo route_geo(int D, int E) {
    RouteGeo g;
    g.rpc = (D + kClusterCTAs - 1) / kClusterCTAs;
    g.Q = E / 4;
    g.RG = kRouteThreads / g.Q;
    return g;
}

template <typename XT, int TT>
__global__ void __launch_bounds__(kRouteThreads)
route_cluster_kernel(const XT *__restrict__ x, const float *__restrict__ W,
                     const float *__restrict__ bias, int T, int D, int E, int k, int renorm,
                     int32_t *__restrict__ ids, float *__restrict__ gates,
                     float *__restrict__ logits_out, int32_t *__restrict__ counts,
                     int32_t *__restrict__ offsets, int32_t *__restrict__ perm,
                     int32_t *__restrict__ inv) {
    // TT: tokens rounded up to 1, 2, 4, 8 or 16 (padding tokens are zero)
    extern __shared__ __align__(128) uint8_t smem_rc[];
    __shared__ int32_t scratch[32 + 8 * 32 + 1];
    constexpr int CS = kClusterCTAs;
    cg::cluster_group cluster = cg::this_cluster();
    const int rank = (int)cluster.block_rank();
    const int tid = threadIdx.x;
    const RouteGeo geo = route_geo(D, E);
    const int r0 = min(D, rank * geo.rpc), r1 = min(D, r0 + geo.rpc);
    const int rows = r1 - r0;
    const int q = tid % geo.Q, rg = tid / geo.Q;
    // the expert-FFN grid that follows may launch now: it stages its
    // activations and then waits (griddepcontrol.wait) for this grid
    pdl_launch_dependents();

    float *xs = (float *)smem_rc;                             // [rpc][TT]
    float *red = xs + round_up((size_t)geo.rpc * TT, 4);      // [RG][TT][E]; red[0] = P_r
    float *bias_s = red + route_red_floats(geo, TT, E);       // [E]
    float *Lrow = bias_s + E;                                 // [E]
    unsigned *key = (unsigned *)(Lrow + E);                   // [E]
    float *sel_v = (float *)(key + E);                        // [32]
    int32_t *sel_i = (int32_t *)(sel_v + 32);                 // [32]
    int32_t *ids_all = sel_i + 32;                            // [T * k] (rank 0)
    int32_t *hist = (int32_t *)red;                           // [8 * E] (rank 0, after step 2)

    // activations of this CTA's rows and the bias: first loads in flight
    for (int i = tid; i < rows * TT; i += kRouteThreads) {
        const int r = i / TT, t = i % TT;
        xs[i] = (t < T) ? load_act(x, (size_t)t * D + r0 + r) : 0.f;
    }
    for (int e = tid; e < E; e += kRouteThreads) bias_s[e] = bias ? __ldg(bias + e) : 0.f;

    float acc[4][TT];
#pragma unroll
    for (int j = 0; j < 4; j++)
#pragma unroll
        for (int t = 0; t < TT; t++) acc[j][t] = 0.f;
    const bool active = rg < geo.RG;
    const int my_rows = active ? (rows - rg + geo.RG - 1) / geo.RG : 0;
    const float4 *Wq = reinterpret_cast<const float4 *>(W + (size_t)(r0 + rg) * E) + q;
    const size_t wstep = (size_t)geo.RG * E / 4;              // float4s between my rows
    bool synced = false;
    for (int b0 = 0; b0 < my_rows || !synced; b0 += kRouteBatch) {
        float4 w[kRouteBatch];
#pragma unroll
        for (int i = 0; i < kRouteBatch; i++)
            if (b0 + i < my_rows) w[i] = __ldg(Wq + (size_t)(b0 + i) * wstep);
        if (!synced) {                     // xs complete (its loads were issued first)
            __syncthreads();
            synced = true;
        }
#pragma unroll
        for (int i = 0; i < kRouteBatch; i++) {
            if (b0 + i >= my_rows) break;
            const float *xr = xs + (size_t)(rg + (b0 + i) * geo.RG) * TT;
            float xv[TT];
            if constexpr (TT % 4 == 0) {
#pragma unroll
                for (int t = 0; t < TT; t += 4) {
                    const float4 q4 = *reinterpret_cast<const float4 *>(xr + t);
                    xv[t] = q4.x; xv[t + 1] = q4.y; xv[t + 2] = q4.z; xv[t + 3] = q4.w;
                }
            } else {
#pragma unroll
                for (int t = 0; t < TT; t++) xv[t] = xr[t];
            }
#pragma unroll
            for (int t = 0; t < TT; t++) {
                acc[0][t] = fmaf(xv[t], w[i].x, acc[0][t]);
                acc[1][t] = fmaf(xv[t], w[i].y, acc[1][t]);
                acc[2][t] = fmaf(xv[t], w[i].z, acc[2][t]);
                acc[3][t] = fmaf(xv[t], w[i].w, acc[3][t]);
            }
        }
    }
    // row groups -> P_r[t][e] (= red[0]), summed in row-group order
    if (active)
#pragma unroll
        for (int t = 0; t < TT; t++)
            *reinterpret_cast<float4 *>(red + ((size_t)rg * TT + t) * E + 4 * q) =
                make_float4(acc[0][t], acc[1][t], acc[2][t], acc[3][t]);
    __syncthreads();
    if (geo.RG > 1)
        for (int i = tid; i < T * E; i += kRouteThreads) {
            float v = red[i];
            for (int g = 1; g < geo.RG; g++) v += red[(size_t)g * TT * E + i];
            red[i] = v;
        }
    cluster.sync();

    // finalise this CTA's tokens: partials summed in rank order (DSMEM)
    int32_t *ids0 = cluster.map_shared_rank(ids_all, 0);
    for (int t = rank; t < T; t += CS) {
        for (int e = tid; e < E; e += kRouteThreads) {
            float pv[CS];
#pragma unroll
            for (int r = 0; r < CS; r++) pv[r] = cluster.map_shared_rank(red, r)[t * E + e];
            float v = 0.f;
#pragma unroll
            for (int r = 0; r < CS; r++) v += pv[r];
            v += bias_s[e];
            Lrow[e] = v;
            if (logits_out) logits_out[(size_t)t * E + e] = v;
        }
        __syncthreads();
        block_select(Lrow, key, sel_v, sel_i, E, k, renorm, ids + (size_t)t * k, gates + (size_t)t * k,
                     perm ? ids0 + t * k : nullptr);
    }
    cluster.sync();                        // ids in CTA 0; partials no longer read
    if (perm && rank == 0)
        block_permute<kRouteThreads / 32>(ids_all, T * k, E, hist, scratch, counts, offsets, perm, inv);
}

// ------------------------------------------ given logits: select + permute
// One CTA (small T): warps select tokens, then the stable permutation.
__global__ void __launch_bounds__(kRouteThreads)
select_permute_kernel(const float *__restrict__ logits, const float *__restrict__ bias, int T,
                      int E, int k, int renorm, int32_t *__restrict__ ids,
                      float *__restrict__ gates, float *__restrict__ logits_copy,
                      int32_t *__restrict__ counts, int32_t *__restrict__ offsets,
                      int32_t *__restrict__ perm, int32_t *__restrict__ inv) {
    extern __shared__ __align__(128) uint8_t smem_sp[];
    __shared__ int32_t scratch[32 + 8 * 32 + 1];
    float *Ls = (float *)smem_sp;                                // [T][E]
    int32_t *ids_s = (int32_t *)(Ls + (size_t)T * E);         // [T * k]
    int32_t *hist = ids_s + T * k;                            // [8][E]
    for (int i = threadIdx.x; i < T * E; i += kRouteThreads) {
        float v = logits[i];
        if (bias) v += __ldg(bias + i % E);
        Ls[i] = v;
        if (logits_copy) logits_copy[i] = v;
    }
    __syncthreads();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int t = warp; t < T; t += kRouteThreads / 32) {
        warp_select(Ls + (size_t)t * E, E, k, renorm, ids + (size_t)t * k, gates + (size_t)t * k);
        __syncwarp();
        if (lane < k) ids_s[t * k + lane] = __ldcg(ids + (size_t)t * k + lane);
    }
    __syncthreads();
    if (perm) block_permute<kRouteThreads / 32>(ids_s, T * k, E, hist, scratch, counts, offsets, perm, inv);
}

// ------------------------------------------------------------------- host
// The split-K router launch shared by moe_route (T <= 16 without the cluster
// kernel) and moe_route_noalloc.
static moe_status launch_splitk(const void *x, int x_dtype, const float *w_router,
                                const float *bias, int T, int D, int E, int k, int renorm,
                                int nsplit, float *partial, unsigned *ticket, int32_t *ids,
                                float *gates, float *logits, cudaStream_t s, const char *what) {
    int threads = (int)round_up(E, 32);
    if (threads < 128) threads = 128;
    const size_t sm = (size_t)std::max(T * kSplitRows, T * E) * sizeof(float);
    cudaError_t e;
    if (x_dtype == MOE_BF16) {
        auto kern = route_splitk_kernel<__nv_bfloat16>;
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
        if (e != cudaSuccess) return cuda_status(e, what);
        kern<<<nsplit, threads, sm, s>>>((const __nv_bfloat16 *)x, w_router, bias, T, D, E, k,
                                         renorm, nsplit, partial, ticket, ids, gates, logits);
    } else {
        auto kern = route_splitk_kernel<float>;
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
        if (e != cudaSuccess) return cuda_status(e, what);
        kern<<<nsplit, threads, sm, s>>>((const float *)x, w_router, bias, T, D, E, k, renorm,
                                         nsplit, partial, ticket, ids, gates, logits);
    }
    return cuda_status(cudaGetLastError(), what);
}

static size_t splitk_partial_bytes(int T, int D, int E) {
    int nsplit = (D + kSplitRows - 1) / kSplitRows;
    return (size_t)nsplit * T * E * sizeof(float);
}

size_t route_ws_bytes(int T, int D, int E, int k) {
    (void)k;
    Carver c(nullptr, 0);
    c.take<unsigned>(64);
    if (T <= kSplitMaxT) {
        c.take<char>(splitk_partial_bytes(T, D, E));
    } else {
        c.take<float>((size_t)T * E);    // logits scratch when none requested
        if (logits_nsplit(T, D) > 1) c.take<float>((size_t)logits_nsplit(T, D) * T * E);   // partials
    }
    return c.off;
}

static int t_bucket(int T) { return T <= 1 ? 1 : T <= 2 ? 2 : T <= 4 ? 4 : T <= 8 ? 8 : 16; }

static size_t cluster_smem_bytes(int T, int D, int E, int k) {
    const RouteGeo g = route_geo(D, E);
    const int TT = t_bucket(T);
    return (round_up((size_t)g.rpc * TT, 4) + route_red_floats(g, TT, E) + 3 * (size_t)E + 64) * 4 +
           (size_t)T * k * 4 + 256;
}

static bool cluster_route_ok(int T, int D, int E, int k, const void *w_router) {
    return w_router && T >= 1 && T <= kSplitMaxT && E % 4 == 0 && E / 4 <= kRouteThreads &&
           cluster_smem_bytes(T, D, E, k) <= 200 * 1024;
}

static bool select_permute_ok(int T, int E, int k) {
    return (size_t)T * E * 4 + (size_t)T * k * 4 + 8 * (size_t)E * 4 <= 200 * 1024 && T <= 64;
}

template <typename XT, int TT>
static cudaError_t launch_cluster(const void *x, const float *W, const float *bias, int T, int D,
                                  int E, int k, int renorm, int32_t *ids, float *gates,
                                  float *logits, int32_t *counts, int32_t *offsets, int32_t *perm,
                                  int32_t *inv, cudaStream_t s) {
    auto kern = route_cluster_kernel<XT, TT>;
    const size_t sm = cluster_smem_bytes(T, D, E, k);
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(kClusterCTAs);
    cfg.blockDim = dim3(kRouteThreads);
    cfg.dynamicSmemBytes = sm;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = kClusterCTAs;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, (const XT *)x, W, bias, T, D, E, k, renorm, ids, gates,
                              logits, counts, offsets, perm, inv);
}

moe_status launch_route_permute(const void *x, int x_dtype, const float *w_router,
                                const float *bias, int T, int D, int E, int k, int renorm,
                                int32_t *ids, float *gates, float *logits, int32_t *counts,
                                int32_t *offsets, int32_t *perm, int32_t *inv, int *err,
                                void *ws, size_t ws_bytes, cudaStream_t s, Tracer *tr,
                                bool *permuted) {
    *permuted = false;
    if (cluster_route_ok(T, D, E, k, w_router)) {
        mark(tr, MOE_KERNEL_ROUTE);
        cudaError_t e;
        const bool bf = x_dtype == MOE_BF16;
        const int tt = t_bucket(T);
#define MOE_CL(TB)                                                                                \
    e = bf ? launch_cluster<__nv_bfloat16, TB>(x, w_router, bias, T, D, E, k, renorm, ids, gates, \
                                               logits, counts, offsets, perm, inv, s)             \
           : launch_cluster<float, TB>(x, w_router, bias, T, D, E, k, renorm, ids, gates, logits, \
                                       counts, offsets, perm, inv, s)
        if (tt == 1) MOE_CL(1); else if (tt == 2) MOE_CL(2); else if (tt == 4) MOE_CL(4);
        else if (tt == 8) MOE_CL(8); else MOE_CL(16);
#undef MOE_CL
        if (e != cudaSuccess) return cuda_status(e, "route_cluster_kernel");
        *permuted = perm != nullptr;
        return MOE_OK;
    }
    if (!w_router && perm && select_permute_ok(T, E, k)) {
        const size_t sm = (size_t)T * E * 4 + (size_t)T * k * 4 + 8 * (size_t)E * 4;
        cudaError_t e = cudaFuncSetAttribute(select_permute_kernel,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
        if (e != cudaSuccess) return cuda_status(e, "select_permute_kernel smem attribute");
        mark(tr, MOE_KERNEL_ROUTE_SELECT);
        select_permute_kernel<<<1, kRouteThreads, sm, s>>>((const float *)x, bias, T, E, k, renorm,
                                                           ids, gates, logits, counts, offsets,
                                                           perm, inv);
        *permuted = true;
        return cuda_status(cudaGetLastError(), "select_permute_kernel");
    }
    return launch_route(x, x_dtype, w_router, bias, T, D, E, k, renorm, ids, gates, logits, ws,
                        ws_bytes, s, tr);
}

moe_status launch_route(const void *x, int x_dtype, const float *w_router,
                        const float *bias, int T, int D, int E, int k, int renorm,
                        int32_t *ids, float *gates, float *logits, void *ws,
                        size_t ws_bytes, cudaStream_t s, Tracer *tr) {
    Carver c(ws, ws_bytes);
    // 64-word header: word 0 is the status word, word 1 the completion ticket
    unsigned *ticket = c.take<unsigned>(64) + 1;
    if (w_router == nullptr) {
        // x holds the logits [T, E] fp32
        float *copy = logits;
        if (bias && !copy) {
            copy = c.take<float>((size_t)T * E);
            if (!c.fits()) { set_error("moe_route: workspace too small"); return MOE_ERR_WORKSPACE; }
        }
        int blocks = (T * 32 + 255) / 256;
        mark(tr, MOE_KERNEL_ROUTE_SELECT);
        route_select_kernel<<<blocks, 256, 0, s>>>((const float *)x, bias, T, E, k, renorm,
                                                   ids, gates, copy);
        return cuda_status(cudaGetLastError(), "route_select_kernel");
    }
    if (T <= kSplitMaxT) {
        float *partial = (float *)c.take<char>(splitk_partial_bytes(T, D, E));
        if (!c.fits()) { set_error("moe_route: workspace too small"); return MOE_ERR_WORKSPACE; }
        const int nsplit = (D + kSplitRows - 1) / kSplitRows;
        mark(tr, MOE_KERNEL_ROUTE);
        return launch_splitk(x, x_dtype, w_router, bias, T, D, E, k, renorm, nsplit, partial,
                             ticket, ids, gates, logits, s, "route_splitk_kernel");
    }
    float *L = logits;
    if (!L) {
        L = c.take<float>((size_t)T * E);
        if (!c.fits()) { set_error("moe_route: workspace too small"); return MOE_ERR_WORKSPACE; }
    }
    mark(tr, MOE_KERNEL_ROUTE_LOGITS);
    const int nsplit = E % 4 == 0 ? logits_nsplit(T, D) : 1;
    float *part = nullptr;
    if (nsplit > 1) {
        part = c.take<float>((size_t)nsplit * T * E);
        if (!c.fits()) { set_error("moe_route: workspace too small"); return MOE_ERR_WORKSPACE; }
    }
    if (E % 4 == 0) {
        const dim3 grid((T + kSM - 1) / kSM, (E + kSN - 1) / kSN, nsplit);
        const size_t sm = (size_t)(2 * kSK * (kSM + 1) + 2 * kSK * (kSN + 4)) * sizeof(float);
        float *dst = nsplit > 1 ? part : L;
        // 16-byte loads of 8 activations: x 16-byte aligned (rows then are too: D % 32 == 0)
        const int xvec = ((uintptr_t)x % 16) == 0;
        cudaError_t e;
        if (x_dtype == MOE_BF16) {
            e = cudaFuncSetAttribute(route_logits_sgemm_kernel<__nv_bfloat16>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
            if (e == cudaSuccess)
                route_logits_sgemm_kernel<__nv_bfloat16><<<grid, 256, sm, s>>>(
                    (const __nv_bfloat16 *)x, w_router, bias, T, D, E, dst, D / nsplit, xvec);
        } else {
            e = cudaFuncSetAttribute(route_logits_sgemm_kernel<float>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
            if (e == cudaSuccess)
                route_logits_sgemm_kernel<float><<<grid, 256, sm, s>>>((const float *)x, w_router,
                                                                       bias, T, D, E, dst, D / nsplit, xvec);
        }
        if (e != cudaSuccess) return cuda_status(e, "route_logits_sgemm_kernel attribute");
        if (nsplit > 1) {
            if ((e = cudaGetLastError()) != cudaSuccess) return cuda_status(e, "route_logits_sgemm_kernel");
            const int blocks = (T * 32 + 255) / 256;
            mark(tr, MOE_KERNEL_ROUTE_SELECT);
            route_reduce_select_kernel<<<blocks, 256, 0, s>>>(part, nsplit, bias, T, E, k, renorm, ids,
                                                             gates, L);
            return cuda_status(cudaGetLastError(), "route_reduce_select_kernel");
        }
    } else {
        dim3 grid((T + kTM - 1) / kTM, (E + kTN - 1) / kTN);
        if (x_dtype == MOE_BF16)
            route_logits_tiled_kernel<__nv_bfloat16><<<grid, 256, 0, s>>>(
                (const __nv_bfloat16 *)x, w_router, bias, T, D, E, L);
        else
            route_logits_tiled_kernel<float><<<grid, 256, 0, s>>>((const float *)x, w_router, bias,
                                                                  T, D, E, L);
    }
    moe_status st = cuda_status(cudaGetLastError(), "route_logits_tiled_kernel");
    if (st != MOE_OK) return st;
    int blocks = (T * 32 + 255) / 256;
    mark(tr, MOE_KERNEL_ROUTE_SELECT);
    route_select_kernel<<<blocks, 256, 0, s>>>(L, nullptr, T, E, k, renorm, ids, gates, nullptr);
    return cuda_status(cudaGetLastError(), "route_select_kernel");
}

}  // namespace moe

// ---------------------------------------------------------------------------
// Allocation-free routing entry point.
//
// Some callers cannot allocate device memory at the point where they route:
// code running inside a custom allocator's own callbacks, serving loops that
// forbid allocation after start-up so their memory footprint stays fixed,
// and embedders whose runtime owns every device allocation and offers no
// scratch buffer.  For them moe_route_noalloc runs the small-T router (the
// split-K logits + top-k kernel above) with its scratch in a fixed
// file-scope device array instead of a caller workspace.
//
// kNoAllocFloats bounds the scratch: ceil(D/32) * T * E fp32 partial sums
// (T <= 16) must fit in it; one more word is the completion ticket.  The
// array lives in every GPU that loads this library until the process exits.
// Every call on a device shares it, so calls that overlap on the GPU (other
// streams, other host threads) race and must be serialised by the caller.
// The ticket is cleared with a memset before each launch; the partial sums
// are fully written before they are read and need no clearing.
// ---------------------------------------------------------------------------
namespace moe {

constexpr size_t kNoAllocFloats = size_t(1) << 19;     // 2 MiB of partial sums

static __device__ __align__(256) float g_route_scratch[kNoAllocFloats + 64];

// Device address of g_route_scratch, looked up once per device (host code
// cannot use the array's name as a device pointer).
static void *noalloc_scratch_address(int dev, moe_status *st) {
    static std::mutex mu;
    static void *addr[128] = {nullptr};
    std::lock_guard<std::mutex> lock(mu);
    if (dev < 0 || dev >= 128) {
        set_error("moe_route_noalloc: device ordinal %d out of range", dev);
        *st = MOE_ERR_INVALID_ARG;
        return nullptr;
    }
    if (!addr[dev]) {
        void *p = nullptr;
        cudaError_t e = cudaGetSymbolAddress(&p, g_route_scratch);
        if (e != cudaSuccess) {
            *st = cuda_status(e, "moe_route_noalloc: cudaGetSymbolAddress");
            return nullptr;
        }
        addr[dev] = p;
    }
    *st = MOE_OK;
    return addr[dev];
}

}  // namespace moe

extern "C" moe_status moe_route_noalloc(const void *x, int32_t x_dtype, const float *w_router,
                                        const float *bias, int T, int D, int E, int k, int renorm,
                                        int32_t *ids, float *gates, float *logits,
                                        moe_stream stream) {
    using namespace moe;
    if (T < 0 || D <= 0 || E <= 0 || k <= 0 || D % QK || k > E || E > MOE_MAX_EXPERTS ||
        k > MOE_MAX_TOPK) {
        set_error("moe_route_noalloc: bad shape (T=%d D=%d E=%d k=%d)", T, D, E, k);
        return MOE_ERR_SHAPE;
    }
    if (x_dtype != MOE_F32 && x_dtype != MOE_BF16) {
        set_error("moe_route_noalloc: x dtype %d not F32/BF16", x_dtype);
        return MOE_ERR_INVALID_ARG;
    }
    if (renorm != 0 && renorm != 1) {
        set_error("moe_route_noalloc: renorm must be 0 or 1");
        return MOE_ERR_INVALID_ARG;
    }
    if (T == 0) return MOE_OK;
    if (!x || !w_router || !ids || !gates) {
        set_error("moe_route_noalloc: NULL x, w_router, ids or gates");
        return MOE_ERR_INVALID_ARG;
    }
    const int nsplit = (D + kSplitRows - 1) / kSplitRows;
    if (T > kSplitMaxT || (size_t)nsplit * T * E > kNoAllocFloats) {
        set_error("moe_route_noalloc: T=%d D=%d E=%d needs T <= %d and ceil(D/32)*T*E <= %zu "
                  "scratch floats", T, D, E, kSplitMaxT, kNoAllocFloats);
        return MOE_ERR_SHAPE;
    }
    int dev = 0;
    cudaError_t ce = cudaGetDevice(&dev);
    if (ce != cudaSuccess) return cuda_status(ce, "moe_route_noalloc: cudaGetDevice");
    moe_status st;
    float *scratch = (float *)noalloc_scratch_address(dev, &st);
    if (!scratch) return st;
    cudaStream_t s = (cudaStream_t)stream;
    unsigned *ticket = (unsigned *)(scratch + kNoAllocFloats);
    float *partial = scratch;
    ce = cudaMemsetAsync(ticket, 0, sizeof(unsigned), s);
    if (ce != cudaSuccess) return cuda_status(ce, "moe_route_noalloc: ticket clear");
    return launch_splitk(x, x_dtype, w_router, bias, T, D, E, k, renorm, nsplit, partial, ticket,
                         ids, gates, logits, s, "moe_route_noalloc: route_splitk_kernel");
}
