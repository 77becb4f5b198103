// permute.cu -- deterministic token -> expert grouping (count, scan, scatter).
//
// The T*k flat entries n = t*k + j are grouped by expert with a STABLE order
// (expert, then t, then j): perm[pos] = n, inv[n] = pos, counts[e] and the
// exclusive prefix offsets[e].  One CTA of 32 warps does it without any
// atomics deciding an order:
//   1. warp w owns a contiguous chunk of the entries and counts its experts
//      into its own histogram row hist[w][e] (__match_any_sync groups equal
//      ids inside a 32-entry step, the group's leader adds the group size);
//   2. one thread per expert turns the column hist[.][e] into the start
//      position of each warp's run, after an exclusive scan of the counts;
//   3. each warp walks its chunk again in order; an entry's position is its
//      warp's cursor for that expert plus its rank among equal ids of lower
//      lanes in the step.
// Chunks are contiguous and processed in order, so the result is the stable
// sort.  Dynamic shared memory: 32 * E + 2 * (E + 1) ints (<= 136 KB).
#include "moe_internal.cuh"

namespace moe {

constexpr int kPermWarps = 32;

__global__ void __launch_bounds__(kPermWarps * 32)
permute_kernel(const int32_t *__restrict__ ids, int N, int E,
               int32_t *__restrict__ counts, int32_t *__restrict__ offsets,
               int32_t *__restrict__ perm, int32_t *__restrict__ inv) {
    extern __shared__ int32_t sm[];
    int32_t *hist = sm;                           // [kPermWarps][E]
    int32_t *s_off = sm + kPermWarps * E;         // [E + 1]
    __shared__ int32_t warp_tot[kPermWarps];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    for (int i = tid; i < kPermWarps * E; i += blockDim.x) hist[i] = 0;
    __syncthreads();

    // chunk of warp w: [c0, c1), a multiple of 32 long
    const int per = ((N + kPermWarps - 1) / kPermWarps + 31) & ~31;
    const int c0 = min(N, warp * per), c1 = min(N, c0 + per);
    const unsigned lt_mask = (1u << lane) - 1u;

    for (int base = c0; base < c1; base += 32) {
        int n = base + lane;
        int e = (n < c1) ? __ldg(ids + n) : -1;
        if (e >= E) e = -1;                       // out-of-range ids are dropped
        unsigned grp = __match_any_sync(0xffffffffu, e);
        if (e >= 0 && (grp & lt_mask) == 0u) hist[warp * E + e] += __popc(grp);
        __syncwarp();
    }
    __syncthreads();

    // counts and exclusive scan over experts (blockDim >= E when E <= 1024)
    int cnt = 0;
    if (tid < E)
        for (int w = 0; w < kPermWarps; w++) cnt += hist[w * E + tid];
    // block-wide exclusive scan of cnt
    int incl = cnt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        int v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
    }
    if (lane == 31) warp_tot[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        int v = warp_tot[lane];
        int vi = v;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            int u = __shfl_up_sync(0xffffffffu, vi, o);
            if (lane >= o) vi += u;
        }
        warp_tot[lane] = vi - v;                  // exclusive warp prefix
    }
    __syncthreads();
    const int excl = warp_tot[warp] + incl - cnt;
    if (tid < E) {
        s_off[tid] = excl;
        counts[tid] = cnt;
        offsets[tid] = excl;
        if (tid == E - 1) offsets[E] = excl + cnt;
        int run = excl;
        for (int w = 0; w < kPermWarps; w++) {
            int c = hist[w * E + tid];
            hist[w * E + tid] = run;
            run += c;
        }
    }
    __syncthreads();

    for (int base = c0; base < c1; base += 32) {
        int n = base + lane;
        int e = (n < c1) ? __ldg(ids + n) : -1;
        if (e >= E) e = -1;
        unsigned grp = __match_any_sync(0xffffffffu, e);
        int pos = -1;
        if (e >= 0) pos = hist[warp * E + e] + __popc(grp & lt_mask);
        __syncwarp();
        if (e >= 0) {
            perm[pos] = n;
            inv[n] = pos;
            if ((grp & lt_mask) == 0u) hist[warp * E + e] += __popc(grp);
        }
        __syncwarp();
    }
}

moe_status launch_permute(const int32_t *ids, int T, int k, int E, int32_t *counts,
                          int32_t *offsets, int32_t *perm, int32_t *inv,
                          cudaStream_t s, Tracer *tr) {
    const int N = T * k;
    size_t sm = (size_t)(kPermWarps * E + E + 1) * sizeof(int32_t);
    cudaError_t e = cudaFuncSetAttribute(permute_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    if (e != cudaSuccess) return cuda_status(e, "permute_kernel smem attribute");
    mark(tr, MOE_KERNEL_PERMUTE);
    permute_kernel<<<1, kPermWarps * 32, sm, s>>>(ids, N, E, counts, offsets, perm, inv);
    return cuda_status(cudaGetLastError(), "permute_kernel");
}

}  // namespace moe
