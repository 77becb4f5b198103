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
// sort.  The algorithm is block_permute (permute.cuh); this kernel runs it
// with 32 warps.  Dynamic shared memory: 32 * E ints (<= 128 KB).
#include "permute.cuh"

namespace moe {

constexpr int kPermWarps = 32;

__global__ void __launch_bounds__(kPermWarps * 32)
permute_kernel(const int32_t *__restrict__ ids, int N, int E,
               int32_t *__restrict__ counts, int32_t *__restrict__ offsets,
               int32_t *__restrict__ perm, int32_t *__restrict__ inv) {
    extern __shared__ int32_t sm[];
    __shared__ int32_t scratch[32 + kPermWarps * 32 + 1];
    block_permute<kPermWarps>(ids, N, E, sm, scratch, counts, offsets, perm, inv);
}

// ------------------------------------------------- many CTAs (large T*k)
// The same stable grouping over kPermCtas CTAs, each owning a contiguous
// chunk of the entries:
//   1. permute_count_kernel: CTA b counts its chunk's experts into
//      hist[b][e] (global scratch; shared-memory atomics: counts only);
//   2. permute_scatter_kernel: every CTA reads the whole histogram; expert
//      e's run starts at the exclusive scan of the totals, and CTA b's part
//      of it after the counts of CTAs b' < b; inside its chunk a CTA places
//      entries as block_permute does (warp chunks in order, ranks among
//      equal ids of lower lanes).  CTA 0 writes counts and offsets.
// Chunks and warps are walked in order, so the result is the same stable
// sort as the one-CTA kernel's.
constexpr int kPermCtas = 64;
constexpr int kScatWarps = 16;

size_t permute_scratch_ints(int E) { return (size_t)kPermCtas * E; }

__global__ void __launch_bounds__(256)
permute_count_kernel(const int32_t *__restrict__ ids, int N, int E, int chunk,
                     int32_t *__restrict__ hist) {
    extern __shared__ int32_t h[];
    for (int e = threadIdx.x; e < E; e += blockDim.x) h[e] = 0;
    __syncthreads();
    const int c0 = min(N, (int)blockIdx.x * chunk), c1 = min(N, c0 + chunk);
    for (int n = c0 + threadIdx.x; n < c1; n += blockDim.x) {
        const int e = __ldg(ids + n);
        if (e >= 0 && e < E) atomicAdd(&h[e], 1);
    }
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x) hist[(size_t)blockIdx.x * E + e] = h[e];
}

__global__ void __launch_bounds__(kScatWarps * 32)
permute_scatter_kernel(const int32_t *__restrict__ ids, int N, int E, int chunk,
                       const int32_t *__restrict__ hist, int32_t *__restrict__ counts,
                       int32_t *__restrict__ offsets, int32_t *__restrict__ perm,
                       int32_t *__restrict__ inv) {
    extern __shared__ int32_t wh[];                 // [kScatWarps][E] warp cursors
    __shared__ int32_t tot_scan[32];
    constexpr int NT = kScatWarps * 32;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int b = blockIdx.x;
    const int c0 = min(N, b * chunk), c1 = min(N, c0 + chunk);
    // this CTA's start of each expert's run: scan of the totals plus the
    // counts of the CTAs before it (thread tid owns experts [tid*ep, +ep))
    const int ep = (E + NT - 1) / NT;
    int tot[8], bef[8];                             // ep <= 8 (E <= 4096)
    int local = 0;
#pragma unroll
    for (int q = 0; q < 8; q++) {
        tot[q] = bef[q] = 0;
        const int e = tid * ep + q;
        if (q < ep && e < E) {
            for (int bb = 0; bb < gridDim.x; bb++) {
                const int c = __ldg(hist + (size_t)bb * E + e);
                tot[q] += c;
                if (bb < b) bef[q] += c;
            }
            local += tot[q];
        }
    }
    int incl = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
    }
    if (lane == 31) tot_scan[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        const int v = lane < kScatWarps ? tot_scan[lane] : 0;
        int vi = v;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int u = __shfl_up_sync(0xffffffffu, vi, o);
            if (lane >= o) vi += u;
        }
        if (lane < kScatWarps) tot_scan[lane] = vi - v;
    }
    __syncthreads();
    int run = tot_scan[warp] + incl - local;          // start of expert tid*ep's run
    int cta_start[8];
#pragma unroll
    for (int q = 0; q < 8; q++) {
        const int e = tid * ep + q;
        cta_start[q] = run + bef[q];
        if (q < ep && e < E) {
            if (b == 0) {
                counts[e] = tot[q];
                offsets[e] = run;
                if (e == E - 1) offsets[E] = run + tot[q];
            }
            run += tot[q];
        }
    }
    // warp chunks inside the CTA chunk, counted per warp
    for (int i = tid; i < kScatWarps * E; i += NT) wh[i] = 0;
    __syncthreads();
    const int per = ((c1 - c0 + kScatWarps - 1) / kScatWarps + 31) & ~31;
    const int w0 = min(c1, c0 + warp * per), w1 = min(c1, w0 + per);
    const unsigned lt_mask = (1u << lane) - 1u;
    for (int base = w0; base < w1; base += 32) {
        const int n = base + lane;
        int e = (n < w1) ? __ldg(ids + n) : -1;
        if (e >= E) e = -1;
        const unsigned grp = __match_any_sync(0xffffffffu, e);
        if (e >= 0 && (grp & lt_mask) == 0u) wh[warp * E + e] += __popc(grp);
        __syncwarp();
    }
    __syncthreads();
    // column e: warp w's cursor = the CTA's start + the counts of warps < w
#pragma unroll
    for (int q = 0; q < 8; q++) {
        const int e = tid * ep + q;
        if (q < ep && e < E) {
            int cur = cta_start[q];
            for (int w = 0; w < kScatWarps; w++) {
                const int c = wh[w * E + e];
                wh[w * E + e] = cur;
                cur += c;
            }
        }
    }
    __syncthreads();
    for (int base = w0; base < w1; base += 32) {
        const int n = base + lane;
        int e = (n < w1) ? __ldg(ids + n) : -1;
        if (e >= E) e = -1;
        const unsigned grp = __match_any_sync(0xffffffffu, e);
        int pos = -1;
        if (e >= 0) pos = wh[warp * E + e] + __popc(grp & lt_mask);
        __syncwarp();
        if (e >= 0) {
            perm[pos] = n;
            inv[n] = pos;
            if ((grp & lt_mask) == 0u) wh[warp * E + e] += __popc(grp);
        }
        __syncwarp();
    }
}

moe_status launch_permute(const int32_t *ids, int T, int k, int E, int32_t *counts,
                          int32_t *offsets, int32_t *perm, int32_t *inv,
                          cudaStream_t s, Tracer *tr, int32_t *scratch) {
    const int N = T * k;
    if (scratch && N >= 8192 && E <= 8 * kScatWarps * 32) {
        const int chunk = (N + kPermCtas - 1) / kPermCtas;
        const size_t sm1 = (size_t)E * sizeof(int32_t), sm2 = (size_t)kScatWarps * E * sizeof(int32_t);
        cudaError_t e = cudaFuncSetAttribute(permute_scatter_kernel,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm2);
        if (e != cudaSuccess) return cuda_status(e, "permute_scatter_kernel smem attribute");
        mark(tr, MOE_KERNEL_PERMUTE);
        permute_count_kernel<<<kPermCtas, 256, sm1, s>>>(ids, N, E, chunk, scratch);
        if ((e = cudaGetLastError()) != cudaSuccess) return cuda_status(e, "permute_count_kernel");
        permute_scatter_kernel<<<kPermCtas, kScatWarps * 32, sm2, s>>>(ids, N, E, chunk, scratch, counts,
                                                                      offsets, perm, inv);
        return cuda_status(cudaGetLastError(), "permute_scatter_kernel");
    }
    size_t sm = (size_t)(kPermWarps * E) * sizeof(int32_t);
    cudaError_t e = cudaFuncSetAttribute(permute_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    if (e != cudaSuccess) return cuda_status(e, "permute_kernel smem attribute");
    mark(tr, MOE_KERNEL_PERMUTE);
    permute_kernel<<<1, kPermWarps * 32, sm, s>>>(ids, N, E, counts, offsets, perm, inv);
    return cuda_status(cudaGetLastError(), "permute_kernel");
}

}  // namespace moe
