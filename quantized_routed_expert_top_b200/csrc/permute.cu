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

moe_status launch_permute(const int32_t *ids, int T, int k, int E, int32_t *counts,
                          int32_t *offsets, int32_t *perm, int32_t *inv,
                          cudaStream_t s, Tracer *tr) {
    const int N = T * k;
    size_t sm = (size_t)(kPermWarps * E) * sizeof(int32_t);
    cudaError_t e = cudaFuncSetAttribute(permute_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    if (e != cudaSuccess) return cuda_status(e, "permute_kernel smem attribute");
    mark(tr, MOE_KERNEL_PERMUTE);
    permute_kernel<<<1, kPermWarps * 32, sm, s>>>(ids, N, E, counts, offsets, perm, inv);
    return cuda_status(cudaGetLastError(), "permute_kernel");
}

}  // namespace moe
