// permute.cuh -- block-level stable grouping of the T*k (token, slot)
// entries by expert, shared by the stand-alone permutation kernel and the
// small-batch routing kernel (which permutes in the same launch).
//
// Entries n = t*k + j are grouped by expert with a STABLE order (expert,
// then t, then j): perm[pos] = n, inv[n] = pos, counts[e] and the exclusive
// prefix offsets[e] (offsets[E] = N).  No atomics decide an order:
//   1. warp w owns a contiguous chunk of the entries and counts its experts
//      into its own histogram row hist[w][e] (__match_any_sync groups equal
//      ids inside a 32-entry step; the group's leader adds the group size);
//   2. the counts are scanned over experts, and each expert's column of the
//      histogram becomes the start position of every warp's run;
//   3. each warp walks its chunk again in order; an entry's position is its
//      warp's cursor for that expert plus its rank among equal ids of lower
//      lanes in the step.
// Chunks are contiguous and walked in order, so the result is the stable
// sort.  Ids outside [0, E) are dropped.
#pragma once
#include "moe_internal.cuh"

namespace moe {

// All NW*32 threads of the block call this.  hist: shared int[NW * E];
// scratch: shared int[32 + NW * 32 + 1].
template <int NW>
__device__ void block_permute(const int32_t *ids, int N, int E, int32_t *hist, int32_t *scratch,
                              int32_t *counts, int32_t *offsets, int32_t *perm, int32_t *inv) {
    constexpr int NT = NW * 32;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    for (int i = tid; i < NW * E; i += NT) hist[i] = 0;
    __syncthreads();

    const int per = ((N + NW - 1) / NW + 31) & ~31;
    const int c0 = min(N, warp * per), c1 = min(N, c0 + per);
    const unsigned lt_mask = (1u << lane) - 1u;
    for (int base = c0; base < c1; base += 32) {
        const int n = base + lane;
        int e = (n < c1) ? ids[n] : -1;
        if (e >= E) e = -1;
        const unsigned grp = __match_any_sync(0xffffffffu, e);
        if (e >= 0 && (grp & lt_mask) == 0u) hist[warp * E + e] += __popc(grp);
        __syncwarp();
    }
    __syncthreads();

    // exclusive scan of the expert counts; thread tid owns the experts
    // [tid*ep, tid*ep + ep)
    const int ep = (E + NT - 1) / NT;
    int local = 0;
    for (int q = 0; q < ep; q++) {
        const int e = tid * ep + q;
        if (e < E)
            for (int w = 0; w < NW; w++) local += hist[w * E + e];
    }
    int incl = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
    }
    int *warp_tot = scratch;
    if (lane == 31) warp_tot[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        const int v = (lane < NW) ? warp_tot[lane] : 0;
        int vi = v;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int u = __shfl_up_sync(0xffffffffu, vi, o);
            if (lane >= o) vi += u;
        }
        if (lane < NW) warp_tot[lane] = vi - v;
    }
    __syncthreads();
    int run = warp_tot[warp] + incl - local;
    for (int q = 0; q < ep; q++) {
        const int e = tid * ep + q;
        if (e >= E) break;
        int cnt = 0;
        offsets[e] = run;
        for (int w = 0; w < NW; w++) {
            const int c = hist[w * E + e];
            hist[w * E + e] = run + cnt;
            cnt += c;
        }
        counts[e] = cnt;
        run += cnt;
        if (e == E - 1) offsets[E] = run;
    }
    __syncthreads();

    for (int base = c0; base < c1; base += 32) {
        const int n = base + lane;
        int e = (n < c1) ? ids[n] : -1;
        if (e >= E) e = -1;
        const unsigned grp = __match_any_sync(0xffffffffu, e);
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

}  // namespace moe
