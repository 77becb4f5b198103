// combine.cu -- gate-weighted combine back to token order.
//
// y[t, d] = sum_{j<k} g[t, j] * rows[inv[t*k + j], d]  (+ shared[t, d]),
// summed in fp32 in j order (deterministic), stored as F32, BF16 or F16.
// Four consecutive d per thread (16-byte loads when D % 4 == 0).
#include "moe_internal.cuh"

namespace moe {

template <typename YT> __device__ __forceinline__ void store_out(YT *p, float v);
template <> __device__ __forceinline__ void store_out<float>(float *p, float v) { *p = v; }
template <> __device__ __forceinline__ void store_out<__nv_bfloat16>(__nv_bfloat16 *p, float v) {
    *p = __float2bfloat16_rn(v);
}
template <> __device__ __forceinline__ void store_out<__half>(__half *p, float v) {
    *p = __float2half_rn(v);
}

template <typename YT>
__global__ void __launch_bounds__(256)
combine_kernel(const float *__restrict__ rows, const int32_t *__restrict__ inv,
               const float *__restrict__ gates, int T, int k, int D,
               const float *__restrict__ shared_rows, YT *__restrict__ y) {
    const int t = blockIdx.x;
    const int d0 = (blockIdx.y * blockDim.x + threadIdx.x) * 4;
    if (d0 >= D) return;
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    for (int j = 0; j < k; j++) {
        const float g = __ldg(gates + (size_t)t * k + j);
        const float *r = rows + (size_t)__ldg(inv + (size_t)t * k + j) * D + d0;
#pragma unroll
        for (int q = 0; q < 4; q++)
            if (d0 + q < D) acc[q] = fmaf(g, __ldg(r + q), acc[q]);
    }
#pragma unroll
    for (int q = 0; q < 4; q++) {
        if (d0 + q >= D) break;
        float v = acc[q];
        if (shared_rows) v += __ldg(shared_rows + (size_t)t * D + d0 + q);
        store_out<YT>(y + (size_t)t * D + d0 + q, v);
    }
}

moe_status launch_combine(const float *rows, const int32_t *inv, const float *gates, int T,
                          int k, int D, const float *shared_rows, void *y, int y_dtype,
                          cudaStream_t s, Tracer *tr) {
    dim3 grid(T, (D + 1023) / 1024);
    if (y_dtype == MOE_F32 || y_dtype == MOE_BF16 || y_dtype == MOE_F16) mark(tr, MOE_KERNEL_COMBINE);
    switch (y_dtype) {
    case MOE_F32:
        combine_kernel<float><<<grid, 256, 0, s>>>(rows, inv, gates, T, k, D, shared_rows,
                                                   (float *)y);
        break;
    case MOE_BF16:
        combine_kernel<__nv_bfloat16><<<grid, 256, 0, s>>>(rows, inv, gates, T, k, D, shared_rows,
                                                           (__nv_bfloat16 *)y);
        break;
    case MOE_F16:
        combine_kernel<__half><<<grid, 256, 0, s>>>(rows, inv, gates, T, k, D, shared_rows,
                                                    (__half *)y);
        break;
    default:
        set_error("moe_combine: unsupported output dtype %d", y_dtype);
        return MOE_ERR_INVALID_ARG;
    }
    return cuda_status(cudaGetLastError(), "combine_kernel");
}

}  // namespace moe
