// moe_internal.cuh -- helpers shared by the kernels of libmoe (sm_100a).
//
// Block formats decoded here are the ggml Standard-family types named in the
// FreeToken fork README ("Quant types" table): Q8_0 = {fp16 d; int8 q[32]},
// value q*d; Q4_0 = {fp16 d; uint8 qs[16]}, value (q-8)*d with byte j holding
// element j (low nibble) and element j+16 (high nibble).
#pragma once

#include <cuda_runtime.h>
#include <cuda_fp16.h>
#include <cuda_bf16.h>
#include <stdint.h>
#include <stddef.h>

#include "../../include/moe.h"

namespace moe {

constexpr int QK = 32;
constexpr int kQ4Bytes = MOE_Q4_0_BLOCK_BYTES;
constexpr int kQ8Bytes = MOE_Q8_0_BLOCK_BYTES;

// ---------------------------------------------------------------- host side
void set_error(const char *fmt, ...);
moe_status cuda_status(cudaError_t e, const char *what);
int num_sms();

// A bump allocator over a caller-owned workspace (256-byte aligned pieces).
struct Carver {
    char *base;
    size_t cap, off;
    explicit Carver(void *b, size_t c) : base((char *)b), cap(c), off(0) {}
    template <class T> T *take(size_t n) {
        off = (off + 255) & ~size_t(255);
        T *p = base ? (T *)(base + off) : nullptr;
        off += n * sizeof(T);
        return p;
    }
    bool fits() const { return off <= cap; }
};

__host__ __device__ inline size_t round_up(size_t a, size_t b) { return (a + b - 1) / b * b; }

// Records the caller's events around each kernel of a call (moe_trace).
struct Tracer {
    moe_trace *t = nullptr;
    cudaStream_t s = nullptr;
    bool open = false;
    cudaError_t err = cudaSuccess;
    // inside stream capture a plain record only orders the graph; the
    // external flag makes it a record node that timestamps at replay
    cudaError_t record(cudaEvent_t ev) {
        cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
        cudaStreamIsCapturing(s, &cs);
        if (cs == cudaStreamCaptureStatusActive)
            return cudaEventRecordWithFlags(ev, s, cudaEventRecordExternal);
        return cudaEventRecord(ev, s);
    }
    // before launching a kernel of `kind`
    void mark(int kind) {
        if (!t || t->count >= t->capacity || t->count >= MOE_TRACE_MAX) return;
        cudaError_t e = record((cudaEvent_t)t->events[t->count]);
        if (e != cudaSuccess && err == cudaSuccess) err = e;
        t->kinds[t->count] = kind;
        t->count++;
        open = true;
    }
    // after the last kernel
    void end() {
        if (!t || !open || t->count >= t->capacity) return;
        cudaError_t e = record((cudaEvent_t)t->events[t->count]);
        if (e != cudaSuccess && err == cudaSuccess) err = e;
        t->kinds[t->count] = 0;
        t->count++;
        open = false;
    }
};
inline void mark(Tracer *tr, int kind) { if (tr) tr->mark(kind); }

// ------------------------------------------------------------- device side
__device__ __forceinline__ float bf16_bits_to_f32(uint16_t b) {
    return __uint_as_float(((uint32_t)b) << 16);
}
__device__ __forceinline__ float half_bits_to_f32(uint16_t h) {
    return __half2float(__ushort_as_half(h));
}

template <typename XT> __device__ __forceinline__ float load_act(const XT *p, size_t i);
template <> __device__ __forceinline__ float load_act<float>(const float *p, size_t i) {
    return __ldg(p + i);
}
template <> __device__ __forceinline__ float load_act<__nv_bfloat16>(const __nv_bfloat16 *p, size_t i) {
    return bf16_bits_to_f32(__ldg(reinterpret_cast<const unsigned short *>(p) + i));
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

__device__ __forceinline__ float silu(float z) { return z / (1.0f + expf(-z)); }
// the same with the hardware exponential and an approximate division (a few
// fp32 ulp): for results rounded to fp16 right after, where those ulps vanish;
// no slow path for huge or non-finite arguments
__device__ __forceinline__ float silu_fast(float z) { return __fdividef(z, 1.0f + __expf(-z)); }

// Decode one block (32 weights) from global memory into w[32] (fp32).
// The block start is 2-byte aligned (18- or 34-byte stride), so 16-bit loads.
template <int QT>
__device__ __forceinline__ void decode_block_global(const uint8_t *blk, float *w) {
    const uint16_t *p = reinterpret_cast<const uint16_t *>(blk);
    float d = half_bits_to_f32(__ldg(p));
    if constexpr (QT == MOE_Q8_0) {
#pragma unroll
        for (int i = 0; i < 16; i++) {
            uint16_t two = __ldg(p + 1 + i);
            w[2 * i] = (float)(int8_t)(two & 0xff) * d;
            w[2 * i + 1] = (float)(int8_t)(two >> 8) * d;
        }
    } else {
#pragma unroll
        for (int i = 0; i < 8; i++) {
            uint16_t two = __ldg(p + 1 + i);
            int b0 = two & 0xff, b1 = two >> 8;
            w[2 * i] = (float)((b0 & 0xf) - 8) * d;
            w[2 * i + 16] = (float)((b0 >> 4) - 8) * d;
            w[2 * i + 1] = (float)((b1 & 0xf) - 8) * d;
            w[2 * i + 17] = (float)((b1 >> 4) - 8) * d;
        }
    }
}

template <int QT> __host__ __device__ constexpr int block_bytes() {
    return QT == MOE_Q8_0 ? kQ8Bytes : kQ4Bytes;
}

// Slot of an expert in a pool (identity when no map).
__device__ __forceinline__ int slot_of(const int32_t *map, int e) {
    return map ? __ldg(map + e) : e;
}

// ------------------------------------------------------- kernel launchers
// route.cu
moe_status launch_route(const void *x, int x_dtype, const float *w_router,
                        const float *bias, int T, int D, int E, int k, int renorm,
                        int32_t *ids, float *gates, float *logits, void *ws,
                        size_t ws_bytes, cudaStream_t s, Tracer *tr = nullptr);
size_t route_ws_bytes(int T, int D, int E, int k);
// routing plus, where a fused kernel exists (small T), the permutation in
// the same launch; *permuted tells the caller whether it still has to permute
moe_status launch_route_permute(const void *x, int x_dtype, const float *w_router,
                                const float *bias, int T, int D, int E, int k, int renorm,
                                int32_t *ids, float *gates, float *logits, int32_t *counts,
                                int32_t *offsets, int32_t *perm, int32_t *inv, int *err,
                                void *ws, size_t ws_bytes, cudaStream_t s, Tracer *tr,
                                bool *permuted);
// permute.cu
moe_status launch_permute(const int32_t *ids, int T, int k, int E, int32_t *counts,
                          int32_t *offsets, int32_t *perm, int32_t *inv,
                          cudaStream_t s, Tracer *tr = nullptr);
// ffn_generic.cu -- portable SIMT path for every shape
moe_status launch_ffn_generic(const void *x, int x_dtype, int T, int D, int F, int E,
                              int k, const int32_t *perm, const int32_t *offsets,
                              const moe_pool &pool, const uint8_t *mask, float *H,
                              float *out_rows, int *err, cudaStream_t s, Tracer *tr = nullptr,
                              bool shared = false);
// ffn_decode.cu -- TMA-streamed grouped GEMV for small T (see file header)
bool decode_path_ok(int T, int D, int F, int sF);
size_t decode_hs_halves(int T, int k, int F, int sF);
size_t decode_rows_floats(int T, int k, int D);
// ffn_prefill.cu -- large T on the tensor cores: x -> fp16, gate/up grouped
// GEMM (H fp16), down grouped GEMM (Y fp32 rows, then the combine kernel)
bool prefill_path_ok(int T, int D, int F, int sF, int E);
size_t prefill_x16_halves(int T, int D);
size_t prefill_h_halves(int T, int k, int F, int sF);
size_t prefill_y_floats(int T, int k, int D, int sF);
// routed: run the routed experts the mask (if any) admits; shared != NULL:
// run the shared expert too (rows T*k .. T*k+T-1 of H and Y)
moe_status launch_ffn_prefill(const void *x, int x_dtype, int T, int D, int F, int E, int k,
                              const int32_t *perm, const int32_t *offsets, const moe_pool &pool,
                              const uint8_t *mask, bool routed, const moe_pool *shared, int sF,
                              __half *x16, __half *H, float *Y, int *err, cudaStream_t s,
                              Tracer *tr);
// gates != NULL: fused layer (gates folded into the rows; rows_out holds
// [T*k + T, D] gated rows); gates == NULL: rows mode (un-gated Y rows [T*k, D]
// in permuted order).  routed: run the routed experts the mask admits;
// shared != NULL: run the shared expert (rows T*k..); y != NULL: combine the
// rows into y afterwards (adding the shared rows when comb_shared).
moe_status launch_ffn_decode(const void *x, int x_dtype, int T, int D, int F, int E, int k,
                             const int32_t *perm, const int32_t *inv, const int32_t *offsets,
                             const float *gates, const moe_pool &pool, const uint8_t *mask,
                             bool routed, const moe_pool *shared, int sF, bool comb_shared,
                             __half *Hs, void *y, int y_dtype, float *rows_out, int *err,
                             cudaStream_t s, Tracer *tr);
// combine.cu
moe_status launch_combine(const float *rows, const int32_t *inv, const float *gates,
                          int T, int k, int D, const float *shared_rows, void *y,
                          int y_dtype, cudaStream_t s, Tracer *tr = nullptr);

}  // namespace moe
