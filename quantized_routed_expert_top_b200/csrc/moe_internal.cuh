// moe_internal.cuh -- helpers shared by the kernels of libmoe (sm_100a).
//
// Block formats decoded here are the ggml Standard-family types named in the
// FreeToken fork README ("Quant types" table; the layouts are ggml's
// published ones), 32 weights a block, fields little endian:
//   Q8_0 {fp16 d; int8 q[32]}                      value q*d
//   Q4_0 {fp16 d; uint8 qs[16]}                    value (q-8)*d
//   Q4_1 {fp16 d; fp16 m; uint8 qs[16]}            value q*d + m
//   Q5_0 {fp16 d; uint8 qh[4]; uint8 qs[16]}       value (q-16)*d
//   Q5_1 {fp16 d; fp16 m; uint8 qh[4]; uint8 qs[16]}  value q*d + m
// qs byte j: low four bits of element j (low nibble) and of element j+16
// (high nibble); bit i of the word qh: bit 4 of element i.
// K-quants (256 weights a block; the same table's K-quants row):
//   Q4_K {fp16 d; fp16 dmin; uint8 scales[12]; uint8 qs[128]}  value
//        d*sc_j*q - dmin*m_j for 32-weight sub-block j (6-bit sc_j, m_j
//        packed in scales[]); weight 64c+l: low nibble of qs[32c+l],
//        weight 64c+32+l: its high nibble
//   Q6_K {uint8 ql[128]; uint8 qh[64]; int8 scales[16]; fp16 d}  value
//        d*scales[i/16]*(q-32); weight 128h+32r+l: low four bits in nibble
//        r/2 of ql[64h+32(r%2)+l], high two in bits 2r, 2r+1 of qh[32h+l]
// Kernels address both as rows of 32-weight units: unit b of a row lies in
// block b / 8 (sub-block b % 8).
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

// Field layout of a block type (byte offsets inside the block).
__host__ __device__ constexpr int qt_bytes(int q) {
    return q == MOE_Q8_0 ? MOE_Q8_0_BLOCK_BYTES : q == MOE_Q4_0 ? MOE_Q4_0_BLOCK_BYTES
         : q == MOE_Q4_1 ? MOE_Q4_1_BLOCK_BYTES : q == MOE_Q5_0 ? MOE_Q5_0_BLOCK_BYTES
         : q == MOE_Q5_1 ? MOE_Q5_1_BLOCK_BYTES : q == MOE_Q4_K ? MOE_Q4_K_BLOCK_BYTES
         : q == MOE_Q6_K ? MOE_Q6_K_BLOCK_BYTES : 0;
}
__host__ __device__ constexpr bool qt_known(int q) { return qt_bytes(q) != 0; }
__host__ __device__ constexpr bool qt_is_k(int q) { return q == MOE_Q4_K || q == MOE_Q6_K; }
// weights per block
__host__ __device__ constexpr int qt_weights(int q) {
    return !qt_known(q) ? 0 : qt_is_k(q) ? MOE_QK_K : QK;
}
// bytes per 32 weights where that is a whole number (0 for Q6_K: 26.25)
__host__ __device__ constexpr int qt_unit_bytes(int q) {
    return q == MOE_Q6_K ? 0 : qt_is_k(q) ? qt_bytes(q) / 8 : qt_bytes(q);
}
// bytes of a row of ncols weights (ncols a multiple of the block)
__host__ __device__ constexpr size_t qt_row_bytes(int q, int ncols) {
    return (size_t)(ncols / qt_weights(q)) * (size_t)qt_bytes(q);
}
__host__ __device__ constexpr bool qt_has_min(int q) {
    return q == MOE_Q4_1 || q == MOE_Q5_1 || q == MOE_Q4_K;
}
__host__ __device__ constexpr bool qt_has_high(int q) { return q == MOE_Q5_0 || q == MOE_Q5_1; }
// offset of the high-bit word qh (5-bit types) and of the codes
__host__ __device__ constexpr int qt_qh_off(int q) { return qt_has_min(q) ? 4 : 2; }
__host__ __device__ constexpr int qt_qs_off(int q) {
    return 2 + (qt_has_min(q) ? 2 : 0) + (qt_has_high(q) ? 4 : 0);
}
// the code of value zero in the _0 types (0 for the signed Q8_0 and for the
// _1 types, whose values are q*d + m)
__host__ __device__ constexpr int qt_zero(int q) {
    return q == MOE_Q4_0 ? 8 : q == MOE_Q5_0 ? 16 : 0;
}

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

// Decode one block (32 weights) from global memory into w[32] (fp32):
// (q - zero) * d, or q * d + m for the _1 types, each in fp32 (one rounding
// of the product, one of the sum).  Every block size is even and every field
// offset even, so 16-bit loads.
template <int QT>
__device__ __forceinline__ void decode_block_global(const uint8_t *blk, float *w) {
    const uint16_t *p = reinterpret_cast<const uint16_t *>(blk);
    const float d = half_bits_to_f32(__ldg(p));
    if constexpr (QT == MOE_Q8_0) {
#pragma unroll
        for (int i = 0; i < 16; i++) {
            uint16_t two = __ldg(p + 1 + i);
            w[2 * i] = (float)(int8_t)(two & 0xff) * d;
            w[2 * i + 1] = (float)(int8_t)(two >> 8) * d;
        }
    } else {
        const float m = qt_has_min(QT) ? half_bits_to_f32(__ldg(p + 1)) : 0.f;
        uint32_t qh = 0;
        if constexpr (qt_has_high(QT))
            qh = (uint32_t)__ldg(p + qt_qh_off(QT) / 2) | ((uint32_t)__ldg(p + qt_qh_off(QT) / 2 + 1) << 16);
        const uint16_t *qs = p + qt_qs_off(QT) / 2;
        auto value = [&](int i, int nib) {
            const int q = nib | (int)(((qh >> i) & 1u) << 4);
            return qt_has_min(QT) ? fmaf((float)q, d, m) : (float)(q - qt_zero(QT)) * d;
        };
#pragma unroll
        for (int i = 0; i < 8; i++) {
            uint16_t two = __ldg(qs + i);
            int b0 = two & 0xff, b1 = two >> 8;
            w[2 * i] = value(2 * i, b0 & 0xf);
            w[2 * i + 16] = value(2 * i + 16, b0 >> 4);
            w[2 * i + 1] = value(2 * i + 1, b1 & 0xf);
            w[2 * i + 17] = value(2 * i + 17, b1 >> 4);
        }
    }
}

template <int QT> __host__ __device__ constexpr int block_bytes() { return qt_bytes(QT); }

// Q4_K: the 6-bit scale and min of sub-block j from the block's scales[12]
// (as bytes): j < 4 in the low six bits of bytes j and j+4; j >= 4 in the
// nibbles of byte j+4 (scale low, min high) with the top two bits of bytes
// j-4 (scale) and j (min).
__host__ __device__ __forceinline__ void q4k_scale_min(const uint8_t *sc, int j, int *s, int *m) {
    if (j < 4) {
        *s = sc[j] & 63;
        *m = sc[j + 4] & 63;
    } else {
        *s = (sc[j + 4] & 15) | ((sc[j - 4] >> 6) << 4);
        *m = (sc[j + 4] >> 4) | ((sc[j] >> 6) << 4);
    }
}

// Decode 32-weight unit b of a row (row: the row's first byte) into w[32],
// fp32.  For the 32-weight types the unit is block b; for the K-quants it is
// sub-block b % 8 of block b / 8 (Q6_K: its scales 2j and 2j+1).
template <int QT>
__device__ __forceinline__ void decode_unit_global(const uint8_t *row, int b, float *w) {
    if constexpr (!qt_is_k(QT)) {
        decode_block_global<QT>(row + (size_t)b * qt_bytes(QT), w);
    } else if constexpr (QT == MOE_Q4_K) {
        const uint8_t *blk = row + (size_t)(b >> 3) * qt_bytes(QT);
        const int j = b & 7;
        const uint16_t *p = reinterpret_cast<const uint16_t *>(blk);
        const float d = half_bits_to_f32(__ldg(p)), dmin = half_bits_to_f32(__ldg(p + 1));
        uint8_t sc[12];
#pragma unroll
        for (int i = 0; i < 6; i++) {
            const uint16_t two = __ldg(p + 2 + i);
            sc[2 * i] = (uint8_t)(two & 0xff);
            sc[2 * i + 1] = (uint8_t)(two >> 8);
        }
        int s, m;
        q4k_scale_min(sc, j, &s, &m);
        const float ds = d * (float)s, dm = dmin * (float)m;
        const uint16_t *qs = p + 8 + 16 * (j >> 1);            // bytes 16 + 32 (j / 2)
        const int sh = 4 * (j & 1);
#pragma unroll
        for (int i = 0; i < 16; i++) {
            const uint16_t two = __ldg(qs + i);
            w[2 * i] = fmaf(ds, (float)((two >> sh) & 15), -dm);
            w[2 * i + 1] = fmaf(ds, (float)((two >> (8 + sh)) & 15), -dm);
        }
    } else {
        const uint8_t *blk = row + (size_t)(b >> 3) * qt_bytes(QT);
        const int j = b & 7, h = j >> 2, r = j & 3;
        const uint16_t *ql = reinterpret_cast<const uint16_t *>(blk + 64 * h + 32 * (r & 1));
        const uint16_t *qh = reinterpret_cast<const uint16_t *>(blk + 128 + 32 * h);
        const float d = half_bits_to_f32(__ldg(reinterpret_cast<const uint16_t *>(blk + 208)));
        const uint16_t sc2 = __ldg(reinterpret_cast<const uint16_t *>(blk + 192 + 2 * j));
        const float s0 = d * (float)(int8_t)(sc2 & 0xff), s1 = d * (float)(int8_t)(sc2 >> 8);
        const int lsh = 4 * (r >> 1), hsh = 2 * r;
#pragma unroll
        for (int i = 0; i < 16; i++) {
            const uint16_t lo2 = __ldg(ql + i), hi2 = __ldg(qh + i);
#pragma unroll
            for (int e = 0; e < 2; e++) {
                const int l = 2 * i + e;
                const int q = ((lo2 >> (8 * e + lsh)) & 15) | (((hi2 >> (8 * e + hsh)) & 3) << 4);
                w[l] = (l < 16 ? s0 : s1) * (float)(q - 32);
            }
        }
    }
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
// scratch: NULL (one CTA) or permute_scratch_ints(E) ints of device memory,
// which lets large T*k run over many CTAs (the same result)
moe_status launch_permute(const int32_t *ids, int T, int k, int E, int32_t *counts,
                          int32_t *offsets, int32_t *perm, int32_t *inv,
                          cudaStream_t s, Tracer *tr = nullptr, int32_t *scratch = nullptr);
size_t permute_scratch_ints(int E);
// ffn_generic.cu -- portable SIMT path for every shape
moe_status launch_ffn_generic(const void *x, int x_dtype, int T, int D, int F, int E,
                              int k, const int32_t *perm, const int32_t *offsets,
                              const moe_pool &pool, const uint8_t *mask, float *H,
                              float *out_rows, int *err, cudaStream_t s, Tracer *tr = nullptr,
                              bool shared = false);
// ffn_decode.cu -- TMA-streamed grouped GEMV for small T (see file header)
// qt, sqt: block types of the routed and the shared experts (sqt ignored
// when sF == 0)
bool decode_path_ok(int T, int D, int F, int sF, int qt, int sqt);
size_t decode_hs_halves(int T, int k, int F, int sF);
size_t decode_rows_floats(int T, int k, int D);
// ffn_prefill.cu -- large T on the tensor cores: x -> fp16, gate/up grouped
// GEMM (H fp16), down grouped GEMM (Y fp32 rows, then the combine kernel)
// allow_f16: the caller can give fp16 copies of the pools (prefill_f16_halves),
// which lets any block type (Q6_K needs it) take the tensor-core path
bool prefill_path_ok(int T, int D, int F, int sF, int E, int qt, int sqt, bool allow_f16 = false);
bool prefill_needs_f16(int qt, int sqt, int sF);
size_t prefill_f16_halves(int n_slots, int D, int F, int sF);
size_t prefill_x16_halves(int T, int D);
size_t prefill_h_halves(int T, int k, int F, int sF);
size_t prefill_y_floats(int T, int k, int D, int sF);
// routed: run the routed experts the mask (if any) admits; shared != NULL:
// run the shared expert too (rows T*k .. T*k+T-1 of H and Y)
moe_status launch_ffn_prefill(const void *x, int x_dtype, int T, int D, int F, int E, int k,
                              const int32_t *perm, const int32_t *offsets, const moe_pool &pool,
                              const uint8_t *mask, bool routed, const moe_pool *shared, int sF,
                              __half *x16, __half *H, float *Y, int *err, cudaStream_t s,
                              Tracer *tr, __half *w16 = nullptr);
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
// The same with 8-bit activation blocks into every expert matmul (the W4A8 /
// W8A8 mode): decode shapes, Q4_0 / Q8_0 experts; hq, hs: the h codes and
// their (scale, code sum) pairs (decode_a8_hq_bytes, decode_a8_hs_bytes).
bool decode_a8_ok(int T, int D, int F, int sF, int qt, int sqt);
size_t decode_a8_hq_bytes(int T, int k, int F, int sF);
size_t decode_a8_hs_bytes(int T, int k, int F, int sF);
moe_status launch_ffn_decode_a8(const void *x, int x_dtype, int T, int D, int F, int E, int k,
                                const int32_t *perm, const int32_t *inv, const int32_t *offsets,
                                const float *gates, const moe_pool &pool, const uint8_t *mask,
                                bool routed, const moe_pool *shared, int sF, bool comb_shared,
                                int8_t *hq, float2 *hs, void *y, int y_dtype, float *rows_out,
                                int *err, cudaStream_t s, Tracer *tr);
// combine.cu
moe_status launch_combine(const float *rows, const int32_t *inv, const float *gates,
                          int T, int k, int D, const float *shared_rows, void *y,
                          int y_dtype, cudaStream_t s, Tracer *tr = nullptr);

}  // namespace moe
