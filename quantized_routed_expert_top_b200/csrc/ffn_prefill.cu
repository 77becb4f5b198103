// ffn_prefill.cu -- the prefill expert FFN (large T) on the 5th-generation
// tensor cores (tcgen05, accumulators in tensor memory).
//
// Prefill is a grouped GEMM: every expert multiplies its segment of tokens
// (rows of the permuted order) by its weights.  Two launches:
//
//  * gate/up: H[p, f] = silu(x_t . Wg[f]) * (x_t . Wu[f]) for the rows p of
//    expert e (token t = perm[p] / k), tile = 128 rows x 128 columns of F of
//    both matrices (one MMA of N=256: the weight stage holds the 128 gate
//    rows, then the 128 up rows), K = D.
//  * down:    Y[p, d] = H[p] . Wd[d], tile = 128 rows x 256 columns of D,
//    K = F.  Y rows are fp32 in permuted order; the gate-weighted combine is
//    the separate deterministic combine kernel.
//
// The weights stay in their ggml blocks in HBM.  They cannot feed the tensor
// cores directly (a per-32 fp16 scale), so B-producer warps dequantise each
// K-slice (64 weights of 256 rows) into fp16, d*q rounded once, written in the
// 128-byte-swizzled K-major layout the MMA descriptors name.  Their input is
// a ring of raw windows (four blocks of every weight row, two K-slices, per
// tensor copy); each B warp works through its 32 rows on its own and
// releases a window when done, the last release letting the window be
// refilled.  A-producer warps copy the activation rows (gathered through the
// permutation from an fp16 copy of x, or the contiguous rows of H) into their
// own ring with asynchronous copies whose arrivals are themselves
// asynchronous.  One thread issues tcgen05.mma (M=128, K=16 steps) once both
// rings hold the stage and commits each stage back to both; two TMEM
// accumulators (2 x 256 columns) let the epilogue warps drain one tile while
// the next accumulates.
//
// Numerics: weights (q - z)*d, or q*d + m for the _1 types, rounded once to
// fp16 (relative error <= 2^-11 per weight),
// activations fp16 (a bf16 x in fp16's normal range converts exactly; an fp32
// x is rounded to fp16's 11 significant bits), fp32 accumulation; H is
// stored fp16.
//
// Experts: the tile list covers the experts that have tokens, that this
// call runs (the routed ones the mask admits, and the shared one when
// present) and whose slot lies in [0, n_slots); an expert with tokens whose
// slot does not is left out and recorded as kErrBadSlot, so no address is
// ever formed from it.
#include "moe_internal.cuh"
#include "sm100.cuh"

#include <cuda.h>
#include <algorithm>
#include <cstring>

namespace moe {

constexpr int kPM = 128;                 // tile rows = MMA M
constexpr int kPK = 64;                  // K per stage: one 128-byte row of fp16
constexpr int kPNg = 128;                // gate/up: F columns per tile (per matrix)
constexpr int kPNd = 256;                // down: D columns per tile
constexpr int kPSA = 3;                  // activation stages (16 KB)
constexpr int kPSB = 2;                  // dequantised weight stages (32 KB)
constexpr int kPR = 3;                   // raw weight windows in flight (36 KB, two K stages each)
constexpr int kPStageA = kPM * kPK * 2;  // 16 KB
constexpr int kPStageB = 256 * kPK * 2;  // 32 KB (256 weight rows)

constexpr int kPAW = 2, kPBW = 8, kPEW = 4;                  // A copiers, B dequantisers, epilogue
constexpr int kPMmaWarp = kPAW + kPBW;                       // warp 10
constexpr int kPThreads = (kPAW + kPBW + 1 + kPEW) * 32;     // 480
constexpr int kPARows = kPM / (kPAW * 32 / 8);               // rows per A thread (16)
constexpr int kPTmemCols = 512;                              // 2 accumulators x 256
// A raw window holds four blocks (K = 128, two MMA stages) of each of the
// 256 weight rows: the 16-byte-aligned bytes around them (pf_window_bytes).
// Four blocks of 18, 22 or 34 bytes start 0 or 8 bytes past a 16-byte
// boundary (every other window), four of 20 or 24 bytes always on one.
constexpr int kPRawRow = 144;
constexpr int kPRaw = 256 * kPRawRow;    // one raw window buffer (36 KB)
constexpr int kPfMaxExperts = 720;       // segs + tcum of E + 2 entries each fit with the rings
// A ring | B ring | raw ring | barriers + TMEM slot (256 B) | segs, tcum [2][E+2]
__host__ __device__ inline size_t pf_smem_bytes(int E) {
    return (size_t)kPSA * kPStageA + (size_t)kPSB * kPStageB + (size_t)kPR * kPRaw + 256 +
           2 * (size_t)(E + 2) * 4 + 1024;
}

enum : int { kPGateUp = 0, kPDown = 1 };

// K stages (of 64 weights) per raw window: two (four 32-weight blocks), or
// four for Q4_K (one 144-byte block: its scales sit at the block's head)
__host__ __device__ constexpr int pf_stages_per_window(int qt) { return qt == MOE_Q4_K ? 4 : 2; }
// row bytes a window covers
__host__ __device__ constexpr int pf_window_span(int qt) {
    return pf_stages_per_window(qt) * 2 * qt_unit_bytes(qt);
}
// bytes of a raw window row: 144 (Q8_0, Q4_K), 80 (Q4_0, Q4_1), 96 (Q5_0, Q5_1)
__host__ __device__ constexpr int pf_window_bytes(int qt) {
    return pf_window_span(qt) % 16 == 0 ? pf_window_span(qt) : (pf_window_span(qt) + 8 + 15) / 16 * 16;
}

// Tensor maps over the weight pools (8-byte elements, one row of blocks per
// tensor row), boxes of one raw window (the 16-byte-aligned 144 or 80 bytes
// holding four blocks) x 128 rows (gate, up) or 256 rows (down).
struct PfMaps {
    CUtensorMap w0, w1;           // gate/up: gate, up; down: down, -
    CUtensorMap s0, s1;           // the shared expert's
};

struct PfArgs {
    int T, D, F, E, k;
    int qt;                       // block type (ggml id) of the routed pool
    int shared, sqt;              // this call runs the shared expert (F columns, its type)
    int routed;                   // this call runs the routed experts the mask admits
    int n_slots;                  // slots of the routed pool
    const uint8_t *mask;          // [E] or NULL
    const int32_t *perm, *offsets;
    const uint8_t *gate, *up, *down;
    const int32_t *slot_map;
    const uint8_t *sh_gate, *sh_up, *sh_down;
    const __half *x16;            // [T, D]
    __half *H;                    // [T*k + T, F]
    float *Y;                     // [T*k + T, D]
    int *err;
};

// ----------------------------------------------------------- PTX wrappers
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// D[tmem] (+)= A[smem desc] * B[smem desc]^T, kind::f16, fp32 accumulate
__device__ __forceinline__ void tc_mma(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                       uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
        " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}"
        ::"r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}
// arrive (once) on an mbarrier when every tcgen05.mma issued so far by this
// thread has completed
__device__ __forceinline__ void tc_commit(uint64_t *bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
                 ::"r"(smem_u32(bar)) : "memory");
}
// 32 lanes x 32 columns of fp32 from TMEM: thread i gets lane (base + i)
__device__ __forceinline__ void tc_ld32(uint32_t taddr, uint32_t *r) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,"
        "%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
          "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
          "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
          "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
}
__device__ __forceinline__ void tc_wait_ld() {
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// Shared-memory matrix descriptor: K-major, 128-byte swizzle, 8-row groups
// 1024 bytes apart (start address and offsets in 16-byte units; version 1;
// layout type 2 = 128-byte swizzle).
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFF);
    d |= (uint64_t)1 << 16;                       // leading byte offset (unused with swizzle)
    d |= (uint64_t)(1024 >> 4) << 32;             // stride byte offset: 8 rows x 128 B
    d |= (uint64_t)1 << 46;                       // descriptor version
    d |= (uint64_t)2 << 61;                       // 128-byte swizzle
    return d;
}
// Instruction descriptor, kind::f16: fp32 accumulator, A and B fp16, both
// K-major, M = 128, N = n.
__host__ __device__ constexpr uint32_t f16_idesc(int n) {
    return (1u << 4) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(kPM >> 4) << 24);
}

// byte offset of 16-byte chunk j (0..7) of row r in a 128-byte-swizzled tile
__device__ __forceinline__ uint32_t sw128_off(int r, int j) {
    return (uint32_t)(r * 128 + ((j ^ (r & 7)) << 4));
}

// ------------------------------------------------------------- dequantise
// 64 consecutive weights (two blocks starting at an even block index) of one
// row into 8 chunks of 8 fp16, natural order.  w: the row's raw window as
// 32-bit words; the pair starts at word O.
template <int O>
__device__ __forceinline__ void dq_pair_q8(const uint32_t *w, uint4 *out) {
    const uint32_t *v = w + O;
    const uint32_t d0 = v[0] & 0xFFFFu, d1 = v[8] >> 16;
    const uint32_t dd0 = d0 | (d0 << 16), dd1 = d1 | (d1 << 16);
    const uint32_t OFF = 0x64806480u, HI = 0x64646464u;
    uint32_t h[32];
#pragma unroll
    for (int i = 0; i < 8; i++) {
        // block 0 codes start at byte 2 of the pair; block 1 codes at byte 36
        const uint32_t c0 = __funnelshift_r(v[i], v[i + 1], 16) ^ 0x80808080u;
        const uint32_t c1 = v[9 + i] ^ 0x80808080u;
        h[2 * i] = hmul2_u(hsub2_u(prmt(c0, HI, 0x5140), OFF), dd0);
        h[2 * i + 1] = hmul2_u(hsub2_u(prmt(c0, HI, 0x7362), OFF), dd0);
        h[16 + 2 * i] = hmul2_u(hsub2_u(prmt(c1, HI, 0x5140), OFF), dd1);
        h[16 + 2 * i + 1] = hmul2_u(hsub2_u(prmt(c1, HI, 0x7362), OFF), dd1);
    }
#pragma unroll
    for (int c = 0; c < 8; c++) out[c] = make_uint4(h[4 * c], h[4 * c + 1], h[4 * c + 2], h[4 * c + 3]);
}

// Q4_0 pair: 36 bytes; byte j of a block = element j | element j+16 << 4.
template <int O>
__device__ __forceinline__ void dq_pair_q4(const uint32_t *w, uint4 *out) {
    const uint32_t *v = w + O;
    const uint32_t d0 = v[0] & 0xFFFFu, d1 = v[4] >> 16;
    const uint32_t dd0 = d0 | (d0 << 16), dd1 = d1 | (d1 << 16);
    const uint32_t OFF = 0x64086408u, M = 0x000F000Fu, MAG = 0x64006400u;
    uint32_t lo[16], hi[16];    // per block: elements 0..15 (lo), 16..31 (hi) as half2
#pragma unroll
    for (int b = 0; b < 2; b++) {
        const uint32_t dd = b ? dd1 : dd0;
#pragma unroll
        for (int i = 0; i < 4; i++) {
            const uint32_t c = b ? v[5 + i] : __funnelshift_r(v[i], v[i + 1], 16);
            const uint32_t t0 = prmt(c, 0u, 0x4140), t1 = prmt(c, 0u, 0x4342);   // bytes 0,1 / 2,3
            lo[8 * b + 2 * i] = hmul2_u(hsub2_u(lop3_and_or(t0, M, MAG), OFF), dd);
            lo[8 * b + 2 * i + 1] = hmul2_u(hsub2_u(lop3_and_or(t1, M, MAG), OFF), dd);
            hi[8 * b + 2 * i] = hmul2_u(hsub2_u(lop3_and_or(t0 >> 4, M, MAG), OFF), dd);
            hi[8 * b + 2 * i + 1] = hmul2_u(hsub2_u(lop3_and_or(t1 >> 4, M, MAG), OFF), dd);
        }
    }
    // chunks: block b -> elements 32b + [0..7], [8..15] (low nibbles), [16..23], [24..31]
#pragma unroll
    for (int b = 0; b < 2; b++) {
        out[4 * b + 0] = make_uint4(lo[8 * b + 0], lo[8 * b + 1], lo[8 * b + 2], lo[8 * b + 3]);
        out[4 * b + 1] = make_uint4(lo[8 * b + 4], lo[8 * b + 5], lo[8 * b + 6], lo[8 * b + 7]);
        out[4 * b + 2] = make_uint4(hi[8 * b + 0], hi[8 * b + 1], hi[8 * b + 2], hi[8 * b + 3]);
        out[4 * b + 3] = make_uint4(hi[8 * b + 4], hi[8 * b + 5], hi[8 * b + 6], hi[8 * b + 7]);
    }
}

// 32-bit word / 16-bit field at an even byte offset of a run of words
__device__ __forceinline__ uint32_t word_at(const uint32_t *w, int byte) {
    return (byte & 3) ? __funnelshift_r(w[byte >> 2], w[(byte >> 2) + 1], 16) : w[byte >> 2];
}
__device__ __forceinline__ uint32_t half_at(const uint32_t *w, int byte) {
    return (w[byte >> 2] >> (8 * (byte & 3))) & 0xFFFFu;
}

// Q4_1, Q5_0, Q5_1 pair starting at byte P of w (natural order, 8 chunks as
// above): the low four bits from qs (element j low nibble, j+16 high), the
// fifth from bit i of qh, v = 1024 + q exact in fp16, then (v - 1040) * d
// (Q5_0) or (v - 1024) * d + m (the _1 types) with one rounding.
template <int QT, int P>
__device__ __forceinline__ void dq_pair_std(const uint32_t *w, uint4 *out) {
    constexpr int BS = qt_bytes(QT), QS = qt_qs_off(QT), QH = qt_qh_off(QT);
    const uint32_t M = 0x000F000Fu, MAG = 0x64006400u;
    const uint32_t OFF = 0x64006400u + 0x00010001u * (uint32_t)qt_zero(QT);
    uint32_t lo[16], hi[16];
#pragma unroll
    for (int b = 0; b < 2; b++) {
        const int B = P + b * BS;
        const uint32_t d = half_at(w, B), dd = d | (d << 16);
        uint32_t mm = 0, qh = 0;
        if constexpr (qt_has_min(QT)) {
            const uint32_t m = half_at(w, B + 2);
            mm = m | (m << 16);
        }
        if constexpr (qt_has_high(QT)) qh = word_at(w, B + QH);
#pragma unroll
        for (int i = 0; i < 4; i++) {
            const uint32_t c = word_at(w, B + QS + 4 * i);        // bytes 4i .. 4i+3
            // v: elements (4i, 4i+1), (4i+2, 4i+3), (16+4i, 17+4i), (18+4i, 19+4i)
            uint32_t v[4];
            if constexpr (qt_has_high(QT)) {
                // 5-bit codes as bytes (bit 4 of element j from bit j of qh),
                // then bytes into halves
                const uint32_t h = qh >> (4 * i);
                const uint32_t lo = lop3_and_or(c, 0x0F0F0F0Fu, spread4_bit4(h & 0xFu));
                const uint32_t hi = lop3_and_or(c >> 4, 0x0F0F0F0Fu, spread4_bit4((h >> 16) & 0xFu));
                const uint32_t HI = 0x64646464u;
                v[0] = prmt(lo, HI, 0x5140);
                v[1] = prmt(lo, HI, 0x7362);
                v[2] = prmt(hi, HI, 0x5140);
                v[3] = prmt(hi, HI, 0x7362);
            } else {
                const uint32_t t0 = prmt(c, 0u, 0x4140), t1 = prmt(c, 0u, 0x4342);
                v[0] = lop3_and_or(t0, M, MAG);
                v[1] = lop3_and_or(t1, M, MAG);
                v[2] = lop3_and_or(t0 >> 4, M, MAG);
                v[3] = lop3_and_or(t1 >> 4, M, MAG);
            }
#pragma unroll
            for (int q = 0; q < 4; q++)
                v[q] = qt_has_min(QT) ? hfma2_u(hsub2_u(v[q], OFF), dd, mm)
                                      : hmul2_u(hsub2_u(v[q], OFF), dd);
            lo[8 * b + 2 * i] = v[0];
            lo[8 * b + 2 * i + 1] = v[1];
            hi[8 * b + 2 * i] = v[2];
            hi[8 * b + 2 * i + 1] = v[3];
        }
    }
#pragma unroll
    for (int b = 0; b < 2; b++) {
        out[4 * b + 0] = make_uint4(lo[8 * b + 0], lo[8 * b + 1], lo[8 * b + 2], lo[8 * b + 3]);
        out[4 * b + 1] = make_uint4(lo[8 * b + 4], lo[8 * b + 5], lo[8 * b + 6], lo[8 * b + 7]);
        out[4 * b + 2] = make_uint4(hi[8 * b + 0], hi[8 * b + 1], hi[8 * b + 2], hi[8 * b + 3]);
        out[4 * b + 3] = make_uint4(hi[8 * b + 4], hi[8 * b + 5], hi[8 * b + 6], hi[8 * b + 7]);
    }
}

// The pair of a K stage of a Q4_1 / Q5_0 / Q5_1 row: it starts P bytes into
// the row's window (rp, 16-byte aligned; rows pf_window_bytes apart).  Loads
// the 16-byte vectors from P rounded down to 16 through 2 bytes past the
// pair (a misaligned last word reads them): at most 16 bytes past the
// window, which is the next row's landed window or, for the last row, the
// unused tail of the raw buffer (sized for 144-byte rows).
template <int QT, int P>
__device__ __forceinline__ void dq_stage_std(const uint8_t *rp, uint4 *out) {
    constexpr int B0 = P & ~15, NV = (P - B0 + 2 * qt_bytes(QT) + 2 + 15) / 16;
    static_assert(255 * pf_window_bytes(QT) + B0 + 16 * NV <= kPRaw,
                  "the last row's reads stay inside its raw buffer");
    uint32_t w[4 * NV];
#pragma unroll
    for (int q = 0; q < NV; q++) {
        const uint4 v = *reinterpret_cast<const uint4 *>(rp + B0 + 16 * q);
        w[4 * q] = v.x; w[4 * q + 1] = v.y; w[4 * q + 2] = v.z; w[4 * q + 3] = v.w;
    }
    dq_pair_std<QT, P - B0>(w, out);
}

// Q4_K: K stage P (0..3) of a 144-byte block (rp, 16-byte aligned) is its
// 32-byte chunk P: the low nibbles are sub-block 2P (weights 0..31 of the
// stage), the high nibbles sub-block 2P+1 (weights 32..63).  Each weight is
// D * q - M with D = d * sc_j and M = dmin * m_j rounded to fp16, then one
// fp16 multiply-add (three roundings in all).
template <int P>
__device__ __forceinline__ void dq_stage_q4k(const uint8_t *rp, uint4 *out) {
    const uint4 h = *reinterpret_cast<const uint4 *>(rp);          // d, dmin, scales[12]
    const uint4 q0 = *reinterpret_cast<const uint4 *>(rp + 16 + 32 * P);
    const uint4 q1 = *reinterpret_cast<const uint4 *>(rp + 32 + 32 * P);
    const float d = __half2float(__ushort_as_half((unsigned short)(h.x & 0xFFFFu)));
    const float dmin = __half2float(__ushort_as_half((unsigned short)(h.x >> 16)));
    uint8_t sb[12];
#pragma unroll
    for (int i = 0; i < 4; i++) {
        sb[i] = (uint8_t)(h.y >> (8 * i));
        sb[4 + i] = (uint8_t)(h.z >> (8 * i));
        sb[8 + i] = (uint8_t)(h.w >> (8 * i));
    }
    uint32_t Dh[2], Mh[2];
#pragma unroll
    for (int u = 0; u < 2; u++) {
        int sc, m;
        q4k_scale_min(sb, 2 * P + u, &sc, &m);
        const __half2 dd = __float2half2_rn(d * (float)sc), mm = __float2half2_rn(-dmin * (float)m);
        Dh[u] = *reinterpret_cast<const uint32_t *>(&dd);
        Mh[u] = *reinterpret_cast<const uint32_t *>(&mm);
    }
    const uint32_t qw[8] = {q0.x, q0.y, q0.z, q0.w, q1.x, q1.y, q1.z, q1.w};
    const uint32_t HI = 0x64646464u, MAG = 0x64006400u, M4 = 0x0F0F0F0Fu;
    uint32_t v[2][16];                       // [sub-block][pair of elements]
#pragma unroll
    for (int i = 0; i < 8; i++) {
#pragma unroll
        for (int u = 0; u < 2; u++) {
            const uint32_t n = (qw[i] >> (4 * u)) & M4;             // elements 4i .. 4i+3
            v[u][2 * i] = hfma2_u(hsub2_u(prmt(n, HI, 0x5140), MAG), Dh[u], Mh[u]);
            v[u][2 * i + 1] = hfma2_u(hsub2_u(prmt(n, HI, 0x7362), MAG), Dh[u], Mh[u]);
        }
    }
#pragma unroll
    for (int u = 0; u < 2; u++)
#pragma unroll
        for (int k = 0; k < 4; k++)
            out[4 * u + k] = make_uint4(v[u][4 * k], v[u][4 * k + 1], v[u][4 * k + 2], v[u][4 * k + 3]);
}

// ------------------------------------------------------------------ tiles
// Virtual experts 0..E-1 (segments of the permutation) and, with a shared
// expert, E (rows T*k .. T*k+T-1, token = row - T*k).  Tiles are listed
// expert-major, then by column tile, then by row tile, so the row tiles that
// share a weight tile run on neighbouring CTAs at about the same time.
struct PfTile {
    int v, seg0, rows, m, n;      // rows = the expert's row count
};

__device__ __forceinline__ PfTile pf_tile(const int *tcum, const int *segs, int nv, int nt, int tau) {
    int lo = 0, hi = nv - 1;      // last v with tcum[v] <= tau
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (tcum[mid] <= tau) lo = mid; else hi = mid - 1;
    }
    PfTile t;
    t.v = lo;
    t.seg0 = segs[lo];
    t.rows = segs[lo + 1] - segs[lo];
    const int r = tau - tcum[lo];
    const int mt = (t.rows + kPM - 1) / kPM;
    t.n = r / mt;
    t.m = r % mt;
    return t;
}

// BK, how the weights reach the B stages: kBkBasic, Q4_0 / Q8_0 dequantised
// from raw windows; kBkAll, any 32-weight type or Q4_K dequantised the same
// way (a separate instantiation keeps their code out of the two types'
// kernel); kBkF16, fp16 weights (a pool converted by pf_dequant_f16_kernel)
// copied straight into the swizzled stages by tensor copies, no
// dequantising warps.  ONE >= 0: every expert of the call has block type
// ONE, and the kernel carries only that type's dequantiser (11-13% faster
// GEMMs than the kernel with every type's code).
enum : int { kBkBasic = 0, kBkAll = 1, kBkF16 = 2 };

template <int MODE, int BK, int ONE = -1>
__global__ void __launch_bounds__(kPThreads, 1) pf_gemm_kernel(PfArgs a, const __grid_constant__ PfMaps maps) {
    constexpr bool ALL = BK == kBkAll;
    extern __shared__ __align__(1024) uint8_t smem_pf[];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    uint8_t *ringA = smem_pf + ((1024u - (smem_u32(smem_pf) & 1023u)) & 1023u);
    uint8_t *ringB = ringA + (size_t)kPSA * kPStageA;
    uint8_t *raw = ringB + (size_t)kPSB * kPStageB;           // raw weight windows
    uint64_t *fullA = (uint64_t *)(raw + (size_t)kPR * kPRaw);
    uint64_t *emptyA = fullA + kPSA;
    uint64_t *fullB = emptyA + kPSA;
    uint64_t *emptyB = fullB + kPSB;
    uint64_t *rfull = emptyB + kPSB;                          // raw window landed
    uint64_t *rempty = rfull + kPR;                           // raw window read by every B warp
    uint64_t *accf = rempty + kPR;                            // [2] accumulator ready
    uint64_t *acce = accf + 2;                                // [2] accumulator drained
    uint64_t *mma_done = acce + 2;                            // every MMA of the CTA completed
    uint32_t *tmem_slot = (uint32_t *)(mma_done + 1);
    int *segs = (int *)(tmem_slot + 4);                       // [nv + 1] segment starts
    int *tcum = segs + (a.E + 2);                             // [nv + 1] first tile of each expert

    const int Tk = a.T * a.k;
    const int nv = a.E + (a.shared ? 1 : 0);
    const int N = MODE == kPGateUp ? a.F : a.D;    // output columns
    const int K = MODE == kPGateUp ? a.D : a.F;    // reduction length
    const int BN = MODE == kPGateUp ? kPNg : kPNd;
    const int nt = N / BN, nk = K / kPK;

    if (tid == 0) {
        for (int s = 0; s < kPSA; s++) {
            mbar_init(&fullA[s], kPAW * 32);
            mbar_init(&emptyA[s], 1);
        }
        for (int s = 0; s < kPSB; s++) {
            mbar_init(&fullB[s], BK == kBkF16 ? 1 : kPBW * 32);
            mbar_init(&emptyB[s], 1);
        }
        for (int r = 0; r < kPR; r++) {
            mbar_init(&rfull[r], 1);
            mbar_init(&rempty[r], kPBW);
        }
        for (int b = 0; b < 2; b++) {
            mbar_init(&accf[b], 1);
            mbar_init(&acce[b], kPEW * 32);
        }
        mbar_init(mma_done, 1);
        fence_mbar_init();
    }
    if (warp == kPMmaWarp) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                     ::"r"(smem_u32(tmem_slot)), "r"(kPTmemCols) : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    // the permutation and segments come from the routing kernels
    pdl_wait();
    for (int v = tid; v <= nv; v += blockDim.x)
        segs[v] = v <= a.E ? __ldg(a.offsets + v) : Tk + a.T;
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    if (warp == 0) {
        int base = 0;
        for (int v0 = 0; v0 < nv; v0 += 32) {
            const int v = v0 + lane;
            int ntiles = 0;
            if (v < nv) {
                int cnt = segs[v + 1] - segs[v];
                if (v < a.E && cnt > 0) {
                    if (!a.routed || (a.mask && !__ldg(a.mask + v))) {
                        cnt = 0;
                    } else {
                        const int sl = a.slot_map ? __ldg(a.slot_map + v) : v;
                        if (sl < 0 || sl >= a.n_slots) {
                            atomicCAS(a.err, 0, kErrBadSlot);
                            cnt = 0;
                        }
                    }
                }
                ntiles = (cnt + kPM - 1) / kPM * nt;
            }
            int incl = ntiles;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int t = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += t;
            }
            if (v < nv) tcum[v] = base + incl - ntiles;
            base += __shfl_sync(0xffffffffu, incl, 31);
        }
        if (lane == 0) tcum[nv] = base;
    }
    __syncthreads();
    const int n_tiles = tcum[nv];
    int n_loc = 0;                                   // this CTA's tiles
    for (int tau = blockIdx.x; tau < n_tiles; tau += gridDim.x) n_loc++;
    const int n_st = n_loc * nk;                     // K stages in all

    if (warp < kPAW) {
        // ------------------------------------------ A producers
        const int j = tid & 7, r0 = tid >> 3;
        int g = 0;
        bool ok = true;
        for (int tau = blockIdx.x; tau < n_tiles && ok; tau += gridDim.x) {
            const PfTile t = pf_tile(tcum, segs, nv, nt, tau);
            const __half *src[kPARows];
#pragma unroll
            for (int i = 0; i < kPARows; i++) {
                const int row = t.m * kPM + r0 + 8 * i;
                src[i] = nullptr;
                if (row < t.rows) {
                    const int p = t.seg0 + row;
                    if (MODE == kPGateUp) {
                        const int tok = p < Tk ? __ldg(a.perm + p) / a.k : p - Tk;
                        src[i] = a.x16 + (size_t)tok * a.D;
                    } else {
                        src[i] = a.H + (size_t)p * a.F;
                    }
                }
            }
            for (int ks = 0; ks < nk; ks++, g++) {
                const int s = g % kPSA;
                if (!mbar_wait(&emptyA[s], ((g / kPSA) & 1) ^ 1, a.err, kErrTimeoutEmpty)) { ok = false; break; }
                const uint32_t dst = smem_u32(ringA + (size_t)s * kPStageA);
#pragma unroll
                for (int i = 0; i < kPARows; i++) {
                    const __half *gp = src[i] ? src[i] + ks * kPK + 8 * j : a.x16;
                    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;"
                                 ::"r"(dst + sw128_off(r0 + 8 * i, j)), "l"(gp), "r"(src[i] ? 16 : 0) : "memory");
                }
                asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(&fullA[s]))
                             : "memory");
            }
        }
        asm volatile("cp.async.wait_all;" ::: "memory");
    } else if (warp < kPAW + kPBW) {
        if constexpr (BK == kBkF16) {
            // ------------------------------------ B producer, fp16 weights
            // one thread copies each K stage of the tile's 256 weight rows
            // (64 fp16 = 128 bytes a row) into the stage with the 128-byte
            // swizzle the MMA descriptors name
            if (warp == kPAW && lane == 0) {
                int g = 0;
                bool ok = true;
                for (int tau = blockIdx.x; tau < n_tiles && ok; tau += gridDim.x) {
                    const PfTile t = pf_tile(tcum, segs, nv, nt, tau);
                    const bool sh = t.v == a.E;
                    const int slot = sh ? 0 : (a.slot_map ? __ldg(a.slot_map + t.v) : t.v);
                    for (int ks = 0; ks < nk; ks++, g++) {
                        const int s = g % kPSB;
                        if (!mbar_wait(&emptyB[s], ((g / kPSB) & 1) ^ 1, a.err, kErrTimeoutEmpty)) { ok = false; break; }
                        uint8_t *dst = ringB + (size_t)s * kPStageB;
                        mbar_arrive_expect_tx(&fullB[s], (uint32_t)kPStageB);
                        if (MODE == kPGateUp) {
                            const int y = slot * a.F + t.n * kPNg;
                            tma_load_2d(dst, sh ? &maps.s0 : &maps.w0, ks * kPK, y, &fullB[s]);
                            tma_load_2d(dst + kPStageB / 2, sh ? &maps.s1 : &maps.w1, ks * kPK, y, &fullB[s]);
                        } else {
                            tma_load_2d(dst, sh ? &maps.s0 : &maps.w0, ks * kPK, slot * a.D + t.n * kPNd,
                                        &fullB[s]);
                        }
                    }
                }
                // copies still in flight must land before the CTA exits
                for (int q = g > kPSB ? g - kPSB : 0; q < g; q++)
                    mbar_wait(&fullB[q % kPSB], (uint32_t)((q / kPSB) & 1), a.err, kErrTimeoutDrain);
            }
        } else if constexpr (!ALL) {
            // ------------------------------------ B producers, Q4_0 / Q8_0
            // (the other types' code below ran these two types 5-8% slower)
            // Raw windows (the 16-byte-aligned bytes holding four blocks = two
            // K stages, for all 256 weight rows of the tile) arrive by tensor
            // copies kPR - 1 windows ahead.  Each warp dequantises its 32 rows of the
            // window into the swizzled fp16 stage on its own; lane 0 of the
            // first warp refills a raw buffer once all warps have read it.
            const int bw = warp - kPAW, bt = tid - kPAW * 32;
            const bool issuer = bw == 0 && lane == 0;
            const int nw = nk / 2;                           // windows per tile
            const int n_win = n_loc * nw;
            int gi = 0, ti = -1, wi = nw;                    // window issue cursor
            PfTile tI{};
            auto issue = [&]() -> bool {
                if (gi >= n_win) return true;
                if (gi >= kPR) {                             // the buffer's previous window is read
                    const int q = gi - kPR;
                    if (!mbar_wait(&rempty[q % kPR], (uint32_t)((q / kPR) & 1), a.err, kErrTimeoutEmpty)) return false;
                }
                if (wi == nw) {
                    ti++;
                    wi = 0;
                    tI = pf_tile(tcum, segs, nv, nt, blockIdx.x + ti * gridDim.x);
                }
                const bool sh = tI.v == a.E;
                const bool q8 = (ONE >= 0 ? ONE : sh ? a.sqt : a.qt) == MOE_Q8_0;
                const int bs = q8 ? kQ8Bytes : kQ4Bytes;
                const int wb = q8 ? 144 : 80;                        // window bytes
                const int x = (int)(((size_t)wi * 4 * bs & ~(size_t)15) / 8);
                const int slot = sh ? 0 : (a.slot_map ? __ldg(a.slot_map + tI.v) : tI.v);
                const int r = gi % kPR;
                uint8_t *dst = raw + (size_t)r * kPRaw;
                mbar_arrive_expect_tx(&rfull[r], (uint32_t)(256 * wb));
                if (MODE == kPGateUp) {
                    const int y = slot * a.F + tI.n * kPNg;
                    tma_load_2d(dst, sh ? &maps.s0 : &maps.w0, x, y, &rfull[r]);
                    tma_load_2d(dst + 128 * wb, sh ? &maps.s1 : &maps.w1, x, y, &rfull[r]);
                } else {
                    tma_load_2d(dst, sh ? &maps.s0 : &maps.w0, x, slot * a.D + tI.n * kPNd, &rfull[r]);
                }
                gi++;
                wi++;
                return true;
            };
            bool ok = true;
            if (issuer)
                for (int q = 0; q < kPR - 1 && ok; q++) ok = issue();
            ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
            int g = 0, gw = 0;                               // stage, window counters
            for (int tau = blockIdx.x; tau < n_tiles && ok; tau += gridDim.x) {
                const PfTile t = pf_tile(tcum, segs, nv, nt, tau);
                const bool q8 = (ONE >= 0 ? ONE : (t.v == a.E) ? a.sqt : a.qt) == MOE_Q8_0;
                const int wb = q8 ? 144 : 80;
                for (int ks = 0; ks < nk && ok; ks++, g++) {
                    const int half = ks & 1;                         // which block pair of the window
                    if (half == 0) {
                        bool iok = true;
                        if (issuer) iok = issue();                   // window gw + kPR - 1
                        ok = __shfl_sync(0xffffffffu, iok ? 1 : 0, 0) != 0;
                        if (!ok) break;
                    }
                    const int r = gw % kPR;
                    if (half == 0 &&
                        !mbar_wait_warp(&rfull[r], (uint32_t)((gw / kPR) & 1), a.err, kErrTimeoutFull)) { ok = false; break; }
                    uint4 c[8];
                    // the pair starts 8 * (group % 2) + (2 * bs) * half bytes into the window
                    const int odd = (ks >> 1) & 1;
                    const uint8_t *rp = raw + (size_t)r * kPRaw + bt * wb;
                    if (q8) {
                        // words 16 * half .. +19 hold the pair at word 2*odd + half
                        uint32_t w[20];
    #pragma unroll
                        for (int q = 0; q < 5; q++) {
                            const uint4 v = *reinterpret_cast<const uint4 *>(rp + 64 * half + 16 * q);
                            w[4 * q] = v.x; w[4 * q + 1] = v.y; w[4 * q + 2] = v.z; w[4 * q + 3] = v.w;
                        }
                        switch (2 * odd + half) {
                        case 0: dq_pair_q8<0>(w, c); break;
                        case 1: dq_pair_q8<1>(w, c); break;
                        case 2: dq_pair_q8<2>(w, c); break;
                        default: dq_pair_q8<3>(w, c); break;
                        }
                    } else {
                        // words 8 * half .. +11 hold the pair at word 2*odd + half
                        uint32_t w[12];
    #pragma unroll
                        for (int q = 0; q < 3; q++) {
                            const uint4 v = *reinterpret_cast<const uint4 *>(rp + 32 * half + 16 * q);
                            w[4 * q] = v.x; w[4 * q + 1] = v.y; w[4 * q + 2] = v.z; w[4 * q + 3] = v.w;
                        }
                        switch (2 * odd + half) {
                        case 0: dq_pair_q4<0>(w, c); break;
                        case 1: dq_pair_q4<1>(w, c); break;
                        case 2: dq_pair_q4<2>(w, c); break;
                        default: dq_pair_q4<3>(w, c); break;
                        }
                    }
                    if (half == 1) {
                        __syncwarp();
                        if (lane == 0) mbar_arrive(&rempty[r]);      // this warp is done with the window
                        gw++;
                    }
                    const int s = g % kPSB;
                    if (!mbar_wait_warp(&emptyB[s], ((g / kPSB) & 1) ^ 1, a.err, kErrTimeoutEmpty)) { ok = false; break; }
                    uint8_t *dst = ringB + (size_t)s * kPStageB;
    #pragma unroll
                    for (int jj = 0; jj < 8; jj++) *reinterpret_cast<uint4 *>(dst + sw128_off(bt, jj)) = c[jj];
                    fence_proxy_async_smem();
                    mbar_arrive(&fullB[s]);
                }
            }
            // windows still in flight must land before the CTA exits
            if (issuer)
                for (; gw < gi; gw++)
                    mbar_wait(&rfull[gw % kPR], (uint32_t)((gw / kPR) & 1), a.err, kErrTimeoutDrain);
        } else {
            // ------------------------------------------------- B producers
            // Raw windows (the 16-byte-aligned bytes holding four blocks = two
            // K stages, or one Q4_K block = four, for all 256 weight rows of the
            // tile) arrive by tensor copies kPR - 1 windows ahead.  Each warp
            // dequantises its 32 rows of the window into the swizzled fp16 stage
            // on its own; lane 0 of the first warp refills a raw buffer once all
            // warps have read it.
            const int bw = warp - kPAW, bt = tid - kPAW * 32;
            const bool issuer = bw == 0 && lane == 0;
            int gi = 0, ti = -1, wi = 0, nwI = 0;            // window issue cursor; windows of tile ti
            PfTile tI{};
            auto issue = [&]() -> bool {
                if (wi == nwI) {                             // next tile of this CTA, if any
                    if (ti + 1 >= n_loc) return true;
                    ti++;
                    wi = 0;
                    tI = pf_tile(tcum, segs, nv, nt, blockIdx.x + ti * gridDim.x);
                    nwI = nk / pf_stages_per_window(ONE >= 0 ? ONE : tI.v == a.E ? a.sqt : a.qt);
                }
                if (gi >= kPR) {                             // the buffer's previous window is read
                    const int q = gi - kPR;
                    if (!mbar_wait(&rempty[q % kPR], (uint32_t)((q / kPR) & 1), a.err, kErrTimeoutEmpty)) return false;
                }
                const bool sh = tI.v == a.E;
                const int qt = ONE >= 0 ? ONE : sh ? a.sqt : a.qt;
                const int wb = pf_window_bytes(qt);
                const int x = (int)(((size_t)wi * pf_window_span(qt) & ~(size_t)15) / 8);
                const int slot = sh ? 0 : (a.slot_map ? __ldg(a.slot_map + tI.v) : tI.v);
                const int r = gi % kPR;
                uint8_t *dst = raw + (size_t)r * kPRaw;
                mbar_arrive_expect_tx(&rfull[r], (uint32_t)(256 * wb));
                if (MODE == kPGateUp) {
                    const int y = slot * a.F + tI.n * kPNg;
                    tma_load_2d(dst, sh ? &maps.s0 : &maps.w0, x, y, &rfull[r]);
                    tma_load_2d(dst + 128 * wb, sh ? &maps.s1 : &maps.w1, x, y, &rfull[r]);
                } else {
                    tma_load_2d(dst, sh ? &maps.s0 : &maps.w0, x, slot * a.D + tI.n * kPNd, &rfull[r]);
                }
                gi++;
                wi++;
                return true;
            };
            bool ok = true;
            if (issuer)
                for (int q = 0; q < kPR - 1 && ok; q++) ok = issue();
            ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
            int g = 0, gw = 0;                               // stage, window counters
            for (int tau = blockIdx.x; tau < n_tiles && ok; tau += gridDim.x) {
                const PfTile t = pf_tile(tcum, segs, nv, nt, tau);
                const int qt = ONE >= 0 ? ONE : (t.v == a.E) ? a.sqt : a.qt;
                const int wb = pf_window_bytes(qt);
                const int spw = pf_stages_per_window(qt);
                for (int ks = 0; ks < nk && ok; ks++, g++) {
                    const int pos = ks & (spw - 1);                  // stage within the window
                    const int half = ks & 1;                         // which block pair of the window
                    if (pos == 0) {
                        bool iok = true;
                        if (issuer) iok = issue();                   // window gw + kPR - 1
                        ok = __shfl_sync(0xffffffffu, iok ? 1 : 0, 0) != 0;
                        if (!ok) break;
                    }
                    const int r = gw % kPR;
                    if (pos == 0 &&
                        !mbar_wait_warp(&rfull[r], (uint32_t)((gw / kPR) & 1), a.err, kErrTimeoutFull)) { ok = false; break; }
                    uint4 c[8];
                    // the pair starts skew(window) + (2 * bs) * half bytes into the
                    // window; the skew is 8 for odd windows of 18-, 22- and 34-byte
                    // blocks, else 0
                    const int odd = (ks >> 1) & 1;
                    const uint8_t *rp = raw + (size_t)r * kPRaw + bt * wb;
                    if (qt == MOE_Q4_K) {
                        switch (pos) {
                        case 0: dq_stage_q4k<0>(rp, c); break;
                        case 1: dq_stage_q4k<1>(rp, c); break;
                        case 2: dq_stage_q4k<2>(rp, c); break;
                        default: dq_stage_q4k<3>(rp, c); break;
                        }
                    } else if (qt == MOE_Q4_1) {
                        if (half == 0) dq_stage_std<MOE_Q4_1, 0>(rp, c); else dq_stage_std<MOE_Q4_1, 40>(rp, c);
                    } else if (qt == MOE_Q5_1) {
                        if (half == 0) dq_stage_std<MOE_Q5_1, 0>(rp, c); else dq_stage_std<MOE_Q5_1, 48>(rp, c);
                    } else if (qt == MOE_Q5_0) {
                        switch (2 * odd + half) {
                        case 0: dq_stage_std<MOE_Q5_0, 0>(rp, c); break;
                        case 1: dq_stage_std<MOE_Q5_0, 44>(rp, c); break;
                        case 2: dq_stage_std<MOE_Q5_0, 8>(rp, c); break;
                        default: dq_stage_std<MOE_Q5_0, 52>(rp, c); break;
                        }
                    } else if (qt == MOE_Q8_0) {
                        // words 16 * half .. +19 hold the pair at word 2*odd + half
                        uint32_t w[20];
    #pragma unroll
                        for (int q = 0; q < 5; q++) {
                            const uint4 v = *reinterpret_cast<const uint4 *>(rp + 64 * half + 16 * q);
                            w[4 * q] = v.x; w[4 * q + 1] = v.y; w[4 * q + 2] = v.z; w[4 * q + 3] = v.w;
                        }
                        switch (2 * odd + half) {
                        case 0: dq_pair_q8<0>(w, c); break;
                        case 1: dq_pair_q8<1>(w, c); break;
                        case 2: dq_pair_q8<2>(w, c); break;
                        default: dq_pair_q8<3>(w, c); break;
                        }
                    } else {
                        // words 8 * half .. +11 hold the pair at word 2*odd + half
                        uint32_t w[12];
    #pragma unroll
                        for (int q = 0; q < 3; q++) {
                            const uint4 v = *reinterpret_cast<const uint4 *>(rp + 32 * half + 16 * q);
                            w[4 * q] = v.x; w[4 * q + 1] = v.y; w[4 * q + 2] = v.z; w[4 * q + 3] = v.w;
                        }
                        switch (2 * odd + half) {
                        case 0: dq_pair_q4<0>(w, c); break;
                        case 1: dq_pair_q4<1>(w, c); break;
                        case 2: dq_pair_q4<2>(w, c); break;
                        default: dq_pair_q4<3>(w, c); break;
                        }
                    }
                    if (pos == spw - 1) {
                        __syncwarp();
                        if (lane == 0) mbar_arrive(&rempty[r]);      // this warp is done with the window
                        gw++;
                    }
                    const int s = g % kPSB;
                    if (!mbar_wait_warp(&emptyB[s], ((g / kPSB) & 1) ^ 1, a.err, kErrTimeoutEmpty)) { ok = false; break; }
                    uint8_t *dst = ringB + (size_t)s * kPStageB;
    #pragma unroll
                    for (int jj = 0; jj < 8; jj++) *reinterpret_cast<uint4 *>(dst + sw128_off(bt, jj)) = c[jj];
                    fence_proxy_async_smem();
                    mbar_arrive(&fullB[s]);
                }
            }
            // windows still in flight must land before the CTA exits
            if (issuer)
                for (; gw < gi; gw++)
                    mbar_wait(&rfull[gw % kPR], (uint32_t)((gw / kPR) & 1), a.err, kErrTimeoutDrain);
        }
    } else if (warp == kPMmaWarp) {
        // ----------------------------------------------------- MMA issuer
        if (lane == 0) {
            const uint32_t sA0 = smem_u32(ringA), sB0 = smem_u32(ringB);
            const uint32_t idesc = f16_idesc(256);       // gate|up rows, or 256 down rows
            uint32_t it = 0;
            int lt = 0;
            bool ok = true;
            for (int tau = blockIdx.x; tau < n_tiles && ok; tau += gridDim.x, lt++) {
                const int ab = lt & 1;
                if (!mbar_wait(&acce[ab], (uint32_t)(((lt >> 1) & 1) ^ 1), a.err, kErrTimeoutEmpty)) { ok = false; break; }
                tc_fence_after();
                const uint32_t dacc = tmem + (uint32_t)(ab * 256);
                for (int ks = 0; ks < nk; ks++, it++) {
                    const int sa = it % kPSA, sb = it % kPSB;
                    if (!mbar_wait(&fullA[sa], (it / kPSA) & 1, a.err, kErrTimeoutFull) ||
                        !mbar_wait(&fullB[sb], (it / kPSB) & 1, a.err, kErrTimeoutFull)) { ok = false; break; }
                    fence_proxy_async_smem();
                    tc_fence_after();
                    const uint32_t aa = sA0 + (uint32_t)sa * kPStageA, bb = sB0 + (uint32_t)sb * kPStageB;
#pragma unroll
                    for (int kk = 0; kk < kPK / 16; kk++)
                        tc_mma(dacc, sw128_desc(aa + kk * 32), sw128_desc(bb + kk * 32), idesc, (ks | kk) != 0);
                    tc_commit(&emptyA[sa]);      // the stages are free once these MMAs are done
                    tc_commit(&emptyB[sb]);
                }
                if (!ok) break;
                tc_commit(&accf[ab]);            // the tile's accumulator is complete
            }
            // tensor memory is freed at exit: wait until every MMA issued
            // here has completed (also after a wait that gave up)
            tc_commit(mma_done);
            mbar_wait(mma_done, 0, a.err, kErrTimeoutMma);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------- epilogue
        const int q = warp & 3;                  // TMEM lane quarter of this warp
        const int r = q * 32 + lane;             // tile row
        int lt = 0;
        bool ok = true;
        for (int tau = blockIdx.x; tau < n_tiles && ok; tau += gridDim.x, lt++) {
            const PfTile t = pf_tile(tcum, segs, nv, nt, tau);
            const int ab = lt & 1;
            if (!mbar_wait_warp(&accf[ab], (uint32_t)((lt >> 1) & 1), a.err, kErrTimeoutFull)) { ok = false; break; }
            tc_fence_after();
            const int row = t.m * kPM + r;
            const bool valid = row < t.rows;
            const size_t p = (size_t)t.seg0 + row;
            const uint32_t tq = tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(ab * 256);
            if (MODE == kPGateUp) {
#pragma unroll 1
                for (int c0 = 0; c0 < kPNg; c0 += 32) {
                    uint32_t gv[32], uv[32];
                    tc_ld32(tq + c0, gv);
                    tc_ld32(tq + kPNg + c0, uv);
                    tc_wait_ld();
                    uint32_t hv[16];
#pragma unroll
                    for (int i = 0; i < 16; i++) {
                        const float h0 = silu_fast(__uint_as_float(gv[2 * i])) * __uint_as_float(uv[2 * i]);
                        const float h1 = silu_fast(__uint_as_float(gv[2 * i + 1])) * __uint_as_float(uv[2 * i + 1]);
                        const __half2 hh = __floats2half2_rn(h0, h1);
                        hv[i] = *reinterpret_cast<const uint32_t *>(&hh);
                    }
                    if (valid) {
                        uint4 *dst = reinterpret_cast<uint4 *>(a.H + p * a.F + (size_t)t.n * kPNg + c0);
#pragma unroll
                        for (int i = 0; i < 4; i++)
                            dst[i] = make_uint4(hv[4 * i], hv[4 * i + 1], hv[4 * i + 2], hv[4 * i + 3]);
                    }
                }
            } else {
#pragma unroll 1
                for (int c0 = 0; c0 < kPNd; c0 += 32) {
                    uint32_t y[32];
                    tc_ld32(tq + c0, y);
                    tc_wait_ld();
                    if (valid) {
                        uint4 *dst = reinterpret_cast<uint4 *>(a.Y + p * a.D + (size_t)t.n * kPNd + c0);
#pragma unroll
                        for (int i = 0; i < 8; i++)
                            dst[i] = make_uint4(y[4 * i], y[4 * i + 1], y[4 * i + 2], y[4 * i + 3]);
                    }
                }
            }
            tc_fence_before();
            mbar_arrive(&acce[ab]);
        }
    }
    // everyone is done with the accumulators: release tensor memory
    tc_fence_before();
    __syncthreads();
    if (warp == kPMmaWarp) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;"
                     ::"r"(tmem), "r"(kPTmemCols) : "memory");
    }
}

// x (bf16 or fp32) -> fp16, 8 elements per thread
template <typename XT>
__global__ void __launch_bounds__(256) pf_convert_kernel(const XT *__restrict__ x, __half *__restrict__ y,
                                                         size_t n8) {
    const size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= n8) return;
    uint32_t h[4];
#pragma unroll
    for (int q = 0; q < 4; q++) {
        const __half2 hh = __floats2half2_rn(load_act(x, 8 * i + 2 * q), load_act(x, 8 * i + 2 * q + 1));
        h[q] = *reinterpret_cast<const uint32_t *>(&hh);
    }
    reinterpret_cast<uint4 *>(y)[i] = make_uint4(h[0], h[1], h[2], h[3]);
}

// ------------------------------------------------------------------- host
// K (D for gate/up, F for down) a multiple of 256: a row is then 8m blocks,
// a multiple of 16 bytes; with 18-, 22- or 34-byte blocks its last four
// blocks start 8 bytes past a 16-byte boundary, so every window, the last
// included, ends at or before the row's end and no window reads past a row
// Block types the B producers dequantise: the 32-weight Standard family and
// Q4_K (Q6_K's 210-byte blocks leave rows of F=768 weights unaligned for
// tensor copies; it takes the portable kernels)
static bool pf_type_ok(int qt) { return qt_known(qt) && qt != MOE_Q6_K; }

bool prefill_path_ok(int T, int D, int F, int sF, int E, int qt, int sqt, bool allow_f16) {
    auto ok = [&](int q) { return pf_type_ok(q) || (allow_f16 && qt_known(q)); };
    return T > 16 && D % kPNd == 0 && F % kPNg == 0 && D % 256 == 0 && F % 256 == 0 &&
           (sF == 0 || (sF == F && ok(sqt))) && ok(qt) &&
           E <= kPfMaxExperts && pf_smem_bytes(E) <= 227 * 1024;
}

size_t prefill_x16_halves(int T, int D) { return (size_t)T * D; }
size_t prefill_h_halves(int T, int k, int F, int sF) { return (size_t)(T * k + (sF ? T : 0)) * F; }
size_t prefill_y_floats(int T, int k, int D, int sF) { return (size_t)(T * k + (sF ? T : 0)) * D; }

typedef CUresult (*PfEncodeFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                               const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                               const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                               CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// rows x row_bytes (8-byte elements) at base, boxes of box_bytes x box_rows
static moe_status pf_encode(CUtensorMap *m, const void *base, size_t row_bytes, size_t nrows,
                            int box_bytes, int box_rows) {
    static PfEncodeFn fn = nullptr;
    if (!fn) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = (PfEncodeFn)p;
    }
    if (!fn) { set_error("prefill path: cuTensorMapEncodeTiled unavailable"); return MOE_ERR_CUDA; }
    const cuuint64_t dims[2] = {(cuuint64_t)(row_bytes / 8), (cuuint64_t)nrows};
    const cuuint64_t strides[1] = {(cuuint64_t)row_bytes};
    const cuuint32_t box[2] = {(cuuint32_t)(box_bytes / 8), (cuuint32_t)box_rows};
    const cuuint32_t es[2] = {1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT64, 2, const_cast<void *>(base), dims, strides, box, es,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
        set_error("prefill path: tensor map encoding failed (%d)", (int)r);
        return MOE_ERR_CUDA;
    }
    return MOE_OK;
}

template <int MODE, int BK, int ONE = -1>
static cudaError_t launch_pf1(const PfArgs &a, const PfMaps &m, int grid, cudaStream_t s) {
    const size_t smem = pf_smem_bytes(a.E);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kPThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e = cudaFuncSetAttribute(pf_gemm_kernel<MODE, BK, ONE>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    return cudaLaunchKernelEx(&cfg, pf_gemm_kernel<MODE, BK, ONE>, a, m);
}

template <int MODE>
static cudaError_t launch_pf(const PfArgs &a, const PfMaps &m, int grid, cudaStream_t s, bool f16) {
    if (f16) return launch_pf1<MODE, kBkF16>(a, m, grid, s);
    auto basic = [](int q) { return q == MOE_Q4_0 || q == MOE_Q8_0; };
    const bool all = !basic(a.qt) || (a.shared && !basic(a.sqt));
    if (!a.shared || a.sqt == a.qt) {              // one type: only its code
        switch (a.qt) {
        case MOE_Q4_0: return launch_pf1<MODE, kBkBasic, MOE_Q4_0>(a, m, grid, s);
        case MOE_Q8_0: return launch_pf1<MODE, kBkBasic, MOE_Q8_0>(a, m, grid, s);
        case MOE_Q4_1: return launch_pf1<MODE, kBkAll, MOE_Q4_1>(a, m, grid, s);
        case MOE_Q5_0: return launch_pf1<MODE, kBkAll, MOE_Q5_0>(a, m, grid, s);
        case MOE_Q5_1: return launch_pf1<MODE, kBkAll, MOE_Q5_1>(a, m, grid, s);
        case MOE_Q4_K: return launch_pf1<MODE, kBkAll, MOE_Q4_K>(a, m, grid, s);
        default: break;
        }
    }
    return all ? launch_pf1<MODE, kBkAll>(a, m, grid, s) : launch_pf1<MODE, kBkBasic>(a, m, grid, s);
}

// fp16 tensor maps over a converted pool: [rows][K] halves, boxes of 64
// halves (128 bytes, the 128-byte swizzle's span) x box_rows rows
static moe_status pf_encode_f16(CUtensorMap *m, const __half *base, int K, size_t nrows, int box_rows) {
    static PfEncodeFn fn = nullptr;
    if (!fn) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = (PfEncodeFn)p;
    }
    if (!fn) { set_error("prefill path: cuTensorMapEncodeTiled unavailable"); return MOE_ERR_CUDA; }
    const cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)nrows};
    const cuuint64_t strides[1] = {(cuuint64_t)K * 2};
    const cuuint32_t box[2] = {(cuuint32_t)kPK, (cuuint32_t)box_rows};
    const cuuint32_t es[2] = {1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<__half *>(base), dims, strides, box,
                    es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
        set_error("prefill path: fp16 tensor map encoding failed (%d)", (int)r);
        return MOE_ERR_CUDA;
    }
    return MOE_OK;
}

// A pool's rows of any block type -> fp16 rows (one warp a row, lanes over
// 32-weight units; each weight the portable decoder's fp32 value rounded
// once to fp16)
template <int QT>
__global__ void __launch_bounds__(256)
pf_dequant_f16_kernel(const uint8_t *__restrict__ src, size_t nrows, int ncols, __half *__restrict__ dst) {
    const size_t row = (size_t)blockIdx.x * 8 + (threadIdx.x >> 5);
    if (row >= nrows) return;
    const int lane = threadIdx.x & 31;
    const uint8_t *r = src + row * qt_row_bytes(QT, ncols);
    for (int b = lane; b < ncols / QK; b += 32) {
        float w[32];
        decode_unit_global<QT>(r, b, w);
        uint4 *o = reinterpret_cast<uint4 *>(dst + row * ncols + (size_t)b * QK);
#pragma unroll
        for (int q = 0; q < 4; q++) {
            __half2 h[4];
#pragma unroll
            for (int i = 0; i < 4; i++) h[i] = __floats2half2_rn(w[8 * q + 2 * i], w[8 * q + 2 * i + 1]);
            o[q] = *reinterpret_cast<uint4 *>(h);
        }
    }
}

static moe_status dequant_f16(const uint8_t *src, int qt, size_t nrows, int ncols, __half *dst,
                              cudaStream_t s) {
    const unsigned grid = (unsigned)((nrows + 7) / 8);
    switch (qt) {
#define MOE_DQ(QT) case QT: pf_dequant_f16_kernel<QT><<<grid, 256, 0, s>>>(src, nrows, ncols, dst); break;
        MOE_DQ(MOE_Q4_0)
        MOE_DQ(MOE_Q4_1)
        MOE_DQ(MOE_Q5_0)
        MOE_DQ(MOE_Q5_1)
        MOE_DQ(MOE_Q8_0)
        MOE_DQ(MOE_Q4_K)
        MOE_DQ(MOE_Q6_K)
#undef MOE_DQ
    default:
        set_error("prefill path: unsupported quant type %d", qt);
        return MOE_ERR_UNSUPPORTED_QTYPE;
    }
    return cuda_status(cudaGetLastError(), "pf_dequant_f16_kernel");
}

// halves of the fp16 copies the fp16-weight mode needs (routed pool, then the
// shared expert)
size_t prefill_f16_halves(int n_slots, int D, int F, int sF) {
    return (size_t)n_slots * 3 * D * F + (size_t)3 * D * sF;
}
bool prefill_needs_f16(int qt, int sqt, int sF) { return qt == MOE_Q6_K || (sF > 0 && sqt == MOE_Q6_K); }

moe_status launch_ffn_prefill(const void *x, int x_dtype, int T, int D, int F, int E, int k,
                              const int32_t *perm, const int32_t *offsets, const moe_pool &pool,
                              const uint8_t *mask, bool routed, const moe_pool *shared, int sF,
                              __half *x16, __half *H, float *Y, int *err, cudaStream_t s,
                              Tracer *tr, __half *w16) {
    const bool f16 = prefill_needs_f16(pool.qtype, shared ? shared->qtype : 0, shared ? sF : 0);
    if (f16 && !w16) {
        set_error("prefill path: Q6_K needs the fp16 pool copies (the layer's workspace)");
        return MOE_ERR_UNSUPPORTED_QTYPE;
    }
    if (!f16 && !pf_type_ok(pool.qtype)) {
        set_error("prefill path: unsupported quant type %d", (int)pool.qtype);
        return MOE_ERR_UNSUPPORTED_QTYPE;
    }
    if (!f16 && shared && !pf_type_ok(shared->qtype)) {
        set_error("prefill path: unsupported shared-expert quant type %d", (int)shared->qtype);
        return MOE_ERR_UNSUPPORTED_QTYPE;
    }
    if (!prefill_path_ok(T, D, F, shared ? sF : 0, E, pool.qtype, shared ? shared->qtype : 0, f16)) {
        set_error("prefill path: shape T=%d D=%d F=%d not supported", T, D, F);
        return MOE_ERR_SHAPE;
    }
    PfArgs a{};
    a.T = T; a.D = D; a.F = F; a.E = E; a.k = k;
    a.qt = pool.qtype;
    a.shared = shared ? 1 : 0;
    a.sqt = shared ? shared->qtype : pool.qtype;
    a.routed = routed ? 1 : 0;
    a.n_slots = pool.n_slots;
    a.mask = mask;
    a.perm = perm; a.offsets = offsets;
    a.gate = (const uint8_t *)pool.gate; a.up = (const uint8_t *)pool.up;
    a.down = (const uint8_t *)pool.down; a.slot_map = pool.slot_of_expert;
    if (shared) {
        a.sh_gate = (const uint8_t *)shared->gate; a.sh_up = (const uint8_t *)shared->up;
        a.sh_down = (const uint8_t *)shared->down;
    }
    a.x16 = x16; a.H = H; a.Y = Y; a.err = err;

    // activations to fp16 once (the MMA takes both operands in one type)
    const size_t n8 = (size_t)T * D / 8;
    mark(tr, MOE_KERNEL_CONVERT);
    if (x_dtype == MOE_BF16)
        pf_convert_kernel<__nv_bfloat16><<<(unsigned)((n8 + 255) / 256), 256, 0, s>>>(
            (const __nv_bfloat16 *)x, x16, n8);
    else
        pf_convert_kernel<float><<<(unsigned)((n8 + 255) / 256), 256, 0, s>>>((const float *)x, x16, n8);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_status(e, "pf_convert_kernel");
    PfMaps mg, md;
    memset(&mg, 0, sizeof(mg));
    memset(&md, 0, sizeof(md));
    moe_status st;
    const size_t rows_f = (size_t)pool.n_slots * F, rows_d = (size_t)pool.n_slots * D;
    if (f16) {
        // every slot's weights (and the shared expert's) to fp16 rows, then
        // tensor maps over those
        __half *g16 = w16, *u16 = g16 + rows_f * D, *d16 = u16 + rows_f * D;
        mark(tr, MOE_KERNEL_CONVERT);
        if ((st = dequant_f16((const uint8_t *)pool.gate, pool.qtype, rows_f, D, g16, s)) ||
            (st = dequant_f16((const uint8_t *)pool.up, pool.qtype, rows_f, D, u16, s)) ||
            (st = dequant_f16((const uint8_t *)pool.down, pool.qtype, rows_d, F, d16, s)))
            return st;
        if ((st = pf_encode_f16(&mg.w0, g16, D, rows_f, kPNg)) ||
            (st = pf_encode_f16(&mg.w1, u16, D, rows_f, kPNg)) ||
            (st = pf_encode_f16(&md.w0, d16, F, rows_d, kPNd)))
            return st;
        if (shared) {
            __half *sg16 = d16 + rows_d * F, *su16 = sg16 + (size_t)sF * D, *sd16 = su16 + (size_t)sF * D;
            if ((st = dequant_f16((const uint8_t *)shared->gate, shared->qtype, sF, D, sg16, s)) ||
                (st = dequant_f16((const uint8_t *)shared->up, shared->qtype, sF, D, su16, s)) ||
                (st = dequant_f16((const uint8_t *)shared->down, shared->qtype, D, sF, sd16, s)))
                return st;
            if ((st = pf_encode_f16(&mg.s0, sg16, D, sF, kPNg)) ||
                (st = pf_encode_f16(&mg.s1, su16, D, sF, kPNg)) ||
                (st = pf_encode_f16(&md.s0, sd16, sF, D, kPNd)))
                return st;
        }
        const int grid = num_sms();
        mark(tr, MOE_KERNEL_GATEUP);
        if ((e = launch_pf<kPGateUp>(a, mg, grid, s, true)) != cudaSuccess) return cuda_status(e, "pf_gemm_kernel<gate/up, fp16>");
        mark(tr, MOE_KERNEL_DOWN);
        if ((e = launch_pf<kPDown>(a, md, grid, s, true)) != cudaSuccess) return cuda_status(e, "pf_gemm_kernel<down, fp16>");
        return MOE_OK;
    }
    // weight tensor maps: boxes of one raw window row
    const size_t rg = qt_row_bytes(pool.qtype, D), rd = qt_row_bytes(pool.qtype, F);
    const int wr = pf_window_bytes(pool.qtype);
    if ((st = pf_encode(&mg.w0, pool.gate, rg, rows_f, wr, kPNg)) ||
        (st = pf_encode(&mg.w1, pool.up, rg, rows_f, wr, kPNg)) ||
        (st = pf_encode(&md.w0, pool.down, rd, rows_d, wr, kPNd)))
        return st;
    if (shared) {
        const size_t rgs = qt_row_bytes(shared->qtype, D), rds = qt_row_bytes(shared->qtype, F);
        const int wsh = pf_window_bytes(shared->qtype);
        if ((st = pf_encode(&mg.s0, shared->gate, rgs, F, wsh, kPNg)) ||
            (st = pf_encode(&mg.s1, shared->up, rgs, F, wsh, kPNg)) ||
            (st = pf_encode(&md.s0, shared->down, rds, D, wsh, kPNd)))
            return st;
    }
    const int grid = num_sms();
    mark(tr, MOE_KERNEL_GATEUP);
    if ((e = launch_pf<kPGateUp>(a, mg, grid, s, false)) != cudaSuccess) return cuda_status(e, "pf_gemm_kernel<gate/up>");
    mark(tr, MOE_KERNEL_DOWN);
    if ((e = launch_pf<kPDown>(a, md, grid, s, false)) != cudaSuccess) return cuda_status(e, "pf_gemm_kernel<down>");
    return MOE_OK;
}

}  // namespace moe
