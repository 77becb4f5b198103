// ffn_decode.cu -- the decode (small T) expert FFN: a dequant-fused grouped
// GEMV streamed from HBM by the TMA engine.
//
// Decode reads every active expert's packed blocks once and does a handful
// of FLOPs per weight, so the roofline is HBM bandwidth.  Two persistent
// kernels, one CTA per SM, each with one producer warp and sixteen consumer
// warps around a ring of shared-memory stages:
//
//  * dec_gateup: work unit = (expert, 16-row tile of F).  The producer
//    copies the 16 gate rows and 16 up rows of a K-slice (<= 32 blocks) with
//    cp.async.bulk (one copy per row slice, rows padded so that the
//    consumers' 32-bit loads hit 32 distinct banks).  Consumer warp w takes
//    matrix w / 8 and K-group w % 8.  Codes are turned into exact fp16 values
//    c + q (c = 1024 for Q4_0 codes, 1152 for Q8_0 codes) with bit operations
//    only, and mma.sync m16n8k16 runs with the expert's tokens as the N
//    dimension (the activations are broadcast inside the tensor core).  The
//    constant is removed through the MMA's accumulator input: it starts at
//    -c * sum_k x_k (per block and token, precomputed once), so the block's
//    result is sum (q - off) x exactly up to fp32 rounding, and the block
//    scale d multiplies that fp32 result; no weight is rounded.  The _1
//    types (value q*d + m) add m * sum_k x_k, read from the same table.
//    The other Standard types work the same way: 4-bit codes become
//    1024 + q (Q4_1: off 1024; Q5_0/Q5_1 OR in the fifth bit from the
//    block's qh word: off 1040 / 1024).  A fixed-
//    order cross-warp sum, SwiGLU and the token's gate weight give Hs = g * h
//    in fp16, stored in the fragment order the next kernel reads.
//  * dec_down: work unit = (expert, 64 rows of D): one 2-D box of the
//    expert's down projection over the full F (~28 KB at F=768 Q4_0) and
//    the expert's Hs rows (contiguous in permuted order, one bulk copy).
//    Consumer warps form 4 groups of 4; a group owns every 4th unit of the
//    CTA and a warp one 16-row M-tile of it over the whole reduction, so no
//    partial sums cross warps.  Codes become exact (q - off) fp16 values and
//    the block scale multiplies the fp32 MMA result; for the _1 types a
//    second MMA with an all-ones A gives each column's block sum of Hs,
//    which m multiplies.  Each warp stores its
//    fp32 Y rows (permuted order) to global memory.
//  * dec_combine (fused layer only): y[t] = sum over j of the Y row of
//    (t, j), then the shared expert's row, in that fixed order; the gate
//    weight is already inside Hs.  Without y (the two-phase expert-cache
//    path) the Y rows are the result: un-gated, masked experts skipped.
//
// dec_down is launched with programmatic dependent launch: it copies its
// down-projection weights while dec_gateup is still running and waits
// (griddepcontrol.wait) only before copying Hs.

// Fragment order of an activation block (32 values, one 64-byte row piece):
// for c = 0..3 eight halves [v(4c), v(4c+2), v(4c+1), v(4c+3), v(16+4c),
// v(18+4c), v(17+4c), v(19+4c)], matching the codes one 32-bit word of a
// Q4_0 block gives thread c (byte j = v_j | v_{j+16} << 4), and the two
// words (bytes 4c.., 16+4c..) of a Q8_0 block.
#include "moe_internal.cuh"
#include "sm100.cuh"

#include <cuda.h>
#include <algorithm>
#include <climits>
#include <cstring>

namespace moe {

constexpr int kTile = 16;                       // rows per MMA tile
constexpr int kMaxStages = 8;
constexpr size_t kDecSmemMax = 225 * 1024;      // dynamic; leaves room for static smem
constexpr int kDW = 16;                         // consumer warps
constexpr int kDThreads = (kDW + 1) * 32;       // + producer warp
constexpr int kEW = 2;                          // gate/up epilogue warps
constexpr int kGThreads = kDThreads + kEW * 32; // gate/up block
// gate/up partial-sum buffers between the MMA warps and the epilogue warps
constexpr int kGuRedBufs = 2;
// gate/up units cover at most 8 tokens of an expert (one MMA N tile); an
// expert with more tokens gets one unit per 8-token column group
constexpr int kGuCols = 8;
constexpr int kMaxTk = 16 * MOE_MAX_TOPK;       // T*k entries the token tables hold

struct DecArgs {
    int T, D, F, E, k, sF;         // sF: shared expert's F when this call runs it, else 0
    int qt, sqt;                   // block types (ggml ids) of the routed / shared experts
    int routed;                    // this call runs the routed experts (those mask admits)
    int n_slots;                   // slots of the routed pool
    int comb_shared;               // the combine adds the shared rows (layer has one)
    const int32_t *perm, *offsets;
    const float *gates;            // [T, k] or NULL (rows mode: no gate)
    const uint8_t *mask;           // [E] or NULL
    const uint8_t *gate, *up, *down;
    const int32_t *slot_map;
    const uint8_t *sh_gate, *sh_up, *sh_down;
    const void *x;
    int x_bf16;
    int x_vec;                     // x is 16-byte aligned (vector loads)
    __half *Hs;                    // [T*k + T][hrow] fragment order
    int hrow;                      // halves per Hs row
    void *y;                       // [T, D] (combine mode)
    int y_dtype;
    float *rows_out;               // [T*k (+T), D] Y rows, permuted order (+ shared rows)
    const int32_t *inv;            // [T*k] for the combine (fused layer)
    int *err;
};

// slice geometry: blocks per K-slice (<= 32, a multiple of 8)
__host__ __device__ inline int slice_blocks(int ncols) {
    int nb = ncols / QK;
    return nb <= 32 ? nb : 32;
}
// Staged weight row: the slice plus padding chosen so that the row stride in
// 32-bit words is an odd multiple of 4: threads (g = 0..7, c = 0..3) loading
// word c of row g then touch 32 distinct banks.
__host__ __device__ inline int staged_row_bytes(int sb, int bs) {
    const int w = sb * bs / 4;                  // sb * bs is a multiple of 16
    return sb * bs + ((w % 8 == 0) ? 16 : 32);
}
// Shared-memory pitch of a weight row staged by a 2-D TMA copy: the row
// bytes rounded up to 16 and then to an ODD multiple of 16, so the pitch in
// 32-bit words is 4 x odd: threads (g = 0..7, c = 0..3) loading word c of
// row g hit 32 distinct banks.  The extra bytes are out-of-bounds elements
// of the box, which the copy engine fills with zeros.
__host__ __device__ inline int tma_row_bytes(int rb) {
    int r = (rb + 15) / 16 * 16;
    if (((r / 16) & 1) == 0) r += 16;
    return r;
}
// Shared-memory pitch of a down-projection row (F weights): as
// tma_row_bytes, except Q6_K, whose rows (210 * F / 256 bytes, 2-byte
// aligned when F / 256 is odd) arrive as whole 8-row groups (16-byte
// multiples) and stay packed.
__host__ __device__ inline int dn_pitch(int qt, int F) {
    const int rb = (int)qt_row_bytes(qt, F);
    return qt == MOE_Q6_K ? rb : tma_row_bytes(rb);
}
// Q6_K down rows as a 3-D tensor: 560-byte chunks (70 elements of 8 bytes),
// 3 F / 256 chunks an 8-row group, one group per 8 rows of D
constexpr int kQ6Chunk = 560;

// Blocks per K-slice for a block size: the largest multiple of 8 dividing
// the row's nb blocks whose staged row still fits one box (<= 256 elements
// of 8 bytes = 2048 bytes).
__host__ __device__ inline int slice_blocks_q(int nb, int bs, int max_sb) {
    for (int sb = nb < max_sb ? nb : max_sb; sb >= 8; sb -= 8)
        if (nb % sb == 0 && tma_row_bytes(sb * bs) <= 2048) return sb;
    return 8;
}

// The weight pools as 2-D tensors of 8-byte elements (one row of blocks per
// tensor row), boxes of 16 rows: one TMA request per 16-row tile and slice.
struct DecMaps {
    CUtensorMap gate, up, down;        // routed pool
    CUtensorMap sgate, sup, sdown;     // shared expert
};

// Staged activation row (fp16 fragment order): stride = 64 mod 128 bytes so
// that rows n, n+1 read by one quarter-warp's 16-byte loads do not collide.
__host__ __device__ inline int staged_act_bytes(int ncols) { return ncols * 2 + 64; }

// ---------------------------------------------------------- shared loads
__device__ __forceinline__ uint32_t lds32(uint32_t a) {
    uint32_t v;
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(a));
    return v;
}
__device__ __forceinline__ uint32_t lds16(uint32_t a) {
    unsigned short v;
    asm volatile("ld.shared.u16 %0, [%1];" : "=h"(v) : "r"(a));
    return v;
}
__device__ __forceinline__ uint4 lds128(uint32_t a) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a));
    return v;
}
__device__ __forceinline__ float ldsf(uint32_t a) { return __uint_as_float(lds32(a)); }

// 32-bit word at a shared address whose alignment mod 4 is MIS (0 or 2),
// known at compile time.
template <int MIS>
__device__ __forceinline__ uint32_t lds_word(uint32_t a) {
    if constexpr (MIS == 0) {
        return lds32(a);
    } else {
        const uint32_t lo = lds32(a - 2), hi = lds32(a + 2);
        return __funnelshift_r(lo, hi, 16);
    }
}

__device__ __forceinline__ float h2f(uint32_t bits) {
    return __half2float(__ushort_as_half((unsigned short)bits));
}

// ------------------------------------------------------------ active list
struct Active {
    int n_routed;   // active routed experts
    int n_virt;     // + 1 when a shared expert exists
};

// act: shared int[6 * (E + 1)]: expert id, segment start, token count and
// slot of every active expert (ascending id), then the raw offsets and
// slots.  All threads load the raw tables in one round of global loads;
// one warp then compacts them, so per-unit lookups stay in shared memory.
// An expert is active when it has tokens, this call runs routed experts and
// the mask (if any) admits it.  An active expert whose slot lies outside
// [0, n_slots) is left out and recorded as kErrBadSlot: no address is ever
// formed from such a slot.
constexpr int kMaskedOut = INT_MIN;

__device__ Active build_active_list(const DecArgs &a, int *act) {
    __shared__ int s_n;
    const int E1 = a.E + 1;
    int *aseg = act + E1, *acnt = aseg + E1, *aslot = acnt + E1;
    int *roff = aslot + E1, *ron = roff + E1;
    for (int e = threadIdx.x; e <= a.E; e += blockDim.x) {
        roff[e] = __ldg(a.offsets + e);
        if (e < a.E)
            ron[e] = (a.routed && (!a.mask || __ldg(a.mask + e))) ? slot_of(a.slot_map, e) : kMaskedOut;
    }
    __syncthreads();
    if (threadIdx.x < 32) {
        int base = 0;
        for (int e0 = 0; e0 < a.E; e0 += 32) {
            const int e = e0 + threadIdx.x;
            bool on = false;
            int s0 = 0, c = 0, sl = 0;
            if (e < a.E) {
                s0 = roff[e];
                c = roff[e + 1] - s0;
                sl = ron[e];
                const bool want = c > 0 && sl != kMaskedOut;
                const bool bad = want && (sl < 0 || sl >= a.n_slots);
                if (bad && a.err) atomicCAS(a.err, 0, kErrBadSlot);
                on = want && !bad;
            }
            const unsigned b = __ballot_sync(0xffffffffu, on);
            if (on) {
                const int i = base + __popc(b & ((1u << threadIdx.x) - 1u));
                act[i] = e;
                aseg[i] = s0;
                acnt[i] = c;
                aslot[i] = sl;
            }
            base += __popc(b);
        }
        if (threadIdx.x == 0) s_n = base;
    }
    __syncthreads();
    Active r;
    r.n_routed = s_n;
    r.n_virt = s_n + (a.sF > 0 ? 1 : 0);
    return r;
}

// Virtual expert v: routed act[v] for v < n_routed, else the shared expert.
struct Virt {
    int seg0, cnt, Fv;
    size_t slot;
    bool shared;
    int qt;
};

__device__ __forceinline__ Virt virt(const DecArgs &a, const int *act, int n_routed, int v) {
    Virt r;
    if (v < n_routed) {
        const int *aseg = act + (a.E + 1), *acnt = aseg + (a.E + 1), *aslot = acnt + (a.E + 1);
        r.seg0 = aseg[v];
        r.cnt = acnt[v];
        r.Fv = a.F;
        r.slot = (size_t)aslot[v];
        r.shared = false;
        r.qt = a.qt;
    } else {
        r.seg0 = a.T * a.k;
        r.cnt = a.T;
        r.Fv = a.sF;
        r.slot = 0;
        r.shared = true;
        r.qt = a.sqt;
    }
    return r;
}

// Producer's exit: wait (bounded) until the last fill of every stage it used
// has landed, so no copy still writes shared memory when the CTA ends.  The
// full barrier of a stage completes the phase of a fill when its bytes
// arrive, whatever the consumers did.
__device__ __forceinline__ void drain_fills(uint64_t *full, int S, uint32_t used, uint32_t last_ph,
                                            int *err) {
    for (int s = 0; s < S; s++)
        if ((used >> s) & 1u) mbar_wait(&full[s], (last_ph >> s) & 1u, err, kErrTimeoutDrain);
}

// Token tables in shared memory: tok[pos] = token of permuted entry pos
// (T*k entries) followed by tok[T*k + t] = t for the shared expert; gw[pos]
// = gate weight of entry pos.
__device__ void load_token_tables(const DecArgs &a, int *tok, float *gw) {
    const int Tk = a.T * a.k;
    for (int p = threadIdx.x; p < Tk + a.T; p += blockDim.x) {
        if (p < Tk) {
            const int n = __ldg(a.perm + p);
            tok[p] = n / a.k;
            if (gw) gw[p] = a.gates ? __ldg(a.gates + n) : 1.0f;
        } else {
            tok[p] = p - Tk;
            if (gw) gw[p] = 1.0f;
        }
    }
}

// index (in halves) of row element i (0..31 within its block) in fragment order
__host__ __device__ __forceinline__ int frag_slot(int i) {
    const int c = (i & 15) >> 2, j = i & 3, hi = i >> 4;
    const int jj = (j == 0) ? 0 : (j == 2) ? 1 : (j == 1) ? 2 : 3;
    return c * 8 + hi * 4 + jj;
}

// ---------------------------------------------------- code extraction
// Exact fp16 pairs of (const + code) for the 8 weights of one row that
// thread c owns in a block: r[0] = (v4c, v4c+2), r[1] = (v4c+1, v4c+3),
// r[2] = (v16+4c, v18+4c), r[3] = (v17+4c, v19+4c), where v = 1024 + q for
// the 4- and 5-bit types (0 <= q < 32) or v = 1152 + q (Q8_0, int8 q).
// blk: shared address of the block; MIS = alignment mod 4 of its codes
// (the 5-bit types' qh word sits 4 bytes before them: the same alignment).
template <int QT, int MIS>
__device__ __forceinline__ void magic_codes(uint32_t blk, int c, uint32_t *r) {
    const uint32_t qa = blk + qt_qs_off(QT) + 4 * c;
    if constexpr (qt_has_high(QT)) {
        // 5-bit codes as bytes (low four bits from qs, bit i of qh is bit 4
        // of element i): elements 4c..4c+3 and 16+4c..19+4c, then bytes
        // into the halves of the fragment order
        const uint32_t w = lds_word<MIS>(qa);
        const uint32_t h = lds_word<MIS>(blk + qt_qh_off(QT)) >> (4 * c);
        const uint32_t lo = lop3_and_or(w, 0x0F0F0F0Fu, spread4_bit4(h & 0xFu));
        const uint32_t hi = lop3_and_or(w >> 4, 0x0F0F0F0Fu, spread4_bit4((h >> 16) & 0xFu));
        const uint32_t HI = 0x64646464u;
        r[0] = prmt(lo, HI, 0x4240);
        r[1] = prmt(lo, HI, 0x4341);
        r[2] = prmt(hi, HI, 0x4240);
        r[3] = prmt(hi, HI, 0x4341);
    } else if constexpr (QT != MOE_Q8_0) {
        const uint32_t w = lds_word<MIS>(qa);
        const uint32_t M = 0x000F000Fu, MAG = 0x64006400u;
        r[0] = lop3_and_or(w, M, MAG);
        r[2] = lop3_and_or(w >> 4, M, MAG);
        r[1] = lop3_and_or(w >> 8, M, MAG);
        r[3] = lop3_and_or(w >> 12, M, MAG);
    } else {
        const uint32_t w0 = lds_word<MIS>(qa) ^ 0x80808080u;
        const uint32_t w1 = lds_word<MIS>(qa + 16) ^ 0x80808080u;
        const uint32_t HI = 0x64646464u;
        r[0] = prmt(w0, HI, 0x4240);
        r[1] = prmt(w0, HI, 0x4341);
        r[2] = prmt(w1, HI, 0x4240);
        r[3] = prmt(w1, HI, 0x4341);
    }
}

// the magic constant minus the code of value zero: (v - off) * d is the
// weight of a _0 type, (v - off) * d + m of a _1 type
__host__ __device__ constexpr float magic_off(int qt) {
    return qt == MOE_Q8_0 ? 1152.f : 1024.f + (float)qt_zero(qt);
}
// the same in half2 form (1024 + z is exact in fp16: z < 32)
template <int QT> __device__ __forceinline__ uint32_t magic_off2() {
    constexpr uint32_t h = QT == MOE_Q8_0 ? 0x6480u : 0x6400u + (uint32_t)qt_zero(QT);
    return h | (h << 16);
}
// alignment mod 4 of the codes of block bl when the block group starts at
// alignment MIS0
template <int QT, int MIS0> __device__ __forceinline__ constexpr int codes_mis(int bl) {
    return (MIS0 + bl * qt_bytes(QT) + qt_qs_off(QT)) & 3;
}

// ---------------------------------------------------------------- gate/up
// One K-slice of one 16-row tile for one warp: WB blocks starting at the
// warp's first block.  row: shared address of row g at that block; xa: the B
// row of column g (and g+8) at that block; sa: the -off*sum(x) entries of
// columns 2c, 2c+1 (and +8) at that block.  MIS0 = alignment mod 4 of the
// first block's start (the code bytes start 2 bytes later; BS is 2 mod 4).
// For the _1 types the table entries are -1024 * sum(x), so m * sum(x) =
// (-m / 1024) * entry, the scaling by a power of two being exact.
template <int QT, int NTILE, int WB, int MIS0>
__device__ __forceinline__ void gateup_slice(uint32_t row, uint32_t r8, const uint32_t *xa,
                                             const uint32_t (*sa)[2], int c, float (*acc)[4]) {
    constexpr int BS = qt_bytes(QT);
#pragma unroll
    for (int bl = 0; bl < WB; bl++) {
        const uint32_t blk = row + bl * BS;
        uint32_t lo[4], hi[4];
        if (codes_mis<QT, MIS0>(bl) == 0) {
            magic_codes<QT, 0>(blk, c, lo);
            magic_codes<QT, 0>(blk + r8, c, hi);
        } else {
            magic_codes<QT, 2>(blk, c, lo);
            magic_codes<QT, 2>(blk + r8, c, hi);
        }
        const float dlo = h2f(lds16(blk)), dhi = h2f(lds16(blk + r8));
        float mlo = 0.f, mhi = 0.f;
        if constexpr (qt_has_min(QT)) {
            mlo = h2f(lds16(blk + 2)) * (-1.f / 1024.f);
            mhi = h2f(lds16(blk + r8 + 2)) * (-1.f / 1024.f);
        }
        const uint32_t a0[4] = {lo[0], hi[0], lo[1], hi[1]};
        const uint32_t a1[4] = {lo[2], hi[2], lo[3], hi[3]};
#pragma unroll
        for (int nt = 0; nt < NTILE; nt++) {
            const uint4 b = lds128(xa[nt] + bl * 64);
            const float s0 = ldsf(sa[nt][0] + bl * 4), s1 = ldsf(sa[nt][1] + bl * 4);
            float p[4] = {s0, s1, s0, s1};
            mma_16816(p, a0, b.x, b.y, p);
            mma_16816(p, a1, b.z, b.w, p);
            acc[nt][0] = fmaf(dlo, p[0], acc[nt][0]);
            acc[nt][1] = fmaf(dlo, p[1], acc[nt][1]);
            acc[nt][2] = fmaf(dhi, p[2], acc[nt][2]);
            acc[nt][3] = fmaf(dhi, p[3], acc[nt][3]);
            if constexpr (qt_has_min(QT)) {
                acc[nt][0] = fmaf(mlo, s0, acc[nt][0]);
                acc[nt][1] = fmaf(mlo, s1, acc[nt][1]);
                acc[nt][2] = fmaf(mhi, s0, acc[nt][2]);
                acc[nt][3] = fmaf(mhi, s1, acc[nt][3]);
            }
        }
    }
}

// ---------------------------------------------------------------- Q4_K
// Q4_K rows are runs of 144-byte blocks (16-byte aligned in a staged row):
// unit b of a row (32 weights) is sub-block b % 8 of block b / 8.  Its codes
// for thread c, in the fragment order above, are nibble (j & 1) of the two
// words at bytes 4c and 16 + 4c of the block's 32-byte chunk j / 2.
__device__ __forceinline__ void q4k_codes(uint32_t blk, int j, int c, uint32_t *r) {
    const uint32_t qa = blk + 16 + 32 * (j >> 1) + 4 * c;
    const int sh = 4 * (j & 1);
    const uint32_t w0 = (lds32(qa) >> sh) & 0x0F0F0F0Fu, w1 = (lds32(qa + 16) >> sh) & 0x0F0F0F0Fu;
    const uint32_t HI = 0x64646464u;
    r[0] = prmt(w0, HI, 0x4240);
    r[1] = prmt(w0, HI, 0x4341);
    r[2] = prmt(w1, HI, 0x4240);
    r[3] = prmt(w1, HI, 0x4341);
}
// A Q4_K block's head: d, dmin and its eight 6-bit scales and mins, unpacked
// four to a word (byte j & 3 of word j / 4) with a few word-wide masks and
// shifts: sub-block j < 4 keeps the low six bits of byte j of scales[0..3]
// (scale) and scales[4..7] (min); j >= 4 takes the low (scale) or high (min)
// nibble of scales[8 + j - 4] and, as bits 4 and 5, the top two bits of
// byte j - 4 of scales[0..3] (scale) or scales[4..7] (min)
struct Q4kHead {
    uint32_t sc[2], mn[2];
    float d, dmin;
};
__device__ __forceinline__ Q4kHead q4k_head(uint32_t blk) {
    const uint32_t w = lds32(blk), s0 = lds32(blk + 4), s1 = lds32(blk + 8), s2 = lds32(blk + 12);
    Q4kHead h;
    h.sc[0] = s0 & 0x3F3F3F3Fu;
    h.mn[0] = s1 & 0x3F3F3F3Fu;
    h.sc[1] = (s2 & 0x0F0F0F0Fu) | ((s0 >> 2) & 0x30303030u);
    h.mn[1] = ((s2 >> 4) & 0x0F0F0F0Fu) | ((s1 >> 2) & 0x30303030u);
    h.d = h2f(w & 0xFFFFu);
    h.dmin = h2f(w >> 16);
    return h;
}
// Scale D = d * sc_j and min M = dmin * m_j of sub-block j (weight D q - M)
__device__ __forceinline__ void q4k_params(const Q4kHead &h, int j, float *D, float *M) {
    const uint32_t sel = 0x4440u | (uint32_t)(j & 3);          // byte j & 3, zero above
    *D = h.d * (float)prmt(j < 4 ? h.sc[0] : h.sc[1], 0u, sel);
    *M = h.dmin * (float)prmt(j < 4 ? h.mn[0] : h.mn[1], 0u, sel);
}

// As gateup_slice for Q4_K: units kb0 .. kb0 + WB - 1 of the slice whose
// staged row starts at rowbase.  The Sx table entries are -1024 * sum(x),
// so the min's share -M * sum(x) is (M / 1024) * entry.
template <int NTILE, int WB>
__device__ __forceinline__ void gateup_slice_q4k(uint32_t rowbase, uint32_t r8, int kb0,
                                                 const uint32_t *xa, const uint32_t (*sa)[2], int c,
                                                 float (*acc)[4]) {
    // WB dividing 8: the warp's units lie in one block (kb0 a multiple of
    // WB), whose head is read once
    constexpr bool ONE = 8 % WB == 0;
    Q4kHead hlo{}, hhi{};
    if constexpr (ONE) {
        const uint32_t blk0 = rowbase + (uint32_t)(kb0 >> 3) * 144u;
        hlo = q4k_head(blk0);
        hhi = q4k_head(blk0 + r8);
    }
#pragma unroll
    for (int bl = 0; bl < WB; bl++) {
        const int b = kb0 + bl;
        const int j = WB == 8 ? bl : (b & 7);
        const uint32_t blk = rowbase + (uint32_t)((WB == 8 ? kb0 : b) >> 3) * 144u;
        uint32_t lo[4], hi[4];
        q4k_codes(blk, j, c, lo);
        q4k_codes(blk + r8, j, c, hi);
        if constexpr (!ONE) {
            hlo = q4k_head(blk);
            hhi = q4k_head(blk + r8);
        }
        float dlo, mlo, dhi, mhi;
        q4k_params(hlo, j, &dlo, &mlo);
        q4k_params(hhi, j, &dhi, &mhi);
        mlo *= 1.f / 1024.f;
        mhi *= 1.f / 1024.f;
        const uint32_t a0[4] = {lo[0], hi[0], lo[1], hi[1]};
        const uint32_t a1[4] = {lo[2], hi[2], lo[3], hi[3]};
#pragma unroll
        for (int nt = 0; nt < NTILE; nt++) {
            const uint4 b4 = lds128(xa[nt] + bl * 64);
            const float s0 = ldsf(sa[nt][0] + bl * 4), s1 = ldsf(sa[nt][1] + bl * 4);
            float p[4] = {s0, s1, s0, s1};
            mma_16816(p, a0, b4.x, b4.y, p);
            mma_16816(p, a1, b4.z, b4.w, p);
            acc[nt][0] = fmaf(mlo, s0, fmaf(dlo, p[0], acc[nt][0]));
            acc[nt][1] = fmaf(mlo, s1, fmaf(dlo, p[1], acc[nt][1]));
            acc[nt][2] = fmaf(mhi, s0, fmaf(dhi, p[2], acc[nt][2]));
            acc[nt][3] = fmaf(mhi, s1, fmaf(dhi, p[3], acc[nt][3]));
        }
    }
}

// ---------------------------------------------------------------- Q6_K
// Q6_K blocks are 210 bytes (ql[128], qh[64], int8 scales[16], fp16 d), so
// consecutive blocks alternate between 4-byte and 2-byte alignment: MIS is
// the block's alignment mod 4.  Sub-block j (32 weights, unit j of the block)
// lies in half h = j / 4, quarter r = j % 4: weight l of it has its low four
// bits in nibble r / 2 of ql[64h + 32(r % 2) + l] and its high two in bits
// 2r, 2r+1 of qh[32h + l], scale scales[8h + 2r + l / 16].  Codes for thread
// c in the fragment order of magic_codes, as exact fp16 (q - 32).
template <int MIS>
__device__ __forceinline__ void q6k_codes(uint32_t blk, int j, int c, uint32_t *r) {
    const int h = j >> 2, q = j & 3;
    const uint32_t la = blk + 64 * h + 32 * (q & 1) + 4 * c, ha = blk + 128 + 32 * h + 4 * c;
    const int s4 = 4 * (q >> 1), s2 = 2 * q;
    const uint32_t w0 = ((lds_word<MIS>(la) >> s4) & 0x0F0F0F0Fu) |
                        (((lds_word<MIS>(ha) >> s2) & 0x03030303u) << 4);
    const uint32_t w1 = ((lds_word<MIS>(la + 16) >> s4) & 0x0F0F0F0Fu) |
                        (((lds_word<MIS>(ha + 16) >> s2) & 0x03030303u) << 4);
    const uint32_t HI = 0x64646464u, OFF = 0x64206420u;          // 1024 + code, minus 1056
    r[0] = hsub2_u(prmt(w0, HI, 0x4240), OFF);
    r[1] = hsub2_u(prmt(w0, HI, 0x4341), OFF);
    r[2] = hsub2_u(prmt(w1, HI, 0x4240), OFF);
    r[3] = hsub2_u(prmt(w1, HI, 0x4341), OFF);
}
// d * scale of the two 16-weight halves of sub-block j (d: the block's)
__device__ __forceinline__ void q6k_scales(uint32_t blk, int j, float d, float *D0, float *D1) {
    const uint32_t s = lds16(blk + 192 + 2 * j);
    *D0 = d * (float)(int)(int8_t)(s & 0xFFu);
    *D1 = d * (float)(int)(int8_t)(s >> 8);
}
// One Q6_K block (8 units) of a 16-row tile against the B fragments at ba
// (64 bytes a unit): each unit's two 16-weight halves take their own MMA and
// scale.  Used by the gate/up warps (B = activations) and the down warps
// (B = Hs).
template <int MIS, int NTILE>
__device__ __forceinline__ void block_q6k(uint32_t blk, uint32_t r8, const uint32_t *ba, int c,
                                          float (*acc)[4]) {
    const float zero[4] = {0.f, 0.f, 0.f, 0.f};
    const float dl = h2f(lds16(blk + 208)), dh = h2f(lds16(blk + r8 + 208));
#pragma unroll
    for (int j = 0; j < 8; j++) {
        uint32_t lo[4], hi[4];
        q6k_codes<MIS>(blk, j, c, lo);
        q6k_codes<MIS>(blk + r8, j, c, hi);
        float d0lo, d1lo, d0hi, d1hi;
        q6k_scales(blk, j, dl, &d0lo, &d1lo);
        q6k_scales(blk + r8, j, dh, &d0hi, &d1hi);
        const uint32_t a0[4] = {lo[0], hi[0], lo[1], hi[1]};
        const uint32_t a1[4] = {lo[2], hi[2], lo[3], hi[3]};
#pragma unroll
        for (int nt = 0; nt < NTILE; nt++) {
            const uint4 b4 = lds128(ba[nt] + j * 64);
            float p0[4], p1[4];
            mma_16816(p0, a0, b4.x, b4.y, zero);
            mma_16816(p1, a1, b4.z, b4.w, zero);
            acc[nt][0] = fmaf(d1lo, p1[0], fmaf(d0lo, p0[0], acc[nt][0]));
            acc[nt][1] = fmaf(d1lo, p1[1], fmaf(d0lo, p0[1], acc[nt][1]));
            acc[nt][2] = fmaf(d1hi, p1[2], fmaf(d0hi, p0[2], acc[nt][2]));
            acc[nt][3] = fmaf(d1hi, p1[3], fmaf(d0hi, p0[3], acc[nt][3]));
        }
    }
}

// K1 geometry of one quant type at a given D
struct GuGeo {
    int sb, nsl, pitch;                 // blocks per slice, slices, staged row pitch
};
// max_sb: the largest slice (in blocks) a stage may hold
__host__ __device__ inline GuGeo gu_geo(int D, int qt, int max_sb) {
    const int bs = qt_unit_bytes(qt), nb = D / QK;
    GuGeo g;
    if (qt == MOE_Q6_K) {             // whole rows of 8 blocks (D = 2048: 1680 bytes)
        g.sb = nb;
        g.nsl = 1;
        g.pitch = tma_row_bytes((int)qt_row_bytes(qt, D));
        return g;
    }
    g.sb = slice_blocks_q(nb, bs, max_sb);
    g.nsl = nb / g.sb;
    g.pitch = tma_row_bytes(g.sb * bs);
    return g;
}

// ALL: the call has a type other than Q4_0 and Q8_0 (a separate
// instantiation keeps the other types' code out of the two types' kernel);
// ONE >= 0: every expert of the call has block type ONE (an instantiation
// with only that type's code: smaller, fewer instruction-cache misses; the
// Q4_0 decode layer's FFN ran 4-5% faster so)
template <int MAXSB, int WB4, int WB8, bool ALL, int ONE = -1>
__global__ void __launch_bounds__(kGThreads, 1)
dec_gateup_kernel(DecArgs a, int S, const __grid_constant__ DecMaps maps) {
    constexpr int NT = 1;
    extern __shared__ __align__(1024) uint8_t smem[];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g = lane >> 2, c = lane & 3;
    const int T = a.T, D = a.D;
    const int nbD = D / QK;
    constexpr int kMaxSb = MAXSB;
    const GuGeo geoR = gu_geo(D, a.qt, kMaxSb), geoS = gu_geo(D, a.sqt, kMaxSb);
    const int pitch_max = max(geoR.pitch, a.sF > 0 ? geoS.pitch : 0);
    const int stage_bytes = (int)round_up((size_t)2 * kTile * pitch_max, 128);
    const int xrow = staged_act_bytes(D);
    const int mat = warp >> 3, kg = warp & 7;

    // carve (from a 1024-aligned base; tensor copies need 128-byte aligned
    // destinations): xs [T+1 rows, the last zero] | Sx tables [2][T+1][nbD]
    // | stages | red [NB][kDW][NT][32][4] | barriers | act | tok | gw | units
    uint8_t *base = smem + ((1024u - (smem_u32(smem) & 1023u)) & 1023u);
    const size_t xs_bytes = round_up((size_t)(T + 1) * xrow, 16);
    uint8_t *xs = base;
    float *sxt = (float *)(base + xs_bytes);
    uint8_t *stages = base + round_up(xs_bytes + (size_t)2 * (T + 1) * nbD * 4, 1024);
    constexpr int NB = kGuRedBufs;
    float *red = (float *)(stages + (size_t)S * stage_bytes);
    uint64_t *full = (uint64_t *)(red + NB * kDW * NT * 32 * 4);
    uint64_t *empty = full + kMaxStages;
    uint64_t *rfull = empty + kMaxStages;          // [4] partials of a unit written
    uint64_t *rempty = rfull + 4;                  // [4] a unit's epilogue done
    int *act = (int *)(rempty + 4);
    int *tok = act + 6 * (a.E + 1);
    float *gw = (float *)(tok + kMaxTk + 16);
    int4 *utab = reinterpret_cast<int4 *>(                 // this CTA's units
        (reinterpret_cast<uintptr_t>(gw + kMaxTk + 16) + 15) & ~(uintptr_t)15);

    if (tid == 0) {
        for (int s = 0; s < S; s++) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kDW);
        }
        for (int b = 0; b < NB; b++) {
            mbar_init(&rfull[b], kDW);            // one elected lane per MMA warp
            mbar_init(&rempty[b], kEW);           // one per epilogue warp
        }
        fence_mbar_init();
    }
    // The activations do not depend on the routing kernel this grid may
    // overlap with: stage them (fp16, fragment order; row T is zero) and the
    // per-block -off * sum(x) tables before waiting for it.  One (token,
    // block) of 32 values per thread, all of its loads in flight at once.
    for (int idx = tid; idx < (T + 1) * nbD; idx += kGThreads) {
        const int t = idx / nbD, b = idx % nbD;
        float v[32];
        if (t < T) {
            const size_t xb = (size_t)t * D + b * QK;
            if (a.x_vec && a.x_bf16) {
                const uint4 *p = reinterpret_cast<const uint4 *>((const __nv_bfloat16 *)a.x + xb);
                uint4 w[4];
#pragma unroll
                for (int q = 0; q < 4; q++) w[q] = __ldg(p + q);
#pragma unroll
                for (int q = 0; q < 4; q++) {
                    const uint32_t u[4] = {w[q].x, w[q].y, w[q].z, w[q].w};
#pragma unroll
                    for (int r = 0; r < 4; r++) {
                        v[8 * q + 2 * r] = __uint_as_float(u[r] << 16);
                        v[8 * q + 2 * r + 1] = __uint_as_float(u[r] & 0xFFFF0000u);
                    }
                }
            } else if (a.x_vec) {
                const float4 *p = reinterpret_cast<const float4 *>((const float *)a.x + xb);
                float4 w[8];
#pragma unroll
                for (int q = 0; q < 8; q++) w[q] = __ldg(p + q);
#pragma unroll
                for (int q = 0; q < 8; q++) {
                    v[4 * q] = w[q].x; v[4 * q + 1] = w[q].y; v[4 * q + 2] = w[q].z; v[4 * q + 3] = w[q].w;
                }
            } else {
#pragma unroll
                for (int i = 0; i < 32; i++)
                    v[i] = a.x_bf16 ? load_act((const __nv_bfloat16 *)a.x, xb + i)
                                    : load_act((const float *)a.x, xb + i);
            }
        } else {
#pragma unroll
            for (int i = 0; i < 32; i++) v[i] = 0.f;
        }
        uint32_t h[32];
        float sum = 0.f;
#pragma unroll
        for (int i = 0; i < 32; i++) {
            const __half hv = __float2half_rn(v[i]);
            h[i] = (uint32_t)__half_as_ushort(hv);
            sum += __half2float(hv);
        }
        uint8_t *dst = xs + (size_t)t * xrow + b * 64;
#pragma unroll
        for (int cc = 0; cc < 4; cc++) {
            uint4 pk;
            pk.x = h[4 * cc] | (h[4 * cc + 2] << 16);
            pk.y = h[4 * cc + 1] | (h[4 * cc + 3] << 16);
            pk.z = h[16 + 4 * cc] | (h[18 + 4 * cc] << 16);
            pk.w = h[17 + 4 * cc] | (h[19 + 4 * cc] << 16);
            *reinterpret_cast<uint4 *>(dst + cc * 16) = pk;
        }
        sxt[idx] = -magic_off(a.qt) * sum;
        sxt[(size_t)(T + 1) * nbD + idx] = -magic_off(a.sqt) * sum;
    }
    __syncthreads();
    // routing results come from the previous kernel
    pdl_wait();
    pdl_launch_dependents();
    load_token_tables(a, tok, gw);                // in flight with the next loads
    const Active A = build_active_list(a, act);   // includes __syncthreads
    const int tiles_r = a.F / kTile, tiles_s = a.sF / kTile;
    // units: (virtual expert, 8-token column group, 16-row tile), expert-
    // major; ucum[v] = first unit of virtual expert v (in the raw-table
    // space of the active list, free now)
    int *ucum = act + 4 * (a.E + 1);
    if (warp == 0) {
        int base = 0;
        for (int v0 = 0; v0 < A.n_virt; v0 += 32) {
            const int v = v0 + lane;
            int nu = 0;
            if (v < A.n_virt) {
                const Virt vi = virt(a, act, A.n_routed, v);
                nu = (vi.cnt + kGuCols - 1) / kGuCols * (vi.shared ? tiles_s : tiles_r);
            }
            int incl = nu;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int t = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += t;
            }
            if (v < A.n_virt) ucum[v] = base + incl - nu;
            base += __shfl_sync(0xffffffffu, incl, 31);
        }
        if (lane == 0) ucum[A.n_virt] = base;
    }
    __syncthreads();
    const int U = ucum[A.n_virt];
    // unit table: local unit i = global unit blockIdx.x + i * gridDim.x as
    // (virtual expert, tile, first permuted row, token count <= 8)
    const int n_local = U > (int)blockIdx.x ? (U - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;
    for (int i = tid; i < n_local; i += blockDim.x) {
        const int u = blockIdx.x + i * gridDim.x;
        int lo = 0, hi = A.n_virt - 1;               // last v with ucum[v] <= u
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (ucum[mid] <= u) lo = mid; else hi = mid - 1;
        }
        const Virt vi = virt(a, act, A.n_routed, lo);
        const int tv = vi.shared ? tiles_s : tiles_r;
        const int rem = u - ucum[lo], grp = rem / tv, tile = rem % tv;
        utab[i] = make_int4(lo, tile, vi.seg0 + grp * kGuCols, min(kGuCols, vi.cnt - grp * kGuCols));
    }
    __syncthreads();

    if (warp == kDW) {
        // ---------------------------------------------------- producer
        // per (unit, slice): one 16-row box of gate and one of up
        if (lane == 0) {
            const uint64_t pol = l2_evict_first_policy();    // weights: read once
            int stage = 0;
            uint32_t phase = 0;
            uint32_t used = 0u, last_ph = 0u;                 // per stage: issued, parity of its last fill
            bool ok = true;
            for (int i = 0; i < n_local && ok; i++) {
                const int v = utab[i].x, tile = utab[i].y;
                const Virt vi = virt(a, act, A.n_routed, v);
                const int bs = qt_unit_bytes(vi.qt);
                const GuGeo gg = vi.shared ? geoS : geoR;
                const CUtensorMap *mg = vi.shared ? &maps.sgate : &maps.gate;
                const CUtensorMap *mu = vi.shared ? &maps.sup : &maps.up;
                const int y = (vi.shared ? 0 : (int)vi.slot * a.F) + tile * kTile;
                for (int sl = 0; sl < gg.nsl; sl++) {
                    if (!mbar_wait(&empty[stage], phase ^ 1, a.err, kErrTimeoutEmpty)) { ok = false; break; }
                    uint8_t *dst = stages + (size_t)stage * stage_bytes;
                    mbar_arrive_expect_tx(&full[stage], (uint32_t)(2 * kTile * gg.pitch));
                    const int x = sl * gg.sb * bs / 8;
                    tma_load_2d_hint(dst, mg, x, y, &full[stage], pol);
                    tma_load_2d_hint(dst + kTile * gg.pitch, mu, x, y, &full[stage], pol);
                    used |= 1u << stage;
                    last_ph = (last_ph & ~(1u << stage)) | (phase << stage);
                    if (++stage == S) { stage = 0; phase ^= 1; }
                }
            }
            // drain: every copy this thread issued must have landed before the
            // CTA exits (also when a consumer gave up waiting)
            drain_fills(full, S, used, last_ph, a.err);
        }
        return;
    }

    if (warp > kDW) {
        // ----------------------------------------------------- epilogue
        // unit j: the 8 K-group partials of gate and of up summed in
        // K-group order, SwiGLU, the token's gate weight, Hs in fp16
        const int et = tid - kDThreads;
        for (int j = 0; j < n_local; j++) {
            const int b = j % NB;
            if (!mbar_wait_warp(&rfull[b], (uint32_t)((j / NB) & 1), a.err, kErrTimeoutFull)) return;
            const int4 ud = utab[j];
            const int tile = ud.y, seg0 = ud.z, cnt = ud.w;
            const float *redb = red + (size_t)b * kDW * NT * 128;
            for (int o = et; o < kTile * cnt; o += kEW * 32) {
                const int rr = o % kTile, n = o / kTile;
                const int nt = n >> 3, nn = n & 7;
                const int L = (rr & 7) * 4 + (nn >> 1);
                const int q = ((rr >> 3) << 1) | (nn & 1);
                float sg = 0.f, su = 0.f;
#pragma unroll
                for (int w = 0; w < 8; w++) {
                    sg += redb[((size_t)w * NT + nt) * 128 + L * 4 + q];
                    su += redb[((size_t)(8 + w) * NT + nt) * 128 + L * 4 + q];
                }
                const int pos = seg0 + n;
                const float h = silu(sg) * su * gw[pos];
                const int r = tile * kTile + rr;
                a.Hs[(size_t)pos * a.hrow + (r >> 5) * 32 + frag_slot(r & 31)] = __float2half_rn(h);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&rempty[b]);
        }
        return;
    }

    // ------------------------------------------------------ MMA warps
    const uint32_t xs_a = smem_u32(xs), sx_a = smem_u32(sxt), st_a = smem_u32(stages);
    int stage = 0;
    uint32_t phase = 0;
    bool ok = true;
    for (int j = 0; j < n_local && ok; j++) {
        const int4 ud = utab[j];
        const int tile = ud.y, seg0 = ud.z, cnt = ud.w;
        const bool shu = ud.x >= A.n_routed;
        const int qt = ONE >= 0 ? ONE : shu ? a.sqt : a.qt;
        const GuGeo gg = shu ? geoS : geoR;
        const int kb0 = kg * (qt == MOE_Q8_0 ? WB8 : WB4);   // warp's first block in a slice
        // B rows (column g, g+8) and C columns (2c, 2c+1, +8) of this unit
        uint32_t xa[NT], sa[NT][2];
        const uint32_t sxq = sx_a + (shu ? (uint32_t)((T + 1) * nbD * 4) : 0u);
#pragma unroll
        for (int nt = 0; nt < NT; nt++) {
            const int n = g + 8 * nt;
            const int tb = n < cnt ? tok[seg0 + n] : T;
            xa[nt] = xs_a + tb * xrow + kb0 * 64 + c * 16;
#pragma unroll
            for (int jj = 0; jj < 2; jj++) {
                const int m = 8 * nt + 2 * c + jj;
                const int tc = m < cnt ? tok[seg0 + m] : T;
                sa[nt][jj] = sxq + (uint32_t)((tc * nbD + kb0) * 4);
            }
        }
        float acc[NT][4];
#pragma unroll
        for (int nt = 0; nt < NT; nt++)
#pragma unroll
            for (int q = 0; q < 4; q++) acc[nt][q] = 0.f;
        const int bsz = qt_unit_bytes(qt);
        // byte offset of the warp's first unit in a staged row (Q6_K: block kb0 / 8)
        const int uoff = qt == MOE_Q6_K ? (kb0 >> 3) * MOE_Q6_K_BLOCK_BYTES : kb0 * bsz;
        const int mis0 = uoff & 3;                      // 0 or 2
        const uint32_t r8 = 8u * gg.pitch;

        for (int sl = 0; sl < gg.nsl; sl++) {
            if (!mbar_wait_warp(&full[stage], phase, a.err, kErrTimeoutFull)) { ok = false; break; }
            const uint32_t row = st_a + stage * stage_bytes + (mat * kTile + g) * gg.pitch + uoff;
            uint32_t xs_s[NT], sa_s[NT][2];
#pragma unroll
            for (int nt = 0; nt < NT; nt++) {
                xs_s[nt] = xa[nt] + sl * gg.sb * 64;
                sa_s[nt][0] = sa[nt][0] + sl * gg.sb * 4;
                sa_s[nt][1] = sa[nt][1] + sl * gg.sb * 4;
            }
#define MOE_GU(QT, MIS) gateup_slice<QT, 1, (QT == MOE_Q8_0 ? WB8 : WB4), MIS>(row, r8, xs_s, sa_s, c, acc)
            if (!ALL || qt == MOE_Q4_0 || qt == MOE_Q8_0) {
                // with an even number of blocks a warp, an 18-, 22- or 34-byte
                // block group always starts 4-byte aligned (mis0 == 0): the
                // other variant is compiled only where it can run
                if (qt == MOE_Q4_0) { if (WB4 % 2 == 0 || mis0 == 0) MOE_GU(MOE_Q4_0, 0); else MOE_GU(MOE_Q4_0, 2); }
                else { if (WB8 % 2 == 0 || mis0 == 0) MOE_GU(MOE_Q8_0, 0); else MOE_GU(MOE_Q8_0, 2); }
            } else if constexpr (ALL) {
                switch (qt) {
                case MOE_Q5_0: if (WB4 % 2 == 0 || mis0 == 0) MOE_GU(MOE_Q5_0, 0); else MOE_GU(MOE_Q5_0, 2); break;
                case MOE_Q4_1: MOE_GU(MOE_Q4_1, 0); break;      // 20-byte blocks: always aligned
                case MOE_Q5_1: MOE_GU(MOE_Q5_1, 0); break;      // 24-byte blocks: always aligned
                case MOE_Q6_K:                                   // one block a warp (WB4 == 8)
                    if constexpr (WB4 == 8) {
                        if (mis0 == 0) block_q6k<0, 1>(row, r8, xs_s, c, acc);
                        else block_q6k<2, 1>(row, r8, xs_s, c, acc);
                    }
                    break;
                default:                                         // Q4_K
                    gateup_slice_q4k<1, WB4>(row - kb0 * bsz, r8, kb0, xs_s, sa_s, c, acc);
                    break;
                }
            }
#undef MOE_GU
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[stage]);
            if (++stage == S) { stage = 0; phase ^= 1; }
        }
        if (!ok) break;
        // partials of unit j into buffer j % NB, once the epilogue of unit
        // j - NB has read that buffer
        const int b = j % NB;
        if (j >= NB && !mbar_wait_warp(&rempty[b], (uint32_t)((j / NB - 1) & 1), a.err, kErrTimeoutEmpty)) {
            ok = false;
            break;
        }
        float *rw = red + ((size_t)b * kDW + warp) * NT * 128;
#pragma unroll
        for (int nt = 0; nt < NT; nt++)
#pragma unroll
            for (int q = 0; q < 4; q++) rw[nt * 128 + lane * 4 + q] = acc[nt][q];
        __syncwarp();
        if (lane == 0) mbar_arrive(&rfull[b]);
    }
}

// --------------------------------------------------------------------- down
// Work unit = (expert, 64 rows of D): one 2-D box of the expert's down
// projection (64 rows x F/32 blocks, one TMA request of ~28 KB at F=768
// Q4_0) plus the expert's Hs rows, which are contiguous in permuted order
// (one bulk copy).  The 16 consumer warps form 4 groups of 4; group q takes
// every 4th unit of the CTA and warp m of a group one 16-row M-tile of it
// over the FULL reduction length, so no partial sums cross warps.  Each
// warp writes its Y rows (fp32, permuted order) to global memory; the
// combine is a separate, deterministic kernel.
constexpr int kDnRows = 64;

// 8 consecutive blocks of one 16-row tile for one warp; the block group
// starts 4-byte aligned (8 blocks of an even size).  For the _1 types the
// all-ones A of a second MMA pair sums each Hs column over the block, and m
// multiplies that sum.
template <int QT, int NTILE>
__device__ __forceinline__ void down_blocks8(uint32_t row, uint32_t r8, const uint32_t *ha, int c,
                                             float (*acc)[4]) {
    constexpr int BS = qt_bytes(QT);
    const uint32_t off2 = magic_off2<QT>();
    const float zero[4] = {0.f, 0.f, 0.f, 0.f};
    const uint32_t ones[4] = {0x3C003C00u, 0x3C003C00u, 0x3C003C00u, 0x3C003C00u};
#pragma unroll
    for (int bl = 0; bl < 8; bl++) {
        const uint32_t blk = row + bl * BS;
        uint32_t lo[4], hi[4];
        if (codes_mis<QT, 0>(bl) == 0) {
            magic_codes<QT, 0>(blk, c, lo);
            magic_codes<QT, 0>(blk + r8, c, hi);
        } else {
            magic_codes<QT, 2>(blk, c, lo);
            magic_codes<QT, 2>(blk + r8, c, hi);
        }
        const float dlo = h2f(lds16(blk)), dhi = h2f(lds16(blk + r8));
        float mlo = 0.f, mhi = 0.f;
        if constexpr (qt_has_min(QT)) {
            mlo = h2f(lds16(blk + 2));
            mhi = h2f(lds16(blk + r8 + 2));
        }
        const uint32_t a0[4] = {hsub2_u(lo[0], off2), hsub2_u(hi[0], off2), hsub2_u(lo[1], off2),
                                hsub2_u(hi[1], off2)};
        const uint32_t a1[4] = {hsub2_u(lo[2], off2), hsub2_u(hi[2], off2), hsub2_u(lo[3], off2),
                                hsub2_u(hi[3], off2)};
#pragma unroll
        for (int nt = 0; nt < NTILE; nt++) {
            const uint4 b = lds128(ha[nt] + bl * 64);
            float p[4];
            mma_16816(p, a0, b.x, b.y, zero);
            mma_16816(p, a1, b.z, b.w, p);
            acc[nt][0] = fmaf(dlo, p[0], acc[nt][0]);
            acc[nt][1] = fmaf(dlo, p[1], acc[nt][1]);
            acc[nt][2] = fmaf(dhi, p[2], acc[nt][2]);
            acc[nt][3] = fmaf(dhi, p[3], acc[nt][3]);
            if constexpr (qt_has_min(QT)) {
                float hs[4];
                mma_16816(hs, ones, b.x, b.y, zero);
                mma_16816(hs, ones, b.z, b.w, hs);
                acc[nt][0] = fmaf(mlo, hs[0], acc[nt][0]);
                acc[nt][1] = fmaf(mlo, hs[1], acc[nt][1]);
                acc[nt][2] = fmaf(mhi, hs[0], acc[nt][2]);
                acc[nt][3] = fmaf(mhi, hs[1], acc[nt][3]);
            }
        }
    }
}

// As down_blocks8 for Q4_K: the 8 units are one 144-byte block (blk).
template <int NTILE>
__device__ __forceinline__ void down_block_q4k(uint32_t blk, uint32_t r8, const uint32_t *ha, int c,
                                               float (*acc)[4]) {
    const uint32_t off2 = 0x64006400u;
    const float zero[4] = {0.f, 0.f, 0.f, 0.f};
    const uint32_t ones[4] = {0x3C003C00u, 0x3C003C00u, 0x3C003C00u, 0x3C003C00u};
    const Q4kHead hlo = q4k_head(blk), hhi = q4k_head(blk + r8);
#pragma unroll
    for (int j = 0; j < 8; j++) {
        uint32_t lo[4], hi[4];
        q4k_codes(blk, j, c, lo);
        q4k_codes(blk + r8, j, c, hi);
        float dlo, mlo, dhi, mhi;
        q4k_params(hlo, j, &dlo, &mlo);
        q4k_params(hhi, j, &dhi, &mhi);
        const uint32_t a0[4] = {hsub2_u(lo[0], off2), hsub2_u(hi[0], off2), hsub2_u(lo[1], off2),
                                hsub2_u(hi[1], off2)};
        const uint32_t a1[4] = {hsub2_u(lo[2], off2), hsub2_u(hi[2], off2), hsub2_u(lo[3], off2),
                                hsub2_u(hi[3], off2)};
#pragma unroll
        for (int nt = 0; nt < NTILE; nt++) {
            const uint4 b = lds128(ha[nt] + j * 64);
            float p[4], hs[4];
            mma_16816(p, a0, b.x, b.y, zero);
            mma_16816(p, a1, b.z, b.w, p);
            mma_16816(hs, ones, b.x, b.y, zero);
            mma_16816(hs, ones, b.z, b.w, hs);
            acc[nt][0] = fmaf(-mlo, hs[0], fmaf(dlo, p[0], acc[nt][0]));
            acc[nt][1] = fmaf(-mlo, hs[1], fmaf(dlo, p[1], acc[nt][1]));
            acc[nt][2] = fmaf(-mhi, hs[0], fmaf(dhi, p[2], acc[nt][2]));
            acc[nt][3] = fmaf(-mhi, hs[1], fmaf(dhi, p[3], acc[nt][3]));
        }
    }
}

// Local unit i of a CTA goes to consumer group i % G; the stage ring is
// split per group (G * Sg stages, group q owns stages q, q + G, ...), so a
// group only ever waits on stages it consumes itself and can never be two
// phases ahead of one of them.
struct DnSlot {
    int stage;
    uint32_t phase;
};
__device__ __forceinline__ DnSlot dn_slot(int i, int G, int Sg) {
    const int m = i / G;
    return {i % G + G * (m % Sg), (uint32_t)((m / Sg) & 1)};
}

// ALL: the call has a type other than Q4_0 and Q8_0 (a separate
// instantiation keeps the other types' code and registers out of the two
// types' kernel); ONE >= 0: every expert has block type ONE
template <int NT, bool ALL, int ONE = -1>
__global__ void __launch_bounds__(kDThreads, 1)
dec_down_kernel(DecArgs a, int G, int Sg, int hrows, const __grid_constant__ DecMaps maps) {
    extern __shared__ __align__(1024) uint8_t smem[];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g = lane >> 2, c = lane & 3;
    const int D = a.D;
    const int S = G * Sg;
    const int hbytes = a.hrow * 2;                      // staged Hs row = its global stride
    const int pr = dn_pitch(a.qt, a.F);
    const int ps = a.sF > 0 ? dn_pitch(a.sqt, a.sF) : 0;
    const int wbytes = kDnRows * (pr > ps ? pr : ps);
    const int stage_bytes = (int)round_up((size_t)wbytes + (size_t)hrows * hbytes, 128);
    const int grp = warp >> 2, mt = warp & 3;

    // carve (1024-aligned base: tensor copies need 128-byte destinations)
    uint8_t *stages = smem + ((1024u - (smem_u32(smem) & 1023u)) & 1023u);
    uint64_t *full = (uint64_t *)(stages + (size_t)S * stage_bytes);
    uint64_t *empty = full + kMaxStages;
    int *act = (int *)(empty + kMaxStages);
    int2 *ent = reinterpret_cast<int2 *>(act + 6 * (a.E + 1));     // (virtual expert, column group)

    if (tid == 0) {
        for (int s = 0; s < S; s++) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 4);             // the 4 warps of the owning group
        }
        fence_mbar_init();
    }
    // routing (perm/offsets) is complete: the gate/up kernel waited for it
    // before letting this grid launch
    const Active A = build_active_list(a, act);
    // entries: every virtual expert's tokens in column groups of <= 8
    // (one MMA N tile; at most 8 staged Hs rows a unit)
    int *ecum = act + 4 * (a.E + 1);                  // raw-table space, free now
    if (warp == 0) {
        int base = 0;
        for (int v0 = 0; v0 < A.n_virt; v0 += 32) {
            const int v = v0 + lane;
            const int ng = v < A.n_virt ? (virt(a, act, A.n_routed, v).cnt + kGuCols - 1) / kGuCols : 0;
            int incl = ng;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int t2 = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += t2;
            }
            if (v < A.n_virt) ecum[v] = base + incl - ng;
            base += __shfl_sync(0xffffffffu, incl, 31);
        }
        if (lane == 0) ecum[A.n_virt] = base;
    }
    __syncthreads();
    for (int v = tid; v < A.n_virt; v += blockDim.x)
        for (int q = ecum[v]; q < ecum[v + 1]; q++) ent[q] = make_int2(v, q - ecum[v]);
    __syncthreads();
    const int n_ent = ecum[A.n_virt];
    const int tiles = D / kDnRows;
    const int U = n_ent * tiles;
    // the rows of entry q: (first permuted row, count <= 8, shared, slot, type)
    auto entry = [&](int q, Virt *vi) {
        const int2 e2 = ent[q];
        *vi = virt(a, act, A.n_routed, e2.x);
        if (ONE >= 0) vi->qt = ONE;
        vi->seg0 += e2.y * kGuCols;
        vi->cnt = min(kGuCols, vi->cnt - e2.y * kGuCols);
    };

    if (warp == kDW) {
        if (lane == 0) {
            const uint64_t pol = l2_evict_first_policy();    // weights: read once
            bool ok = true, waited = false;
            uint32_t used = 0u, last_ph = 0u;
            int pend_s[kMaxStages], pend_v[kMaxStages];
            int npend = 0;
            auto issue_h = [&](int st, int q) {
                Virt vi;
                entry(q, &vi);
                bulk_g2s(stages + (size_t)st * stage_bytes + wbytes, a.Hs + (size_t)vi.seg0 * a.hrow,
                         (uint32_t)(vi.cnt * hbytes), &full[st]);
            };
            int i = 0;                          // local unit index
            for (int u = blockIdx.x; u < U && ok; u += gridDim.x, i++) {
                const int v = u / tiles, dt = u % tiles;    // v: entry
                const DnSlot sl = dn_slot(i, G, Sg);
                Virt vi;
                entry(v, &vi);
                const int pitch = vi.shared ? ps : pr;
                if (!mbar_wait(&empty[sl.stage], sl.phase ^ 1, a.err, kErrTimeoutEmpty)) { ok = false; break; }
                uint8_t *dst = stages + (size_t)sl.stage * stage_bytes;
                mbar_arrive_expect_tx(&full[sl.stage], (uint32_t)(kDnRows * pitch + vi.cnt * hbytes));
                const int y0 = (vi.shared ? 0 : (int)vi.slot * D) + dt * kDnRows;
                if (vi.qt == MOE_Q6_K)          // 8 whole 8-row groups, rows packed
                    tma_load_3d_hint(dst, vi.shared ? &maps.sdown : &maps.down, 0, 0, y0 / 8,
                                     &full[sl.stage], pol);
                else
                    tma_load_2d_hint(dst, vi.shared ? &maps.sdown : &maps.down, 0, y0, &full[sl.stage], pol);
                used |= 1u << sl.stage;
                last_ph = (last_ph & ~(1u << sl.stage)) | (sl.phase << sl.stage);
                if (waited) {
                    issue_h(sl.stage, v);
                } else {
                    pend_s[npend] = sl.stage; pend_v[npend] = v; npend++;
                    if (npend == S) {
                        // every stage holds prefetched weights: now wait for Hs
                        pdl_wait();
                        waited = true;
                        for (int q = 0; q < npend; q++) issue_h(pend_s[q], pend_v[q]);
                        npend = 0;
                    }
                }
            }
            if (!waited) {
                pdl_wait();
                for (int q = 0; q < npend; q++) issue_h(pend_s[q], pend_v[q]);
            }
            // drain: every copy issued (weights and Hs) must have landed
            drain_fills(full, S, used, last_ph, a.err);
        }
        return;
    }
    if (grp >= G) return;

    // ------------------------------------------------------- consumers
    const uint32_t st_a = smem_u32(stages);
    int i = grp;
    for (int u = blockIdx.x + grp * gridDim.x; u < U; u += G * gridDim.x, i += G) {
        const int v = u / tiles, dt = u % tiles;            // v: entry
        const DnSlot sl = dn_slot(i, G, Sg);
        Virt vi;
        entry(v, &vi);
        const int bsz = qt_unit_bytes(vi.qt);
        const int pitch = vi.shared ? ps : pr;
        const int nb = vi.Fv / QK;
        const int ntile = vi.cnt > 8 ? 2 : 1;
        // Q6_K rows are packed at an even pitch that may be 2 mod 4: warp mt
        // takes the rows of one parity, 2i + (mt & 1) + 32 (mt >> 1) for tile
        // row i, so that a block's alignment is the same in all its rows
        const bool q6 = ALL && vi.qt == MOE_Q6_K;
        const int mrow = q6 ? 32 * (mt >> 1) + (mt & 1) : mt * kTile;   // tile row 0
        const int mstep = q6 ? 2 : 1;                                      // rows per tile row
        float acc[NT][4];
#pragma unroll
        for (int nt = 0; nt < NT; nt++)
#pragma unroll
            for (int q = 0; q < 4; q++) acc[nt][q] = 0.f;
        if (!mbar_wait_warp(&full[sl.stage], sl.phase, a.err, kErrTimeoutFull)) break;
        const uint32_t sbase = st_a + sl.stage * stage_bytes;
        uint32_t row = sbase + (mrow + mstep * g) * pitch;
        const uint32_t r8 = 8u * mstep * pitch;
        uint32_t ha[NT];
#pragma unroll
        for (int nt = 0; nt < NT; nt++) {
            const int n = g + 8 * nt;
            // columns past the expert's token count read whatever the stage
            // holds there; an MMA column depends only on its own B column,
            // and those columns are never stored
            ha[nt] = sbase + wbytes + (n < hrows ? n : 0) * hbytes + c * 16;
        }
        if (q6) {
            if constexpr (ALL) {
                // block b starts (row parity * pitch + 210 b) mod 4 bytes off
                const int nblk = nb / 8;
                const bool mis0 = ((mt & 1) * pitch) & 3;
                for (int b = 0; b < nblk; b += 2) {
                    const uint32_t blk = row + b * MOE_Q6_K_BLOCK_BYTES;
                    if (!mis0) block_q6k<0, 1>(blk, r8, ha, c, acc);
                    else block_q6k<2, 1>(blk, r8, ha, c, acc);
                    if (b + 1 < nblk) {
                        uint32_t hb[1] = {ha[0] + 8 * 64};
                        if (!mis0) block_q6k<2, 1>(blk + MOE_Q6_K_BLOCK_BYTES, r8, hb, c, acc);
                        else block_q6k<0, 1>(blk + MOE_Q6_K_BLOCK_BYTES, r8, hb, c, acc);
                    }
                    ha[0] += 16 * 64;
                }
            }
        } else
        for (int kb = 0; kb < nb; kb += 8) {
#define MOE_DN(QT)                                                     \
    case QT:                                                           \
        if (ntile == 1) down_blocks8<QT, 1>(row, r8, ha, c, acc);      \
        else if (NT > 1) down_blocks8<QT, NT>(row, r8, ha, c, acc);    \
        break;
            if (!ALL || vi.qt == MOE_Q4_0 || vi.qt == MOE_Q8_0) {
                switch (vi.qt) {
                    MOE_DN(MOE_Q4_0)
                    default:
                        if (ntile == 1) down_blocks8<MOE_Q8_0, 1>(row, r8, ha, c, acc);
                        else if (NT > 1) down_blocks8<MOE_Q8_0, NT>(row, r8, ha, c, acc);
                }
            } else if constexpr (ALL) {
                switch (vi.qt) {
                    MOE_DN(MOE_Q4_1)
                    MOE_DN(MOE_Q5_0)
                    MOE_DN(MOE_Q5_1)
                    default:                                 // Q4_K
                        if (ntile == 1) down_block_q4k<1>(row, r8, ha, c, acc);
                        else if (NT > 1) down_block_q4k<NT>(row, r8, ha, c, acc);
                }
            }
#undef MOE_DN
            row += 8 * bsz;
#pragma unroll
            for (int nt = 0; nt < NT; nt++) ha[nt] += 8 * 64;
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[sl.stage]);
        // C fragment: tile rows g / g+8, columns 2c, 2c+1 (+8 nt)
        float *out = a.rows_out + (size_t)vi.seg0 * D + dt * kDnRows + mrow;
#pragma unroll
        for (int nt = 0; nt < NT; nt++)
#pragma unroll
            for (int q = 0; q < 4; q++) {
                const int n = nt * 8 + 2 * c + (q & 1);
                const int r = mstep * (g + ((q >> 1) << 3));
                if (n < vi.cnt) out[(size_t)n * D + r] = acc[nt][q];
            }
    }
}

// ------------------------------------------------------ 8-bit activations
// The W4A8 / W8A8 mode (FreeToken fork README, the note on CUDA W4A8 MMVQ):
// the inputs of every expert matmul are 8-bit blocks of 32 (per block, in
// fp32: d = max|v| / 127, q = round-half-away(v * (1 / d))), and int8 tensor-
// core products (mma.sync m16n8k32, int32 accumulate) are scaled by the
// weight block's d and the activation block's d.  Q8_0 codes are the A
// fragment as they lie in shared memory; Q4_0 nibbles become unsigned bytes
// with two masks, the -8 offset entering through the accumulator input as
// -8 * (sum of the activation codes).  Gate/up units hold 32 rows of F (one
// h block), so the epilogue quantizes h in place; the down kernel scales its
// rows by the gate weight (h is quantized without it).
struct A8Args {
    DecArgs d;
    int8_t *hq;          // [T*k + T][hq_row] h codes, permuted order (+ shared rows)
    float2 *hs;          // [T*k + T][hq_row / 32] (scale, sum of the codes) per h block
    int hq_row;          // bytes per hq row = max(F, shared F)
};
struct A8Maps {
    DecMaps m;           // gate/up: boxes of 32 rows; down: boxes of 64 rows
    CUtensorMap hq;      // h codes: boxes of hrows rows x a padded row
};
constexpr int kA8Rows = 32;
constexpr int kA8MaxSb = 32;                     // blocks per K-slice
__host__ __device__ inline int a8_xrow(int D) { return D + 16; }   // staged x-code row

// 32 activations of token t, block b (bf16 or fp32, as the 16-bit path reads them)
__device__ __forceinline__ void a8_load_block(const DecArgs &a, int t, int b, float *v) {
    const size_t xb = (size_t)t * a.D + (size_t)b * QK;
    if (a.x_vec && a.x_bf16) {
        const uint4 *p = reinterpret_cast<const uint4 *>((const __nv_bfloat16 *)a.x + xb);
        uint4 w[4];
#pragma unroll
        for (int q = 0; q < 4; q++) w[q] = __ldg(p + q);
#pragma unroll
        for (int q = 0; q < 4; q++) {
            const uint32_t u[4] = {w[q].x, w[q].y, w[q].z, w[q].w};
#pragma unroll
            for (int r = 0; r < 4; r++) {
                v[8 * q + 2 * r] = __uint_as_float(u[r] << 16);
                v[8 * q + 2 * r + 1] = __uint_as_float(u[r] & 0xFFFF0000u);
            }
        }
    } else if (a.x_vec) {
        const float4 *p = reinterpret_cast<const float4 *>((const float *)a.x + xb);
#pragma unroll
        for (int q = 0; q < 8; q++) {
            const float4 w = __ldg(p + q);
            v[4 * q] = w.x; v[4 * q + 1] = w.y; v[4 * q + 2] = w.z; v[4 * q + 3] = w.w;
        }
    } else {
#pragma unroll
        for (int i = 0; i < 32; i++)
            v[i] = a.x_bf16 ? load_act((const __nv_bfloat16 *)a.x, xb + i)
                            : load_act((const float *)a.x, xb + i);
    }
}

// 8-bit code of v with block scale reciprocal id (round half away from zero)
__device__ __forceinline__ int a8_code(float v, float id) { return (int)roundf(v * id); }

// A fragment of a Q8_0 / Q4_0 block for rows g (blk_lo) and g+8 (blk_hi);
// MIS: alignment mod 4 of the block's codes
template <bool Q8, int MIS>
__device__ __forceinline__ void a8_weight_frag(uint32_t blk_lo, uint32_t blk_hi, int c, uint32_t *a) {
    const uint32_t o = 2 + 4 * c;
    if constexpr (Q8) {
        a[0] = lds_word<MIS>(blk_lo + o);
        a[1] = lds_word<MIS>(blk_hi + o);
        a[2] = lds_word<MIS>(blk_lo + o + 16);
        a[3] = lds_word<MIS>(blk_hi + o + 16);
    } else {
        const uint32_t wl = lds_word<MIS>(blk_lo + o), wh = lds_word<MIS>(blk_hi + o);
        a[0] = wl & 0x0F0F0F0Fu;
        a[2] = (wl >> 4) & 0x0F0F0F0Fu;
        a[1] = wh & 0x0F0F0F0Fu;
        a[3] = (wh >> 4) & 0x0F0F0F0Fu;
    }
}

// One K-slice of the 32-row unit for one warp: WB blocks from the warp's
// first block; row: staged row g at that block (tile 0); xb: column g's x
// codes at that block + 4c; dx0/dx1, s0/s1: column 2c / 2c+1's block scales
// and code sums at that block.
template <bool Q8, int WB, int MIS0>
__device__ __forceinline__ void gateup_slice_a8(uint32_t row, uint32_t r8, uint32_t r16, uint32_t xb,
                                                uint32_t dx0a, uint32_t dx1a, uint32_t s0a, uint32_t s1a,
                                                int c, float (*acc)[4]) {
    constexpr int BS = Q8 ? kQ8Bytes : kQ4Bytes;
#pragma unroll
    for (int bl = 0; bl < WB; bl++) {
        const uint32_t blk = row + bl * BS;
        const uint32_t b0 = lds32(xb + bl * 32), b1 = lds32(xb + bl * 32 + 16);
        const float dx0 = ldsf(dx0a + bl * 4), dx1 = ldsf(dx1a + bl * 4);
        int ci[4] = {0, 0, 0, 0};
        if constexpr (!Q8) {
            const int c0 = -8 * (int)lds32(s0a + bl * 4), c1 = -8 * (int)lds32(s1a + bl * 4);
            ci[0] = c0; ci[1] = c1; ci[2] = c0; ci[3] = c1;
        }
#pragma unroll
        for (int tt = 0; tt < 2; tt++) {
            const uint32_t bt = blk + tt * r16;
            uint32_t af[4];
            if (((MIS0 + bl * BS + 2) & 3) == 0) a8_weight_frag<Q8, 0>(bt, bt + r8, c, af);
            else a8_weight_frag<Q8, 2>(bt, bt + r8, c, af);
            const float dlo = h2f(lds16(bt)), dhi = h2f(lds16(bt + r8));
            int p[4];
            if constexpr (Q8) imma_s8s8(p, af, b0, b1, ci);
            else imma_u8s8(p, af, b0, b1, ci);
            acc[tt][0] = fmaf(dlo * dx0, (float)p[0], acc[tt][0]);
            acc[tt][1] = fmaf(dlo * dx1, (float)p[1], acc[tt][1]);
            acc[tt][2] = fmaf(dhi * dx0, (float)p[2], acc[tt][2]);
            acc[tt][3] = fmaf(dhi * dx1, (float)p[3], acc[tt][3]);
        }
    }
}

template <int WB>
__global__ void __launch_bounds__(kGThreads, 1)
dec_gateup_a8_kernel(A8Args A, int S, const __grid_constant__ A8Maps maps) {
    const DecArgs &a = A.d;
    extern __shared__ __align__(1024) uint8_t smem[];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g = lane >> 2, c = lane & 3;
    const int T = a.T, D = a.D;
    const int nbD = D / QK;
    const GuGeo geoR = gu_geo(D, a.qt, kA8MaxSb), geoS = gu_geo(D, a.sqt, kA8MaxSb);
    const int pitch_max = max(geoR.pitch, a.sF > 0 ? geoS.pitch : 0);
    const int stage_bytes = (int)round_up((size_t)2 * kA8Rows * pitch_max, 128);
    const int xrow = a8_xrow(D);
    const int mat = warp >> 3, kg = warp & 7;

    // carve (1024-aligned base): x codes [T+1 rows, the last zero] | scales
    // [T+1][nbD] | code sums [T+1][nbD] | stages | red [NB][kDW][2][32][4] |
    // barriers | act | tok | units
    uint8_t *base = smem + ((1024u - (smem_u32(smem) & 1023u)) & 1023u);
    const size_t xs_bytes = round_up((size_t)(T + 1) * xrow, 16);
    uint8_t *xs = base;
    float *dxt = (float *)(base + xs_bytes);
    int *sqt = (int *)(dxt + (size_t)(T + 1) * nbD);
    uint8_t *stages = base + round_up(xs_bytes + (size_t)2 * (T + 1) * nbD * 4, 1024);
    constexpr int NB = kGuRedBufs;
    float *red = (float *)(stages + (size_t)S * stage_bytes);
    uint64_t *full = (uint64_t *)(red + NB * kDW * 2 * 32 * 4);
    uint64_t *empty = full + kMaxStages;
    uint64_t *rfull = empty + kMaxStages;
    uint64_t *rempty = rfull + 4;
    int *act = (int *)(rempty + 4);
    int *tok = act + 6 * (a.E + 1);
    int4 *utab = reinterpret_cast<int4 *>(
        (reinterpret_cast<uintptr_t>(tok + kMaxTk + 16 + kMaxTk + 16) + 15) & ~(uintptr_t)15);

    if (tid == 0) {
        for (int s = 0; s < S; s++) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kDW);
        }
        for (int b = 0; b < NB; b++) {
            mbar_init(&rfull[b], kDW);
            mbar_init(&rempty[b], kEW);
        }
        fence_mbar_init();
    }
    // x -> 8-bit codes, one (token, block) per thread (row T: zero codes),
    // before waiting for the routing kernel this grid may overlap with
    for (int idx = tid; idx < (T + 1) * nbD; idx += kGThreads) {
        const int t = idx / nbD, b = idx % nbD;
        float v[32];
        if (t < T) {
            a8_load_block(a, t, b, v);
        } else {
#pragma unroll
            for (int i = 0; i < 32; i++) v[i] = 0.f;
        }
        float amax = 0.f;
#pragma unroll
        for (int i = 0; i < 32; i++) amax = fmaxf(amax, fabsf(v[i]));
        const float dx = amax / 127.f;
        const float id = dx != 0.f ? 1.f / dx : 0.f;
        uint32_t w[8];
        int sum = 0;
#pragma unroll
        for (int q = 0; q < 8; q++) {
            uint32_t word = 0;
#pragma unroll
            for (int r = 0; r < 4; r++) {
                const int code = a8_code(v[4 * q + r], id);
                sum += code;
                word |= ((uint32_t)code & 0xFFu) << (8 * r);
            }
            w[q] = word;
        }
        uint4 *dst = reinterpret_cast<uint4 *>(xs + (size_t)t * xrow + b * 32);
        dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
        dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
        dxt[idx] = dx;
        sqt[idx] = sum;
    }
    __syncthreads();
    pdl_wait();
    pdl_launch_dependents();
    load_token_tables(a, tok, nullptr);
    const Active Av = build_active_list(a, act);   // includes __syncthreads
    const int tiles_r = a.F / kA8Rows, tiles_s = a.sF / kA8Rows;
    int *ucum = act + 4 * (a.E + 1);
    if (warp == 0) {
        int base_u = 0;
        for (int v0 = 0; v0 < Av.n_virt; v0 += 32) {
            const int v = v0 + lane;
            int nu = 0;
            if (v < Av.n_virt) {
                const Virt vi = virt(a, act, Av.n_routed, v);
                nu = (vi.cnt + kGuCols - 1) / kGuCols * (vi.shared ? tiles_s : tiles_r);
            }
            int incl = nu;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int t2 = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += t2;
            }
            if (v < Av.n_virt) ucum[v] = base_u + incl - nu;
            base_u += __shfl_sync(0xffffffffu, incl, 31);
        }
        if (lane == 0) ucum[Av.n_virt] = base_u;
    }
    __syncthreads();
    const int U = ucum[Av.n_virt];
    const int n_local = U > (int)blockIdx.x ? (U - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;
    for (int i = tid; i < n_local; i += blockDim.x) {
        const int u = blockIdx.x + i * gridDim.x;
        int lo = 0, hi = Av.n_virt - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (ucum[mid] <= u) lo = mid; else hi = mid - 1;
        }
        const Virt vi = virt(a, act, Av.n_routed, lo);
        const int tv = vi.shared ? tiles_s : tiles_r;
        const int rem = u - ucum[lo], grp = rem / tv, tile = rem % tv;
        utab[i] = make_int4(lo, tile, vi.seg0 + grp * kGuCols, min(kGuCols, vi.cnt - grp * kGuCols));
    }
    __syncthreads();

    if (warp == kDW) {
        // ---------------------------------------------------- producer
        if (lane == 0) {
            const uint64_t pol = l2_evict_first_policy();
            int stage = 0;
            uint32_t phase = 0, used = 0u, last_ph = 0u;
            bool ok = true;
            for (int i = 0; i < n_local && ok; i++) {
                const int v = utab[i].x, tile = utab[i].y;
                const Virt vi = virt(a, act, Av.n_routed, v);
                const int bs = qt_bytes(vi.qt);
                const GuGeo gg = vi.shared ? geoS : geoR;
                const CUtensorMap *mg = vi.shared ? &maps.m.sgate : &maps.m.gate;
                const CUtensorMap *mu = vi.shared ? &maps.m.sup : &maps.m.up;
                const int y = (vi.shared ? 0 : (int)vi.slot * a.F) + tile * kA8Rows;
                for (int sl = 0; sl < gg.nsl; sl++) {
                    if (!mbar_wait(&empty[stage], phase ^ 1, a.err, kErrTimeoutEmpty)) { ok = false; break; }
                    uint8_t *dst = stages + (size_t)stage * stage_bytes;
                    mbar_arrive_expect_tx(&full[stage], (uint32_t)(2 * kA8Rows * gg.pitch));
                    const int x = sl * gg.sb * bs / 8;
                    tma_load_2d_hint(dst, mg, x, y, &full[stage], pol);
                    tma_load_2d_hint(dst + kA8Rows * gg.pitch, mu, x, y, &full[stage], pol);
                    used |= 1u << stage;
                    last_ph = (last_ph & ~(1u << stage)) | (phase << stage);
                    if (++stage == S) { stage = 0; phase ^= 1; }
                }
            }
            drain_fills(full, S, used, last_ph, a.err);
        }
        return;
    }

    if (warp > kDW) {
        // ----------------------------------------------------- epilogue
        // unit j: thread (column n = et / 8, row group rg = et % 8) sums the
        // K-group partials of rows 4rg..4rg+3, forms h, and quantizes the
        // column's 32 h values with the 8 threads of its column
        const int et = tid - kDThreads;
        const int n = et >> 3, rg = et & 7;
        for (int j = 0; j < n_local; j++) {
            const int b = j % NB;
            if (!mbar_wait_warp(&rfull[b], (uint32_t)((j / NB) & 1), a.err, kErrTimeoutFull)) return;
            const int4 ud = utab[j];
            const int tile = ud.y, seg0 = ud.z, cnt = ud.w;
            const float *redb = red + (size_t)b * kDW * 2 * 128;
            float h[4];
            float m = 0.f;
#pragma unroll
            for (int r = 0; r < 4; r++) {
                const int row = 4 * rg + r, tt = row >> 4, rr = row & 15;
                const int L = (rr & 7) * 4 + (n >> 1);
                const int q = ((rr >> 3) << 1) | (n & 1);
                float sg = 0.f, su = 0.f;
#pragma unroll
                for (int w = 0; w < 8; w++) {
                    sg += redb[((size_t)w * 2 + tt) * 128 + L * 4 + q];
                    su += redb[((size_t)(8 + w) * 2 + tt) * 128 + L * 4 + q];
                }
                h[r] = silu(sg) * su;
                m = fmaxf(m, fabsf(h[r]));
            }
#pragma unroll
            for (int o = 1; o < 8; o <<= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
            const float dh = m / 127.f;
            const float id = dh != 0.f ? 1.f / dh : 0.f;
            uint32_t word = 0;
            int sum = 0;
#pragma unroll
            for (int r = 0; r < 4; r++) {
                const int code = a8_code(h[r], id);
                sum += code;
                word |= ((uint32_t)code & 0xFFu) << (8 * r);
            }
#pragma unroll
            for (int o = 1; o < 8; o <<= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
            if (n < cnt) {
                const int pos = seg0 + n;
                *reinterpret_cast<uint32_t *>(A.hq + (size_t)pos * A.hq_row + tile * kA8Rows + 4 * rg) = word;
                if (rg == 0) A.hs[(size_t)pos * (A.hq_row / QK) + tile] = make_float2(dh, (float)sum);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&rempty[b]);
        }
        return;
    }

    // ------------------------------------------------------ MMA warps
    const uint32_t xs_a = smem_u32(xs), dx_a = smem_u32(dxt), sq_a = smem_u32(sqt);
    const uint32_t st_a = smem_u32(stages);
    int stage = 0;
    uint32_t phase = 0;
    bool ok = true;
    for (int j = 0; j < n_local && ok; j++) {
        const int4 ud = utab[j];
        const int seg0 = ud.z, cnt = ud.w;
        const bool shu = ud.x >= Av.n_routed;
        const bool q8 = (shu ? a.sqt : a.qt) == MOE_Q8_0;
        const GuGeo gg = shu ? geoS : geoR;
        const int kb0 = kg * WB;
        const int tb = g < cnt ? tok[seg0 + g] : T;
        const int t0 = 2 * c < cnt ? tok[seg0 + 2 * c] : T;
        const int t1 = 2 * c + 1 < cnt ? tok[seg0 + 2 * c + 1] : T;
        const uint32_t xb = xs_a + tb * xrow + kb0 * 32 + c * 4;
        float acc[2][4];
#pragma unroll
        for (int tt = 0; tt < 2; tt++)
#pragma unroll
            for (int q = 0; q < 4; q++) acc[tt][q] = 0.f;
        const int bsz = q8 ? kQ8Bytes : kQ4Bytes;
        const int mis0 = (kb0 * bsz) & 3;
        const uint32_t r8 = 8u * gg.pitch, r16 = 16u * gg.pitch;
        for (int sl = 0; sl < gg.nsl; sl++) {
            if (!mbar_wait_warp(&full[stage], phase, a.err, kErrTimeoutFull)) { ok = false; break; }
            const uint32_t row = st_a + stage * stage_bytes + (mat * kA8Rows + g) * gg.pitch + kb0 * bsz;
            const int kb = sl * gg.sb + kb0;              // first block of this warp in the row
            const uint32_t xbs = xb + sl * gg.sb * 32;
            const uint32_t d0 = dx_a + (uint32_t)((t0 * nbD + kb) * 4), d1 = dx_a + (uint32_t)((t1 * nbD + kb) * 4);
            const uint32_t s0 = sq_a + (uint32_t)((t0 * nbD + kb) * 4), s1 = sq_a + (uint32_t)((t1 * nbD + kb) * 4);
            if (q8) {
                if (mis0 == 0) gateup_slice_a8<true, WB, 0>(row, r8, r16, xbs, d0, d1, s0, s1, c, acc);
                else gateup_slice_a8<true, WB, 2>(row, r8, r16, xbs, d0, d1, s0, s1, c, acc);
            } else {
                if (mis0 == 0) gateup_slice_a8<false, WB, 0>(row, r8, r16, xbs, d0, d1, s0, s1, c, acc);
                else gateup_slice_a8<false, WB, 2>(row, r8, r16, xbs, d0, d1, s0, s1, c, acc);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[stage]);
            if (++stage == S) { stage = 0; phase ^= 1; }
        }
        if (!ok) break;
        const int b = j % NB;
        if (j >= NB && !mbar_wait_warp(&rempty[b], (uint32_t)((j / NB - 1) & 1), a.err, kErrTimeoutEmpty)) {
            ok = false;
            break;
        }
        float *rw = red + ((size_t)b * kDW + warp) * 2 * 128;
#pragma unroll
        for (int tt = 0; tt < 2; tt++)
#pragma unroll
            for (int q = 0; q < 4; q++) rw[tt * 128 + lane * 4 + q] = acc[tt][q];
        __syncwarp();
        if (lane == 0) mbar_arrive(&rfull[b]);
    }
}

// Down with 8-bit h: unit = (expert, 64 rows of D) as the 16-bit kernel; the
// stage holds the 64-row weight box, the expert's h-code rows (one box of
// hrows rows, padded so that the B loads of 8 columns hit distinct banks)
// and their (scale, code sum) pairs.
template <int NT>
__global__ void __launch_bounds__(kDThreads, 1)
dec_down_a8_kernel(A8Args A, int G, int Sg, int hrows, int hpitch, const __grid_constant__ A8Maps maps) {
    const DecArgs &a = A.d;
    extern __shared__ __align__(1024) uint8_t smem[];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g = lane >> 2, c = lane & 3;
    const int D = a.D;
    const int S = G * Sg;
    const int hsrow = A.hq_row / QK * 8;                 // bytes of one row of (scale, sum) pairs
    const int pr = tma_row_bytes((int)qt_row_bytes(a.qt, a.F));
    const int ps = a.sF > 0 ? tma_row_bytes((int)qt_row_bytes(a.sqt, a.sF)) : 0;
    const int wbytes = kDnRows * (pr > ps ? pr : ps);
    const int hbytes = (int)round_up((size_t)hrows * hpitch, 128);
    const int stage_bytes = (int)round_up((size_t)wbytes + hbytes + (size_t)hrows * hsrow, 128);
    const int grp = warp >> 2, mt = warp & 3;

    uint8_t *stages = smem + ((1024u - (smem_u32(smem) & 1023u)) & 1023u);
    uint64_t *full = (uint64_t *)(stages + (size_t)S * stage_bytes);
    uint64_t *empty = full + kMaxStages;
    int *act = (int *)(empty + kMaxStages);

    if (tid == 0) {
        for (int s = 0; s < S; s++) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 4);
        }
        fence_mbar_init();
    }
    const Active Av = build_active_list(a, act);
    const int tiles = D / kDnRows;
    const int U = Av.n_virt * tiles;

    if (warp == kDW) {
        if (lane == 0) {
            const uint64_t pol = l2_evict_first_policy();
            bool ok = true, waited = false;
            uint32_t used = 0u, last_ph = 0u;
            int pend_s[kMaxStages], pend_v[kMaxStages];
            int npend = 0;
            auto issue_h = [&](int st, int v) {
                const Virt vi = virt(a, act, Av.n_routed, v);
                uint8_t *dst = stages + (size_t)st * stage_bytes + wbytes;
                tma_load_2d(dst, &maps.hq, 0, vi.seg0, &full[st]);
                bulk_g2s(dst + hbytes, A.hs + (size_t)vi.seg0 * (A.hq_row / QK),
                         (uint32_t)(vi.cnt * hsrow), &full[st]);
            };
            int i = 0;
            for (int u = blockIdx.x; u < U && ok; u += gridDim.x, i++) {
                const int v = u / tiles, dt = u % tiles;
                const DnSlot sl = dn_slot(i, G, Sg);
                const Virt vi = virt(a, act, Av.n_routed, v);
                const int pitch = vi.shared ? ps : pr;
                if (!mbar_wait(&empty[sl.stage], sl.phase ^ 1, a.err, kErrTimeoutEmpty)) { ok = false; break; }
                uint8_t *dst = stages + (size_t)sl.stage * stage_bytes;
                mbar_arrive_expect_tx(&full[sl.stage],
                                      (uint32_t)(kDnRows * pitch + hrows * hpitch + vi.cnt * hsrow));
                tma_load_2d_hint(dst, vi.shared ? &maps.m.sdown : &maps.m.down, 0,
                                 (vi.shared ? 0 : (int)vi.slot * D) + dt * kDnRows, &full[sl.stage], pol);
                used |= 1u << sl.stage;
                last_ph = (last_ph & ~(1u << sl.stage)) | (sl.phase << sl.stage);
                if (waited) {
                    issue_h(sl.stage, v);
                } else {
                    pend_s[npend] = sl.stage; pend_v[npend] = v; npend++;
                    if (npend == S) {
                        pdl_wait();
                        waited = true;
                        for (int q = 0; q < npend; q++) issue_h(pend_s[q], pend_v[q]);
                        npend = 0;
                    }
                }
            }
            if (!waited) {
                pdl_wait();
                for (int q = 0; q < npend; q++) issue_h(pend_s[q], pend_v[q]);
            }
            drain_fills(full, S, used, last_ph, a.err);
        }
        return;
    }
    if (grp >= G) return;

    const uint32_t st_a = smem_u32(stages);
    int i = grp;
    for (int u = blockIdx.x + grp * gridDim.x; u < U; u += G * gridDim.x, i += G) {
        const int v = u / tiles, dt = u % tiles;
        const DnSlot sl = dn_slot(i, G, Sg);
        const Virt vi = virt(a, act, Av.n_routed, v);
        const bool q8 = vi.qt == MOE_Q8_0;
        const int bsz = q8 ? kQ8Bytes : kQ4Bytes;
        const int pitch = vi.shared ? ps : pr;
        const int nb = vi.Fv / QK;
        float acc[NT][4];
#pragma unroll
        for (int nt = 0; nt < NT; nt++)
#pragma unroll
            for (int q = 0; q < 4; q++) acc[nt][q] = 0.f;
        if (!mbar_wait_warp(&full[sl.stage], sl.phase, a.err, kErrTimeoutFull)) break;
        const uint32_t sbase = st_a + sl.stage * stage_bytes;
        const uint32_t row = sbase + (mt * kTile + g) * pitch;
        const uint32_t r8 = 8u * pitch;
        const uint32_t hq_s = sbase + wbytes;
        const float2 *hs_s = reinterpret_cast<const float2 *>(stages + (size_t)sl.stage * stage_bytes +
                                                              wbytes + hbytes);
        const int hs2 = hsrow / 8;                        // pairs per row
        uint32_t hb[NT];
        const float2 *sc0[NT], *sc1[NT];
#pragma unroll
        for (int nt = 0; nt < NT; nt++) {
            const int n = g + 8 * nt, n0 = 8 * nt + 2 * c, n1 = n0 + 1;
            // columns past the expert's rows read whatever the stage holds
            // there; a column depends only on its own B column and its own
            // scale, and those columns are never stored
            hb[nt] = hq_s + (n < hrows ? n : 0) * hpitch + c * 4;
            sc0[nt] = hs_s + (n0 < hrows ? n0 : 0) * hs2;
            sc1[nt] = hs_s + (n1 < hrows ? n1 : 0) * hs2;
        }
        const int ntile = vi.cnt > 8 ? 2 : 1;
        for (int b = 0; b < nb; b++) {
            const uint32_t blk = row + b * bsz;
            const int mis = (b * bsz + 2) & 3;
            uint32_t af[4];
            if (q8) { if (mis == 0) a8_weight_frag<true, 0>(blk, blk + r8, c, af); else a8_weight_frag<true, 2>(blk, blk + r8, c, af); }
            else { if (mis == 0) a8_weight_frag<false, 0>(blk, blk + r8, c, af); else a8_weight_frag<false, 2>(blk, blk + r8, c, af); }
            const float dlo = h2f(lds16(blk)), dhi = h2f(lds16(blk + r8));
#pragma unroll
            for (int nt = 0; nt < NT; nt++) {
                if (nt >= ntile) break;
                const uint32_t b0 = lds32(hb[nt] + b * 32), b1 = lds32(hb[nt] + b * 32 + 16);
                const float2 h0 = sc0[nt][b], h1 = sc1[nt][b];
                int ci[4] = {0, 0, 0, 0};
                if (!q8) {
                    const int c0 = -8 * (int)h0.y, c1 = -8 * (int)h1.y;
                    ci[0] = c0; ci[1] = c1; ci[2] = c0; ci[3] = c1;
                }
                int p[4];
                if (q8) imma_s8s8(p, af, b0, b1, ci);
                else imma_u8s8(p, af, b0, b1, ci);
                acc[nt][0] = fmaf(dlo * h0.x, (float)p[0], acc[nt][0]);
                acc[nt][1] = fmaf(dlo * h1.x, (float)p[1], acc[nt][1]);
                acc[nt][2] = fmaf(dhi * h0.x, (float)p[2], acc[nt][2]);
                acc[nt][3] = fmaf(dhi * h1.x, (float)p[3], acc[nt][3]);
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[sl.stage]);
        // the gate weight of each column (1 for the shared expert's rows)
        float* out = a.rows_out + (size_t)vi.seg0 * D + dt * kDnRows + mt * kTile;
#pragma unroll
        for (int nt = 0; nt < NT; nt++)
#pragma unroll
            for (int q = 0; q < 4; q++) {
                const int n = nt * 8 + 2 * c + (q & 1);
                const int r = g + ((q >> 1) << 3);
                if (n < vi.cnt) {
                    const float gw = (vi.shared || !a.gates) ? 1.f : __ldg(a.gates + __ldg(a.perm + vi.seg0 + n));
                    out[(size_t)n * D + r] = acc[nt][q] * gw;
                }
            }
    }
}

// y[t, :] = sum_j rows[inv[t*k + j], :] (+ rows[T*k + t, :] for the shared
// expert), in j order; rows already carry the gate weight.
__global__ void __launch_bounds__(256)
dec_combine_kernel(const float *__restrict__ rows, const int32_t *__restrict__ inv, int T, int k,
                   int D, int shared, void *__restrict__ y, int y_dtype) {
    pdl_wait();
    const int t = blockIdx.x;
    const int d0 = (blockIdx.y * blockDim.x + threadIdx.x) * 4;
    if (d0 >= D) return;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int j = 0; j < k; j++) {
        const float4 r = __ldg(reinterpret_cast<const float4 *>(rows + (size_t)__ldg(inv + (size_t)t * k + j) * D + d0));
        acc.x += r.x; acc.y += r.y; acc.z += r.z; acc.w += r.w;
    }
    if (shared) {
        const float4 r = __ldg(reinterpret_cast<const float4 *>(rows + (size_t)(T * k + t) * D + d0));
        acc.x += r.x; acc.y += r.y; acc.z += r.z; acc.w += r.w;
    }
    const size_t yi = (size_t)t * D + d0;
    if (y_dtype == MOE_BF16) {
        __nv_bfloat162 *yp = reinterpret_cast<__nv_bfloat162 *>((__nv_bfloat16 *)y + yi);
        yp[0] = __floats2bfloat162_rn(acc.x, acc.y);
        yp[1] = __floats2bfloat162_rn(acc.z, acc.w);
    } else {
        *reinterpret_cast<float4 *>((float *)y + yi) = acc;
    }
}

// ------------------------------------------------------------------- host
// D: a multiple of 256 with a compiled slice geometry; F, shared F:
// multiples of 256 up to 1024 (one box per expert tile in the down kernel).
static bool gu_shape_ok(int D) { return D == 256 || D == 512 || D == 768 || D == 1024 || D == 2048; }

// Block types the kernels decode at a given D: all of them, Q6_K when its
// gate/up rows (210 * D / 256 bytes) are whole 16-byte units for the tensor
// copies, i.e. D = 2048 (its down rows arrive in 8-row groups, which always
// are)
static bool dec_type_ok(int qt, int D) {
    return qt_known(qt) && (qt != MOE_Q6_K || qt_row_bytes(qt, D) % 16 == 0);
}

bool decode_path_ok(int T, int D, int F, int sF, int qt, int sqt) {
    return T >= 1 && T <= 16 && gu_shape_ok(D) && F % 256 == 0 && F <= 1024 &&
           dec_type_ok(qt, D) && (sF == 0 || (sF % 256 == 0 && sF <= 1024 && dec_type_ok(sqt, D)));
}

// Hs rows are padded by 32 halves (64 bytes): row stride = 64 mod 128 bytes,
// so the down kernel's 16-byte fragment loads of rows n, n+1 do not collide
size_t decode_hs_halves(int T, int k, int F, int sF) {
    return (size_t)(T * k + T) * (size_t)(std::max(F, sF) + 32);
}
size_t decode_rows_floats(int T, int k, int D) { return (size_t)(T * k + T) * D; }

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess && q == cudaDriverEntryPointSuccess)
            fn = (EncodeTiledFn)p;
    }
    return fn;
}

// rows x row_bytes (8-byte elements) at base; boxes of box_rows rows and
// box_bytes (>= the slice, the excess zero-filled out of bounds)
static moe_status encode_rows(CUtensorMap *m, const void *base, size_t row_bytes, size_t nrows,
                              int box_bytes, int box_rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) { set_error("decode path: cuTensorMapEncodeTiled unavailable"); return MOE_ERR_CUDA; }
    const cuuint64_t dims[2] = {(cuuint64_t)(row_bytes / 8), (cuuint64_t)nrows};
    const cuuint64_t strides[1] = {(cuuint64_t)row_bytes};
    const cuuint32_t box[2] = {(cuuint32_t)(box_bytes / 8), (cuuint32_t)box_rows};
    const cuuint32_t es[2] = {1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT64, 2, const_cast<void *>(base), dims, strides,
                    box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
        set_error("decode path: tensor map encoding failed (%d) for %zu x %zu bytes", (int)r, nrows,
                  row_bytes);
        return MOE_ERR_CUDA;
    }
    return MOE_OK;
}

// Q6_K down rows (F weights, nrows rows, nrows a multiple of 8): a 3-D tensor
// of 560-byte chunks, 3 F / 256 of them an 8-row group; boxes of kDnRows rows
// land packed (kDnRows * the row bytes)
static moe_status encode_q6k_down(CUtensorMap *m, const void *base, int F, size_t nrows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) { set_error("decode path: cuTensorMapEncodeTiled unavailable"); return MOE_ERR_CUDA; }
    const size_t group = 8 * qt_row_bytes(MOE_Q6_K, F);          // 1680 * F / 256
    const cuuint32_t nch = (cuuint32_t)(group / kQ6Chunk);
    const cuuint64_t dims[3] = {(cuuint64_t)(kQ6Chunk / 8), nch, (cuuint64_t)(nrows / 8)};
    const cuuint64_t strides[2] = {(cuuint64_t)kQ6Chunk, (cuuint64_t)group};
    const cuuint32_t box[3] = {(cuuint32_t)(kQ6Chunk / 8), nch, (cuuint32_t)(kDnRows / 8)};
    const cuuint32_t es[3] = {1, 1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT64, 3, const_cast<void *>(base), dims, strides,
                    box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
        set_error("decode path: Q6_K tensor map encoding failed (%d) for %zu rows of F = %d", (int)r,
                  nrows, F);
        return MOE_ERR_CUDA;
    }
    return MOE_OK;
}

static moe_status encode_down(CUtensorMap *m, const void *base, int qt, int F, size_t nrows) {
    if (qt == MOE_Q6_K) return encode_q6k_down(m, base, F, nrows);
    const size_t rb = qt_row_bytes(qt, F);
    return encode_rows(m, base, rb, nrows, tma_row_bytes((int)rb), kDnRows);
}

static moe_status encode_maps(const DecArgs &a, int n_slots, int max_sb, DecMaps *m) {
    memset(m, 0, sizeof(*m));
    const size_t rg = qt_row_bytes(a.qt, a.D);
    const GuGeo gr = gu_geo(a.D, a.qt, max_sb);
    moe_status st;
    if ((st = encode_rows(&m->gate, a.gate, rg, (size_t)n_slots * a.F, gr.pitch, kTile)))
        return st;
    if ((st = encode_rows(&m->up, a.up, rg, (size_t)n_slots * a.F, gr.pitch, kTile)))
        return st;
    if ((st = encode_down(&m->down, a.down, a.qt, a.F, (size_t)n_slots * a.D))) return st;
    if (a.sF > 0) {
        const size_t rgs = qt_row_bytes(a.sqt, a.D);
        const GuGeo gs = gu_geo(a.D, a.sqt, max_sb);
        if ((st = encode_rows(&m->sgate, a.sh_gate, rgs, a.sF, gs.pitch, kTile))) return st;
        if ((st = encode_rows(&m->sup, a.sh_up, rgs, a.sF, gs.pitch, kTile))) return st;
        if ((st = encode_down(&m->sdown, a.sh_down, a.sqt, a.sF, a.D))) return st;
    }
    return MOE_OK;
}

template <typename... Args>
static cudaError_t launch_pdl(void (*kern)(Args...), int grid, int block, size_t smem,
                             cudaStream_t s, Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(block);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    return cudaLaunchKernelEx(&cfg, kern, args...);
}

// the gate/up kernel's per-CTA unit table (16 bytes a unit)
// units at most: sum over experts of ceil(tokens / 8) <= E + T*k/8 groups
static int gu_units_max(const DecArgs &a) {
    const int groups = a.E + (a.T * a.k) / kGuCols;
    return groups * (a.F / kTile) + (a.T + kGuCols - 1) / kGuCols * (a.sF / kTile);
}

static size_t unit_table_bytes(const DecArgs &a, int sms) {
    const int U_max = gu_units_max(a);
    const int grid = std::max(1, std::min(sms, U_max));
    return (size_t)((U_max + grid - 1) / grid) * 16 + 16;
}

static size_t tables_bytes(int E) {
    return 6 * (size_t)(E + 1) * sizeof(int) + (size_t)(kMaxTk + 16) * (sizeof(int) + sizeof(float));
}

// one slice per 16-row tile: each stage is a whole unit (two 18.7 KB boxes
// at D=2048, Q4_0)
static int gu_max_sb(int T) { (void)T; return 64; }

// the call has a type other than Q4_0 and Q8_0
static bool dec_all_types(const DecArgs &a) {
    auto basic = [](int q) { return q == MOE_Q4_0 || q == MOE_Q8_0; };
    return !basic(a.qt) || (a.sF > 0 && !basic(a.sqt));
}
// the block type of every expert of the call, when there is one (-1
// otherwise)
static int dec_one_type(const DecArgs &a) {
    return a.sF > 0 && a.sqt != a.qt ? -1 : a.qt;
}

template <bool ALL>
static cudaError_t launch_gateup1(const DecArgs &a, const DecMaps &m, int grid, size_t smem,
                                  cudaStream_t s, int S) {
    const bool wide = gu_max_sb(a.T) == 64;
    switch (a.D) {
    case 256: return launch_pdl(dec_gateup_kernel<32, 1, 1, ALL>, grid, kGThreads, smem, s, a, S, m);
    case 512: return launch_pdl(dec_gateup_kernel<32, 2, 2, ALL>, grid, kGThreads, smem, s, a, S, m);
    case 768: return launch_pdl(dec_gateup_kernel<32, 3, 3, ALL>, grid, kGThreads, smem, s, a, S, m);
    case 1024: return launch_pdl(dec_gateup_kernel<32, 4, 4, ALL>, grid, kGThreads, smem, s, a, S, m);
    default:
        if (!ALL && wide && dec_one_type(a) == MOE_Q4_0)
            return launch_pdl(dec_gateup_kernel<64, 8, 4, false, MOE_Q4_0>, grid, kGThreads, smem, s, a, S, m);
        if (!ALL && wide && dec_one_type(a) == MOE_Q8_0)
            return launch_pdl(dec_gateup_kernel<64, 8, 4, false, MOE_Q8_0>, grid, kGThreads, smem, s, a, S, m);
        if (ALL && wide && dec_one_type(a) >= 0) {
            switch (dec_one_type(a)) {
            case MOE_Q4_1: return launch_pdl(dec_gateup_kernel<64, 8, 4, true, MOE_Q4_1>, grid, kGThreads, smem, s, a, S, m);
            case MOE_Q5_0: return launch_pdl(dec_gateup_kernel<64, 8, 4, true, MOE_Q5_0>, grid, kGThreads, smem, s, a, S, m);
            case MOE_Q5_1: return launch_pdl(dec_gateup_kernel<64, 8, 4, true, MOE_Q5_1>, grid, kGThreads, smem, s, a, S, m);
            case MOE_Q4_K: return launch_pdl(dec_gateup_kernel<64, 8, 4, true, MOE_Q4_K>, grid, kGThreads, smem, s, a, S, m);
            default: return launch_pdl(dec_gateup_kernel<64, 8, 4, true, MOE_Q6_K>, grid, kGThreads, smem, s, a, S, m);
            }
        }
        return wide ? launch_pdl(dec_gateup_kernel<64, 8, 4, ALL>, grid, kGThreads, smem, s, a, S, m)
                    : launch_pdl(dec_gateup_kernel<32, 4, 4, ALL>, grid, kGThreads, smem, s, a, S, m);
    }
}

static cudaError_t launch_gateup(const DecArgs &a, const DecMaps &m, int grid, size_t smem,
                                 cudaStream_t s, int S) {
    return dec_all_types(a) ? launch_gateup1<true>(a, m, grid, smem, s, S)
                            : launch_gateup1<false>(a, m, grid, smem, s, S);
}

template <int NT>
static moe_status run_decode(const DecArgs &a, int n_slots, cudaStream_t s, Tracer *tr) {
    const int sms = num_sms();
    DecMaps maps;
    const int max_sb = a.D <= 1024 ? 32 : gu_max_sb(a.T);
    moe_status st = encode_maps(a, n_slots, max_sb, &maps);
    if (st != MOE_OK) return st;
    // gate/up and down run when this call has routed experts or the shared one
    if (a.routed || a.sF > 0) {
    // ---- gate/up
    {
        const int nbD = a.D / QK;
        const int pitch = std::max(gu_geo(a.D, a.qt, max_sb).pitch,
                                   a.sF > 0 ? gu_geo(a.D, a.sqt, max_sb).pitch : 0);
        const int stage_bytes = (int)round_up((size_t)2 * kTile * pitch, 128);
        // mirrors the kernel's carve; + 1024 for aligning the base
        const size_t fixed = round_up(round_up((size_t)(a.T + 1) * staged_act_bytes(a.D), 16) +
                                      (size_t)2 * (a.T + 1) * nbD * 4, 1024) +
                             (size_t)kGuRedBufs * kDW * 32 * 4 * sizeof(float) +
                             (2 * kMaxStages + 8) * sizeof(uint64_t) + tables_bytes(a.E) +
                             unit_table_bytes(a, sms) + 1024;
        if (fixed >= kDecSmemMax) { set_error("decode path: shared memory too small"); return MOE_ERR_SHAPE; }
        int S = (int)std::min<size_t>(kMaxStages, (kDecSmemMax - fixed) / stage_bytes);
        if (S < 2) { set_error("decode path: shared memory too small"); return MOE_ERR_SHAPE; }
        const size_t smem = fixed + (size_t)S * stage_bytes;
        const int U_max = gu_units_max(a);
        const int grid = std::max(1, std::min(sms, U_max));
        mark(tr, MOE_KERNEL_FFN_DECODE);
        cudaError_t e = launch_gateup(a, maps, grid, smem, s, S);
        if (e != cudaSuccess) return cuda_status(e, "dec_gateup_kernel");
    }
    // ---- down: Y rows
    {
        const int hrows = std::min(a.T, kGuCols);
        const int pr = dn_pitch(a.qt, a.F);
        const int ps = a.sF > 0 ? dn_pitch(a.sqt, a.sF) : 0;
        const size_t wbytes = (size_t)kDnRows * std::max(pr, ps);
        const size_t stage_bytes = round_up(wbytes + (size_t)hrows * a.hrow * 2, 128);
        const size_t fixed = 2 * kMaxStages * sizeof(uint64_t) + tables_bytes(a.E) +
                             (size_t)(a.E + 2 + kMaxTk / kGuCols + 2) * sizeof(int2) + 1024;
        if (fixed + stage_bytes > kDecSmemMax) {
            set_error("decode path: a %zu-byte stage does not fit shared memory", stage_bytes);
            return MOE_ERR_SHAPE;
        }
        // as many consumer groups (4 warps each) as stages fit, up to 4;
        // then up to 2 stages per group
        const int fit = (int)std::min<size_t>(kMaxStages, (kDecSmemMax - fixed) / stage_bytes);
        const int G = fit >= 4 ? 4 : fit >= 2 ? 2 : 1;
        const int Sg = std::min(2, fit / G);
        const size_t smem = fixed + (size_t)G * Sg * stage_bytes;
        const int U_max = (a.E + 1 + a.T * a.k / kGuCols) * (a.D / kDnRows);
        const int grid = std::max(1, std::min(sms, U_max));
        // no trace mark here: an event between the two kernels would cancel
        // their programmatic overlap
        cudaError_t e;
        switch (dec_one_type(a)) {
#define MOE_DN1(QT)                                                                          \
    case QT:                                                                                 \
        e = launch_pdl(dec_down_kernel<NT, !(QT == MOE_Q4_0 || QT == MOE_Q8_0), QT>, grid,   \
                       kDThreads, smem, s, a, G, Sg, hrows, maps);                           \
        break;
            MOE_DN1(MOE_Q4_0)
            MOE_DN1(MOE_Q8_0)
            MOE_DN1(MOE_Q4_1)
            MOE_DN1(MOE_Q5_0)
            MOE_DN1(MOE_Q5_1)
            MOE_DN1(MOE_Q4_K)
            MOE_DN1(MOE_Q6_K)
#undef MOE_DN1
        default:
            e = dec_all_types(a) ? launch_pdl(dec_down_kernel<NT, true>, grid, kDThreads, smem, s, a,
                                              G, Sg, hrows, maps)
                                 : launch_pdl(dec_down_kernel<NT, false>, grid, kDThreads, smem, s, a,
                                              G, Sg, hrows, maps);
        }
        if (e != cudaSuccess) return cuda_status(e, "dec_down_kernel");
    }
    }
    // ---- combine (fused layer only): y = sum of the gated rows (+ shared)
    if (a.y) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(a.T, (a.D / 4 + 255) / 256);
        cfg.blockDim = dim3(256);
        cfg.stream = s;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        cudaError_t e = cudaLaunchKernelEx(&cfg, dec_combine_kernel, (const float *)a.rows_out,
                                           a.inv, a.T, a.k, a.D, a.comb_shared, a.y, a.y_dtype);
        if (e != cudaSuccess) return cuda_status(e, "dec_combine_kernel");
    }
    return MOE_OK;
}

moe_status launch_ffn_decode(const void *x, int x_dtype, int T, int D, int F, int E, int k,
                             const int32_t *perm, const int32_t *inv, const int32_t *offsets,
                             const float *gates, const moe_pool &pool, const uint8_t *mask,
                             bool routed, const moe_pool *shared, int sF, bool comb_shared,
                             __half *Hs, void *y, int y_dtype, float *rows_out, int *err,
                             cudaStream_t s, Tracer *tr) {
    DecArgs a{};
    a.T = T; a.D = D; a.F = F; a.E = E; a.k = k; a.sF = shared ? sF : 0;
    a.routed = routed ? 1 : 0;
    a.n_slots = pool.n_slots;
    a.comb_shared = comb_shared ? 1 : 0;
    a.perm = perm; a.offsets = offsets; a.gates = gates; a.mask = mask;
    a.gate = (const uint8_t *)pool.gate; a.up = (const uint8_t *)pool.up;
    a.down = (const uint8_t *)pool.down; a.slot_map = pool.slot_of_expert;
    if (!dec_type_ok(pool.qtype, D)) {
        set_error("decode path: unsupported quant type %d at D = %d", (int)pool.qtype, D);
        return MOE_ERR_UNSUPPORTED_QTYPE;
    }
    if (T * k > kMaxTk) {
        set_error("decode path: T*k=%d exceeds %d", T * k, kMaxTk);
        return MOE_ERR_SHAPE;
    }
    a.qt = pool.qtype;
    a.sqt = pool.qtype;
    if (shared) {
        a.sh_gate = (const uint8_t *)shared->gate; a.sh_up = (const uint8_t *)shared->up;
        a.sh_down = (const uint8_t *)shared->down;
        if (!dec_type_ok(shared->qtype, D)) {
            set_error("decode path: unsupported shared-expert quant type %d at D = %d",
                      (int)shared->qtype, D);
            return MOE_ERR_UNSUPPORTED_QTYPE;
        }
        a.sqt = shared->qtype;
    }
    a.x = x; a.x_bf16 = (x_dtype == MOE_BF16);
    a.x_vec = ((uintptr_t)x % 16) == 0;
    a.Hs = Hs; a.hrow = std::max(F, a.sF) + 32;
    a.y = y; a.y_dtype = y_dtype; a.rows_out = rows_out; a.err = err;
    a.inv = inv;
    if (y && !rows_out) {
        set_error("decode path: the fused combine needs a rows buffer");
        return MOE_ERR_INVALID_ARG;
    }
    // the down kernel takes at most 8 tokens a unit: one column tile
    return run_decode<1>(a, pool.n_slots, s, tr);
}

// ------------------------------------------------ 8-bit activations: host
static bool a8_type_ok(int q) { return q == MOE_Q4_0 || q == MOE_Q8_0; }

bool decode_a8_ok(int T, int D, int F, int sF, int qt, int sqt) {
    return decode_path_ok(T, D, F, sF, qt, sqt) && a8_type_ok(qt) && (sF == 0 || a8_type_ok(sqt));
}
size_t decode_a8_hq_bytes(int T, int k, int F, int sF) {
    return (size_t)(T * k + T) * (size_t)std::max(F, sF);
}
size_t decode_a8_hs_bytes(int T, int k, int F, int sF) {
    return (size_t)(T * k + T) * (size_t)(std::max(F, sF) / QK) * sizeof(float2);
}

static moe_status encode_maps_a8(const A8Args &A, int n_slots, int hrows, int hpitch, A8Maps *m) {
    memset(m, 0, sizeof(*m));
    const DecArgs &a = A.d;
    const size_t rg = qt_row_bytes(a.qt, a.D);
    const GuGeo gr = gu_geo(a.D, a.qt, kA8MaxSb);
    moe_status st;
    if ((st = encode_rows(&m->m.gate, a.gate, rg, (size_t)n_slots * a.F, gr.pitch, kA8Rows))) return st;
    if ((st = encode_rows(&m->m.up, a.up, rg, (size_t)n_slots * a.F, gr.pitch, kA8Rows))) return st;
    const size_t rbd = qt_row_bytes(a.qt, a.F);
    if ((st = encode_rows(&m->m.down, a.down, rbd, (size_t)n_slots * a.D, tma_row_bytes((int)rbd), kDnRows)))
        return st;
    if (a.sF > 0) {
        const size_t rgs = qt_row_bytes(a.sqt, a.D);
        const GuGeo gs = gu_geo(a.D, a.sqt, kA8MaxSb);
        if ((st = encode_rows(&m->m.sgate, a.sh_gate, rgs, a.sF, gs.pitch, kA8Rows))) return st;
        if ((st = encode_rows(&m->m.sup, a.sh_up, rgs, a.sF, gs.pitch, kA8Rows))) return st;
        const size_t rbs = qt_row_bytes(a.sqt, a.sF);
        if ((st = encode_rows(&m->m.sdown, a.sh_down, rbs, a.D, tma_row_bytes((int)rbs), kDnRows))) return st;
    }
    // h codes: rows of hq_row bytes; a box of hrows rows and hpitch bytes
    // (the bytes past a row read as zeros)
    return encode_rows(&m->hq, A.hq, (size_t)A.hq_row, (size_t)(a.T * a.k + a.T), hpitch, hrows);
}

template <int WB>
static cudaError_t launch_gateup_a8(const A8Args &A, const A8Maps &m, int grid, size_t smem,
                                    cudaStream_t s, int S) {
    return launch_pdl(dec_gateup_a8_kernel<WB>, grid, kGThreads, smem, s, A, S, m);
}

template <int NT>
static moe_status run_decode_a8(const A8Args &A, int n_slots, cudaStream_t s, Tracer *tr) {
    const DecArgs &a = A.d;
    const int sms = num_sms();
    const int hrows = std::min(a.T, 16);
    const int hpitch = tma_row_bytes(A.hq_row);
    A8Maps maps;
    moe_status st = encode_maps_a8(A, n_slots, hrows, hpitch, &maps);
    if (st != MOE_OK) return st;
    if (a.routed || a.sF > 0) {
        // ---- gate/up with h quantized in the epilogue
        const int nbD = a.D / QK;
        const int pitch = std::max(gu_geo(a.D, a.qt, kA8MaxSb).pitch,
                                   a.sF > 0 ? gu_geo(a.D, a.sqt, kA8MaxSb).pitch : 0);
        const int stage_bytes = (int)round_up((size_t)2 * kA8Rows * pitch, 128);
        const int groups = a.E + (a.T * a.k) / kGuCols;
        const int U_max = groups * (a.F / kA8Rows) + (a.T + kGuCols - 1) / kGuCols * (a.sF / kA8Rows);
        const int grid = std::max(1, std::min(sms, U_max));
        const size_t units = (size_t)((U_max + grid - 1) / grid) * 16 + 16;
        const size_t fixed = round_up(round_up((size_t)(a.T + 1) * a8_xrow(a.D), 16) +
                                      (size_t)2 * (a.T + 1) * nbD * 4, 1024) +
                             (size_t)kGuRedBufs * kDW * 2 * 32 * 4 * sizeof(float) +
                             (2 * kMaxStages + 8) * sizeof(uint64_t) + tables_bytes(a.E) + units + 1024;
        if (fixed >= kDecSmemMax) { set_error("decode path (8-bit activations): shared memory too small"); return MOE_ERR_SHAPE; }
        const int S = (int)std::min<size_t>(kMaxStages, (kDecSmemMax - fixed) / stage_bytes);
        if (S < 2) { set_error("decode path (8-bit activations): shared memory too small"); return MOE_ERR_SHAPE; }
        const size_t smem = fixed + (size_t)S * stage_bytes;
        const int WB = std::min(nbD, kA8MaxSb) / 8;
        mark(tr, MOE_KERNEL_FFN_DECODE);
        cudaError_t e;
        switch (WB) {
        case 1: e = launch_gateup_a8<1>(A, maps, grid, smem, s, S); break;
        case 2: e = launch_gateup_a8<2>(A, maps, grid, smem, s, S); break;
        case 3: e = launch_gateup_a8<3>(A, maps, grid, smem, s, S); break;
        default: e = launch_gateup_a8<4>(A, maps, grid, smem, s, S); break;
        }
        if (e != cudaSuccess) return cuda_status(e, "dec_gateup_a8_kernel");
        // ---- down on the h codes
        const int pr = tma_row_bytes((int)qt_row_bytes(a.qt, a.F));
        const int ps = a.sF > 0 ? tma_row_bytes((int)qt_row_bytes(a.sqt, a.sF)) : 0;
        const size_t wbytes = (size_t)kDnRows * std::max(pr, ps);
        const size_t hsrow = (size_t)(A.hq_row / QK) * 8;
        const size_t dstage = round_up(wbytes + round_up((size_t)hrows * hpitch, 128) + hrows * hsrow, 128);
        const size_t dfixed = 2 * kMaxStages * sizeof(uint64_t) + tables_bytes(a.E) + 1024;
        if (dfixed + dstage > kDecSmemMax) {
            set_error("decode path (8-bit activations): a %zu-byte stage does not fit shared memory", dstage);
            return MOE_ERR_SHAPE;
        }
        const int fit = (int)std::min<size_t>(kMaxStages, (kDecSmemMax - dfixed) / dstage);
        const int G = fit >= 4 ? 4 : fit >= 2 ? 2 : 1;
        const int Sg = std::min(2, fit / G);
        const size_t dsmem = dfixed + (size_t)G * Sg * dstage;
        const int dgrid = std::max(1, std::min(sms, (a.E + 1) * (a.D / kDnRows)));
        e = launch_pdl(dec_down_a8_kernel<NT>, dgrid, kDThreads, dsmem, s, A, G, Sg, hrows, hpitch, maps);
        if (e != cudaSuccess) return cuda_status(e, "dec_down_a8_kernel");
    }
    if (a.y) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(a.T, (a.D / 4 + 255) / 256);
        cfg.blockDim = dim3(256);
        cfg.stream = s;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        cudaError_t e = cudaLaunchKernelEx(&cfg, dec_combine_kernel, (const float *)a.rows_out,
                                           a.inv, a.T, a.k, a.D, a.comb_shared, a.y, a.y_dtype);
        if (e != cudaSuccess) return cuda_status(e, "dec_combine_kernel");
    }
    return MOE_OK;
}

moe_status launch_ffn_decode_a8(const void *x, int x_dtype, int T, int D, int F, int E, int k,
                                const int32_t *perm, const int32_t *inv, const int32_t *offsets,
                                const float *gates, const moe_pool &pool, const uint8_t *mask,
                                bool routed, const moe_pool *shared, int sF, bool comb_shared,
                                int8_t *hq, float2 *hs, void *y, int y_dtype, float *rows_out,
                                int *err, cudaStream_t s, Tracer *tr) {
    if (!a8_type_ok(pool.qtype) || (shared && !a8_type_ok(shared->qtype))) {
        set_error("8-bit activations: Q4_0 and Q8_0 experts only (got %d%s%d)", (int)pool.qtype,
                  shared ? ", shared " : "", shared ? (int)shared->qtype : 0);
        return MOE_ERR_UNSUPPORTED_QTYPE;
    }
    if (T * k > kMaxTk) {
        set_error("decode path: T*k=%d exceeds %d", T * k, kMaxTk);
        return MOE_ERR_SHAPE;
    }
    if (!gates || !perm || !inv || !rows_out) {
        set_error("8-bit activations: the fused layer's gates, permutation and rows are needed");
        return MOE_ERR_INVALID_ARG;
    }
    A8Args A{};
    DecArgs &a = A.d;
    a.T = T; a.D = D; a.F = F; a.E = E; a.k = k; a.sF = shared ? sF : 0;
    a.routed = routed ? 1 : 0;
    a.n_slots = pool.n_slots;
    a.comb_shared = comb_shared ? 1 : 0;
    a.perm = perm; a.offsets = offsets; a.gates = gates; a.mask = mask;
    a.gate = (const uint8_t *)pool.gate; a.up = (const uint8_t *)pool.up;
    a.down = (const uint8_t *)pool.down; a.slot_map = pool.slot_of_expert;
    a.qt = pool.qtype;
    a.sqt = pool.qtype;
    if (shared) {
        a.sh_gate = (const uint8_t *)shared->gate; a.sh_up = (const uint8_t *)shared->up;
        a.sh_down = (const uint8_t *)shared->down;
        a.sqt = shared->qtype;
    }
    a.x = x; a.x_bf16 = (x_dtype == MOE_BF16);
    a.x_vec = ((uintptr_t)x % 16) == 0;
    a.y = y; a.y_dtype = y_dtype; a.rows_out = rows_out; a.err = err;
    a.inv = inv;
    A.hq = hq;
    A.hs = hs;
    A.hq_row = std::max(F, a.sF);
    return T > 8 ? run_decode_a8<2>(A, pool.n_slots, s, tr) : run_decode_a8<1>(A, pool.n_slots, s, tr);
}

}  // namespace moe
