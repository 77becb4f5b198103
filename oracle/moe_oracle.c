/*
 * moe_oracle.c -- plain, slow, obviously-correct CPU oracle for one routed
 * MoE FFN layer on ggml-style block-quantized expert weights.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the bench's
 * CPU-baseline leg may load this library.  It shares no code, header, table
 * or constant with the CUDA library; neither includes the other.
 *
 * What it computes (all floating point in double unless stated):
 *
 *   Block formats -- FreeToken fork README, "Quant types" table (Standard
 *   family: Q4_0, Q4_1, Q5_0, Q5_1, Q8_0; the page names the types, the byte
 *   layouts are ggml's published ones).  32 weights per block, fp16 scale d
 *   (and fp16 minimum m for the _1 types), all little endian:
 *     Q8_0 {fp16 d; int8 q[32]}                  value q[i] * d
 *     Q4_0 {fp16 d; uint8 qs[16]}                value (q[i] - 8) * d
 *     Q4_1 {fp16 d; fp16 m; uint8 qs[16]}        value q[i] * d + m
 *     Q5_0 {fp16 d; uint8 qh[4]; uint8 qs[16]}   value (q[i] - 16) * d
 *     Q5_1 {fp16 d; fp16 m; uint8 qh[4]; uint8 qs[16]}   value q[i] * d + m
 *   qs byte j holds the low 4 bits of element j (low nibble) and of element
 *   j+16 (high nibble); for the 5-bit types bit i of the 32-bit word qh is
 *   bit 4 of element i.
 *   K-quants (same table, K-quants row; ggml's published super-block
 *   layouts), 256 weights per block:
 *     Q4_K {fp16 d; fp16 dmin; uint8 scales[12]; uint8 qs[128]} (144 B):
 *       eight sub-blocks of 32, each with a 6-bit scale sc_j and a 6-bit
 *       min m_j packed in scales[] (orc_q4k_scale_min); value
 *       d * sc_j * q - dmin * m_j; weight 64c + l (l < 32) is the low nibble
 *       of qs[32c + l] (sub-block 2c), weight 64c + 32 + l its high nibble
 *       (sub-block 2c + 1).
 *     Q6_K {uint8 ql[128]; uint8 qh[64]; int8 scales[16]; fp16 d} (210 B):
 *       value d * scales[i / 16] * (q_i - 32) with q_i 6-bit: in half h
 *       (weights 128h + 32r + l, r < 4, l < 32) the low 4 bits are nibble
 *       r / 2 of ql[64h + 32(r % 2) + l] and the high 2 bits are bits
 *       2r, 2r+1 of qh[32h + l].
 *   Expert pool layout -- FreeToken fork README, "Known limits": experts back
 *   to back, expert * nrows * (ncols / 32) blocks, no padding, one type.
 *   Per expert: W_gate, W_up are [F rows][D/32 blocks], W_down [D][F/32].
 *
 *   Layer (the routed MoE FFN layer the pages serve; FreeToken wiki
 *   explainer, opening section: a subset of experts is active per token):
 *     L[t,e]  = sum_i x[t,i] W_r[i,e] + b[e]       (double, then rounded to fp32)
 *     S_t     = the k experts of largest L[t,.], ordered by L descending,
 *               ties to the lower expert index
 *     p       = softmax over all E of L[t,.]      (double, max-subtracted)
 *     g[t,j]  = p[S_tj] / sum_{i in S_t} p[i]      (renormalised top-k gates)
 *     h       = silu(x_t . W_gate,e row) * (x_t . W_up,e row), silu(z) = z/(1+e^-z)
 *     Y[t,j]  = W_down,e h                          (e = S_tj)
 *     y_t     = sum_j g[t,j] Y[t,j]  (+ shared-expert FFN of x_t, weight 1)
 *   Permutation: a stable counting sort of the flat (t, j) entries by expert.
 *
 *   Expert cache: a per-layer LRU over a fixed number of device slots
 *   (FreeToken fork README, "About": global LRU expert caching; wiki
 *   explainer: shared LRU expert caching follows token-level routing
 *   locality; kongchang article, "From Static Allocation to Dynamic
 *   Scheduling": VRAM as a cache with the full model in system RAM).
 *   The replacement rules the pages leave open are fixed in orc_lru_request.
 *
 * Parity of every function here is pinned by the CPU tests against closed
 * forms, brute force and hand-packed blocks.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORC_QK 32
#define ORC_Q4_0 2
#define ORC_Q4_1 3
#define ORC_Q5_0 6
#define ORC_Q5_1 7
#define ORC_Q8_0 8
#define ORC_Q4_K 12
#define ORC_Q6_K 14

/* IEEE 754 binary16 -> double, decoded bit by bit (sign, 5-bit exponent with
 * bias 15, 10-bit fraction; subnormals, infinities and NaN included). */
double orc_half_to_double(uint16_t h)
{
    int sign = (h >> 15) & 1;
    int expo = (h >> 10) & 0x1f;
    int frac = h & 0x3ff;
    double v;
    if (expo == 0)
        v = ldexp((double)frac, -24);              /* 2^-14 * frac / 2^10 */
    else if (expo == 31)
        v = frac ? NAN : INFINITY;
    else
        v = ldexp(1.0 + (double)frac / 1024.0, expo - 15);
    return sign ? -v : v;
}

int orc_block_bytes(int qtype)
{
    switch (qtype) {
    case ORC_Q8_0: return 2 + 32;
    case ORC_Q4_0: return 2 + 16;
    case ORC_Q4_1: return 2 + 2 + 16;
    case ORC_Q5_0: return 2 + 4 + 16;
    case ORC_Q5_1: return 2 + 2 + 4 + 16;
    case ORC_Q4_K: return 2 + 2 + 12 + 128;
    case ORC_Q6_K: return 128 + 64 + 16 + 2;
    default: return 0;
    }
}

static double orc_half_at(const uint8_t *p)
{
    return orc_half_to_double((uint16_t)(p[0] | (p[1] << 8)));   /* little endian */
}

/* Weights per block: 256 for the K-quants, 32 for the rest, 0 if unknown. */
int orc_block_weights(int qtype)
{
    if (orc_block_bytes(qtype) == 0) return 0;
    return (qtype == ORC_Q4_K || qtype == ORC_Q6_K) ? 256 : ORC_QK;
}

/* Bytes of a row of ncols weights (ncols a multiple of the block). */
static size_t orc_row_bytes(int qtype, int ncols)
{
    return (size_t)(ncols / orc_block_weights(qtype)) * (size_t)orc_block_bytes(qtype);
}

/* Q4_K: the 6-bit scale and min of sub-block j (0..7) from scales[12].
 * Sub-blocks 0-3 keep theirs in the low six bits of bytes j and j+4;
 * sub-blocks 4-7 in the nibbles of byte j+4 (scale low, min high) plus the
 * top two bits of bytes j-4 (scale) and j (min). */
static void orc_q4k_scale_min(const uint8_t *sc, int j, int *scale, int *min)
{
    if (j < 4) {
        *scale = sc[j] & 63;
        *min = sc[j + 4] & 63;
    } else {
        *scale = (sc[j + 4] & 0x0f) | ((sc[j - 4] >> 6) << 4);
        *min = (sc[j + 4] >> 4) | ((sc[j] >> 6) << 4);
    }
}

static void orc_dequant_q4k(const uint8_t *blk, double *out)
{
    double d = orc_half_at(blk), dmin = orc_half_at(blk + 2);
    const uint8_t *sc = blk + 4, *qs = blk + 16;
    for (int i = 0; i < 256; i++) {
        int j = i / 32, l = i % 32, scale, min;
        orc_q4k_scale_min(sc, j, &scale, &min);
        int byte = qs[32 * (j / 2) + l];
        int q = (j % 2) ? (byte >> 4) : (byte & 0x0f);
        out[i] = d * (double)scale * (double)q - dmin * (double)min;
    }
}

static void orc_dequant_q6k(const uint8_t *blk, double *out)
{
    const uint8_t *ql = blk, *qh = blk + 128;
    const int8_t *sc = (const int8_t *)(blk + 192);
    double d = orc_half_at(blk + 208);
    for (int i = 0; i < 256; i++) {
        int h = i / 128, r = (i % 128) / 32, l = i % 32;
        int lo = ql[64 * h + 32 * (r % 2) + l];
        lo = (r / 2) ? (lo >> 4) : (lo & 0x0f);
        int hi = (qh[32 * h + l] >> (2 * r)) & 3;
        int q = lo | (hi << 4);
        out[i] = d * (double)sc[i / 16] * (double)(q - 32);
    }
}


/* Dequantize one row of ncols weights (a multiple of the block) into out[]. */
int orc_dequant_row(const uint8_t *row, int qtype, int ncols, double *out)
{
    int bs = orc_block_bytes(qtype), bw = orc_block_weights(qtype);
    if (bs == 0 || ncols % bw) return -1;
    if (bw == 256) {
        for (int b = 0; b < ncols / 256; b++) {
            if (qtype == ORC_Q4_K) orc_dequant_q4k(row + (size_t)b * bs, out + 256 * b);
            else orc_dequant_q6k(row + (size_t)b * bs, out + 256 * b);
        }
        return 0;
    }
    const int has_m = qtype == ORC_Q4_1 || qtype == ORC_Q5_1;
    const int has_qh = qtype == ORC_Q5_0 || qtype == ORC_Q5_1;
    for (int b = 0; b < ncols / ORC_QK; b++) {
        const uint8_t *blk = row + (size_t)b * bs;
        double d = orc_half_at(blk);
        double m = has_m ? orc_half_at(blk + 2) : 0.0;
        const uint8_t *qh = blk + 2 + 2 * has_m;          /* 5-bit types only */
        const uint8_t *qs = qh + 4 * has_qh;
        uint32_t hbits = has_qh ? (uint32_t)qh[0] | ((uint32_t)qh[1] << 8) |
                                      ((uint32_t)qh[2] << 16) | ((uint32_t)qh[3] << 24)
                                : 0u;
        for (int i = 0; i < ORC_QK; i++) {
            double v;
            if (qtype == ORC_Q8_0) {
                int q = (int)(int8_t)qs[i];
                v = (double)q * d;
            } else {
                int byte = qs[i % 16];
                int q = (i < 16) ? (byte & 0x0f) : (byte >> 4);
                if (has_qh) q |= (int)((hbits >> i) & 1u) << 4;
                if (qtype == ORC_Q4_0) v = (double)(q - 8) * d;
                else if (qtype == ORC_Q5_0) v = (double)(q - 16) * d;
                else v = (double)q * d + m;
            }
            out[b * ORC_QK + i] = v;
        }
    }
    return 0;
}

/* Router logits in double, rounded once to fp32.  x [T,D], W_r [D,E]
 * row-major, bias [E] or NULL. */
void orc_router_logits(const float *x, const float *w_r, const float *bias,
                       int T, int D, int E, float *logits)
{
    for (int t = 0; t < T; t++)
        for (int e = 0; e < E; e++) {
            double acc = 0.0;
            for (int i = 0; i < D; i++)
                acc += (double)x[(size_t)t * D + i] * (double)w_r[(size_t)i * E + e];
            if (bias) acc += (double)bias[e];
            logits[(size_t)t * E + e] = (float)acc;
        }
}

/* Top-k selection, softmax and renormalisation per token.
 * Selection: repeatedly take the not-yet-taken expert with the largest
 * logit, the lower index on equal logits (a selection sort on the key
 * (L descending, index ascending)).  Gates from the full softmax in double. */
void orc_select(const float *logits, int T, int E, int k, int renorm,
                int32_t *ids, double *gates)
{
    char *taken = (char *)malloc((size_t)E);
    double *p = (double *)malloc(sizeof(double) * (size_t)E);
    for (int t = 0; t < T; t++) {
        const float *L = logits + (size_t)t * E;
        memset(taken, 0, (size_t)E);
        for (int j = 0; j < k; j++) {
            int best = -1;
            for (int e = 0; e < E; e++) {
                if (taken[e]) continue;
                if (best < 0 || L[e] > L[best]) best = e;   /* strict: keeps lower index */
            }
            taken[best] = 1;
            ids[(size_t)t * k + j] = best;
        }
        double m = -INFINITY;
        for (int e = 0; e < E; e++) if ((double)L[e] > m) m = (double)L[e];
        double z = 0.0;
        for (int e = 0; e < E; e++) { p[e] = exp((double)L[e] - m); z += p[e]; }
        for (int e = 0; e < E; e++) p[e] /= z;
        double s = 0.0;
        for (int j = 0; j < k; j++) s += p[ids[(size_t)t * k + j]];
        for (int j = 0; j < k; j++) {
            double pj = p[ids[(size_t)t * k + j]];
            gates[(size_t)t * k + j] = renorm ? pj / s : pj;
        }
    }
    free(taken);
    free(p);
}

/* Stable counting sort of the flat entries n = t*k + j by expert id:
 * counts[e], offsets[e] = sum of earlier counts (offsets[E] = T*k),
 * perm[pos] = n in order (expert, t, j), inv[n] = pos. */
int orc_permute(const int32_t *ids, int T, int k, int E, int32_t *counts,
                int32_t *offsets, int32_t *perm, int32_t *inv)
{
    int N = T * k;
    for (int e = 0; e < E; e++) counts[e] = 0;
    for (int n = 0; n < N; n++) {
        if (ids[n] < 0 || ids[n] >= E) return -1;
        counts[ids[n]]++;
    }
    offsets[0] = 0;
    for (int e = 0; e < E; e++) offsets[e + 1] = offsets[e] + counts[e];
    int32_t *cursor = (int32_t *)malloc(sizeof(int32_t) * (size_t)(E + 1));
    for (int e = 0; e <= E; e++) cursor[e] = offsets[e];
    for (int n = 0; n < N; n++) {
        int pos = cursor[ids[n]]++;
        perm[pos] = n;
        inv[n] = pos;
    }
    free(cursor);
    return 0;
}

static double orc_silu(double z) { return z / (1.0 + exp(-z)); }

/* One expert's SwiGLU FFN of one activation row xt[D] -> Y[D].
 * gate/up/down point at this expert's matrices in the pool. */
static void orc_expert_ffn_row(const double *xt, const uint8_t *gate,
                               const uint8_t *up, const uint8_t *down, int qtype,
                               int D, int F, double *wrow, double *h, double *Y)
{
    size_t gate_row = orc_row_bytes(qtype, D);
    size_t down_row = orc_row_bytes(qtype, F);
    for (int r = 0; r < F; r++) {
        double a = 0.0, u = 0.0;
        orc_dequant_row(gate + r * gate_row, qtype, D, wrow);
        for (int i = 0; i < D; i++) a += xt[i] * wrow[i];
        orc_dequant_row(up + r * gate_row, qtype, D, wrow);
        for (int i = 0; i < D; i++) u += xt[i] * wrow[i];
        h[r] = orc_silu(a) * u;
    }
    for (int d = 0; d < D; d++) {
        double acc = 0.0;
        orc_dequant_row(down + d * down_row, qtype, F, wrow);
        for (int f = 0; f < F; f++) acc += h[f] * wrow[f];
        Y[d] = acc;
    }
}

static size_t orc_expert_stride(int nrows, int ncols, int qtype)
{
    return (size_t)nrows * orc_row_bytes(qtype, ncols);
}

/* The routed layer for a list of tokens.
 *  x [T,D] fp32 values; ids/gates [T,k] from orc_select (any k-subset works);
 *  gate/up/down: pools of E experts in `qtype` (slot = expert id);
 *  sh_*: optional shared expert (its own type sh_qtype, F = sh_F), weight 1;
 *  tok_list[n_tok]: the tokens to evaluate (NULL = all T, n_tok = T);
 *  y [n_tok, D] doubles.  dense != 0 evaluates all E experts per token and
 *  weights each by its gate if selected and by 0 otherwise (the dense,
 *  masked form of the same sum).  Returns 0, or -1 on bad arguments. */
int orc_layer(const float *x, int T, int D, int F, int E, int k, int qtype,
              const uint8_t *gate, const uint8_t *up, const uint8_t *down,
              const int32_t *ids, const double *gates,
              const uint8_t *sh_gate, const uint8_t *sh_up,
              const uint8_t *sh_down, int sh_F, int sh_qtype,
              const int32_t *tok_list, int n_tok, int dense, int nthreads,
              double *y)
{
    int bw = orc_block_weights(qtype);
    if (bw == 0 || D % bw || F % bw || k > E)
        return -1;
    if (sh_gate && (orc_block_weights(sh_qtype) == 0 || D % orc_block_weights(sh_qtype) ||
                    sh_F % orc_block_weights(sh_qtype)))
        return -1;
    if (!tok_list) n_tok = T;
    size_t gstride = orc_expert_stride(F, D, qtype);
    size_t dstride = orc_expert_stride(D, F, qtype);
    int maxF = F > sh_F ? F : sh_F;
    int maxW = D > maxF ? D : maxF;
    int bad = 0;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
#endif
    for (int n = 0; n < n_tok; n++) {
        int t = tok_list ? tok_list[n] : n;
        if (t < 0 || t >= T) { bad |= 1; continue; }
        double *xt = (double *)malloc(sizeof(double) * (size_t)D);
        double *wrow = (double *)malloc(sizeof(double) * (size_t)maxW);
        double *h = (double *)malloc(sizeof(double) * (size_t)maxF);
        double *Y = (double *)malloc(sizeof(double) * (size_t)D);
        double *yt = y + (size_t)n * D;
        for (int i = 0; i < D; i++) { xt[i] = (double)x[(size_t)t * D + i]; yt[i] = 0.0; }
        if (!dense) {
            for (int j = 0; j < k; j++) {
                int e = ids[(size_t)t * k + j];
                if (e < 0 || e >= E) { bad |= 1; break; }
                orc_expert_ffn_row(xt, gate + e * gstride, up + e * gstride,
                                   down + e * dstride, qtype, D, F, wrow, h, Y);
                double g = gates[(size_t)t * k + j];
                for (int i = 0; i < D; i++) yt[i] += g * Y[i];
            }
        } else {
            for (int e = 0; e < E; e++) {
                double g = 0.0;
                for (int j = 0; j < k; j++)
                    if (ids[(size_t)t * k + j] == e) g = gates[(size_t)t * k + j];
                orc_expert_ffn_row(xt, gate + e * gstride, up + e * gstride,
                                   down + e * dstride, qtype, D, F, wrow, h, Y);
                for (int i = 0; i < D; i++) yt[i] += g * Y[i];
            }
        }
        if (sh_gate) {
            orc_expert_ffn_row(xt, sh_gate, sh_up, sh_down, sh_qtype, D, sh_F,
                               wrow, h, Y);
            for (int i = 0; i < D; i++) yt[i] += Y[i];
        }
        free(xt); free(wrow); free(h); free(Y);
    }
    return bad ? -1 : 0;
}

/* Un-combined expert outputs: for each listed permuted position pos, with
 * n = perm[pos], t = n / k, e = the expert of segment pos falls in,
 * Y[i] = FFN_e(x_t) (no gate).  pos_list NULL = all T*k positions. */
int orc_expert_rows(const float *x, int T, int D, int F, int E, int k,
                    int qtype, const uint8_t *gate, const uint8_t *up,
                    const uint8_t *down, const int32_t *perm,
                    const int32_t *offsets, const int32_t *pos_list, int n_pos,
                    int nthreads, double *Y)
{
    int bw = orc_block_weights(qtype);
    if (bw == 0 || D % bw || F % bw) return -1;
    if (!pos_list) n_pos = T * k;
    size_t gstride = orc_expert_stride(F, D, qtype);
    size_t dstride = orc_expert_stride(D, F, qtype);
    int maxW = D > F ? D : F;
    int bad = 0;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
#endif
    for (int n = 0; n < n_pos; n++) {
        int pos = pos_list ? pos_list[n] : n;
        if (pos < 0 || pos >= T * k) { bad |= 1; continue; }
        int e = 0;
        while (e < E && offsets[e + 1] <= pos) e++;
        if (e >= E) { bad |= 1; continue; }
        int t = perm[pos] / k;
        double *xt = (double *)malloc(sizeof(double) * (size_t)D);
        double *wrow = (double *)malloc(sizeof(double) * (size_t)maxW);
        double *h = (double *)malloc(sizeof(double) * (size_t)F);
        for (int i = 0; i < D; i++) xt[i] = (double)x[(size_t)t * D + i];
        orc_expert_ffn_row(xt, gate + e * gstride, up + e * gstride,
                           down + e * dstride, qtype, D, F, wrow, h,
                           Y + (size_t)n * D);
        free(xt); free(wrow); free(h);
    }
    return bad ? -1 : 0;
}

/* ------------------------------------------------------------------
 * 8-bit activations (the pages' W4A8 / W8A8 mode: the FreeToken fork README's
 * note on CUDA W4A8 MMVQ against CPU AVX; the blocks follow ggml's 8-bit
 * activation format).  Per 32-value block, all in fp32:
 *   amax = max |v_i|, d = amax / 127, id = (d != 0) ? 1 / d : 0,
 *   q_i  = round-half-away-from-zero(v_i * id)       (|q_i| <= 127),
 * and q_i stands for the value q_i * d.  Both sides of a parity test take
 * these integer decisions with the same fp32 operations. */
void orc_quantize_act8(const float *v, int n, int8_t *q, float *d)
{
    for (int b = 0; b < n / ORC_QK; b++) {
        const float *vb = v + (size_t)b * ORC_QK;
        float amax = 0.0f;
        for (int i = 0; i < ORC_QK; i++) {
            float a = fabsf(vb[i]);
            if (a > amax) amax = a;
        }
        float db = amax / 127.0f;
        float id = (db != 0.0f) ? 1.0f / db : 0.0f;
        d[b] = db;
        for (int i = 0; i < ORC_QK; i++) {
            float s = vb[i] * id;
            q[(size_t)b * ORC_QK + i] = (int8_t)roundf(s);
        }
    }
}

/* Sum over the blocks of one row of d_b * sum_i w_i q_i (w exact, double). */
static double orc_dot_a8(const double *w, const int8_t *q, const float *d, int n)
{
    double acc = 0.0;
    for (int b = 0; b < n / ORC_QK; b++) {
        double s = 0.0;
        for (int i = 0; i < ORC_QK; i++) s += w[b * ORC_QK + i] * (double)q[b * ORC_QK + i];
        acc += (double)d[b] * s;
    }
    return acc;
}

/* One expert with 8-bit activations: a, u from the quantized x; h = silu(a)
 * u in double, rounded to fp32 and quantized per block; Y = W_down h^.
 * If Bd != NULL, Bd[d] = sum over h elements f whose scaled value h_f * id
 * lies within eps (in code units) of a rounding boundary (k + 1/2) of
 * dh * |W_down[d, f]|: what one code step of such an element, which an fp32
 * computation of h may round the other way, can move Y[d]. */
static void orc_expert_ffn_row_a8(const int8_t *qx, const float *dx, const uint8_t *gate,
                                  const uint8_t *up, const uint8_t *down, int qtype, int D,
                                  int F, double *wrow, float *hf, int8_t *qh, float *dh,
                                  double *Y, double eps, double *Bd)
{
    size_t gate_row = orc_row_bytes(qtype, D);
    size_t down_row = orc_row_bytes(qtype, F);
    for (int r = 0; r < F; r++) {
        orc_dequant_row(gate + r * gate_row, qtype, D, wrow);
        double a = orc_dot_a8(wrow, qx, dx, D);
        orc_dequant_row(up + r * gate_row, qtype, D, wrow);
        double u = orc_dot_a8(wrow, qx, dx, D);
        hf[r] = (float)(orc_silu(a) * u);
    }
    orc_quantize_act8(hf, F, qh, dh);
    for (int d = 0; d < D; d++) {
        orc_dequant_row(down + d * down_row, qtype, F, wrow);
        Y[d] = orc_dot_a8(wrow, qh, dh, F);
        if (Bd) {
            double bsum = 0.0;
            for (int f = 0; f < F; f++) {
                float db = dh[f / ORC_QK];
                float id = (db != 0.0f) ? 1.0f / db : 0.0f;
                double sc = (double)(hf[f] * id);
                double dist = fabs(sc - (floor(sc) + 0.5));
                if (dist < eps) bsum += (double)db * fabs(wrow[f]);
            }
            Bd[d] = bsum;
        }
    }
}

/* The routed layer with 8-bit activations into every expert matmul: x_t
 * quantized per block (orc_quantize_act8), each expert as above, y_t =
 * sum_j g_tj Y_tj (+ the shared expert's Y, weight 1).  Arguments as
 * orc_layer (no dense form; D, F, sh_F multiples of 32 and of the types'
 * blocks).  bound[n_tok, D] (NULL: not wanted) = sum_j g_tj Bd_tj (+ the
 * shared Bd) for the given eps. */
int orc_layer_a8(const float *x, int T, int D, int F, int E, int k, int qtype,
                 const uint8_t *gate, const uint8_t *up, const uint8_t *down,
                 const int32_t *ids, const double *gates,
                 const uint8_t *sh_gate, const uint8_t *sh_up,
                 const uint8_t *sh_down, int sh_F, int sh_qtype,
                 const int32_t *tok_list, int n_tok, int nthreads, double eps,
                 double *y, double *bound)
{
    int bw = orc_block_weights(qtype);
    if (bw == 0 || D % bw || F % bw || k > E || D % ORC_QK || F % ORC_QK) return -1;
    if (sh_gate && (orc_block_weights(sh_qtype) == 0 || D % orc_block_weights(sh_qtype) ||
                    sh_F % orc_block_weights(sh_qtype) || sh_F % ORC_QK))
        return -1;
    if (!tok_list) n_tok = T;
    size_t gstride = orc_expert_stride(F, D, qtype);
    size_t dstride = orc_expert_stride(D, F, qtype);
    int maxF = F > sh_F ? F : sh_F;
    int maxW = D > maxF ? D : maxF;
    int bad = 0;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
#endif
    for (int n = 0; n < n_tok; n++) {
        int t = tok_list ? tok_list[n] : n;
        if (t < 0 || t >= T) { bad |= 1; continue; }
        int8_t *qx = (int8_t *)malloc((size_t)D);
        float *dx = (float *)malloc(sizeof(float) * (size_t)(D / ORC_QK));
        double *wrow = (double *)malloc(sizeof(double) * (size_t)maxW);
        float *hf = (float *)malloc(sizeof(float) * (size_t)maxF);
        int8_t *qh = (int8_t *)malloc((size_t)maxF);
        float *dh = (float *)malloc(sizeof(float) * (size_t)(maxF / ORC_QK));
        double *Y = (double *)malloc(sizeof(double) * (size_t)D);
        double *Bd = bound ? (double *)malloc(sizeof(double) * (size_t)D) : NULL;
        double *yt = y + (size_t)n * D;
        double *bt = bound ? bound + (size_t)n * D : NULL;
        orc_quantize_act8(x + (size_t)t * D, D, qx, dx);
        for (int i = 0; i < D; i++) { yt[i] = 0.0; if (bt) bt[i] = 0.0; }
        for (int j = 0; j < k; j++) {
            int e = ids[(size_t)t * k + j];
            if (e < 0 || e >= E) { bad |= 1; break; }
            orc_expert_ffn_row_a8(qx, dx, gate + e * gstride, up + e * gstride,
                                  down + e * dstride, qtype, D, F, wrow, hf, qh, dh, Y, eps, Bd);
            double g = gates[(size_t)t * k + j];
            for (int i = 0; i < D; i++) {
                yt[i] += g * Y[i];
                if (bt) bt[i] += fabs(g) * Bd[i];
            }
        }
        if (sh_gate) {
            orc_expert_ffn_row_a8(qx, dx, sh_gate, sh_up, sh_down, sh_qtype, D, sh_F, wrow, hf,
                                  qh, dh, Y, eps, Bd);
            for (int i = 0; i < D; i++) {
                yt[i] += Y[i];
                if (bt) bt[i] += Bd[i];
            }
        }
        free(qx); free(dx); free(wrow); free(hf); free(qh); free(dh); free(Y); free(Bd);
    }
    return bad ? -1 : 0;
}

/* ------------------------------------------------------------------------
 * Expert-cache LRU simulation (one layer).
 *
 * Rules (the pages name LRU replacement only; these fill in the rest):
 *  - n_slots device slots, all empty at start;
 *  - a request is a list of distinct expert ids for one step; it fails
 *    (returns -2) if it holds more ids than slots, -1 on a bad id;
 *  - every requested expert is stamped with the step number;
 *  - ids are served in the order given; a resident id is a hit;
 *  - a missing id takes the empty slot of lowest index if there is one,
 *    otherwise evicts the resident expert with the oldest stamp that is not
 *    requested in this step, the lower expert id on equal stamps.
 * Outputs per requested id: slot[i], miss[i] (0/1), evicted[i] (expert id
 * evicted to make room, or -1).  Returns the number of misses.
 * ------------------------------------------------------------------------ */
typedef struct {
    int E, n_slots;
    int64_t step;
    int32_t *slot_expert;   /* [n_slots], -1 = empty */
    int32_t *expert_slot;   /* [E], -1 = not resident */
    int64_t *stamp;         /* [E] */
} orc_lru;

void *orc_lru_new(int E, int n_slots)
{
    orc_lru *c = (orc_lru *)calloc(1, sizeof(orc_lru));
    c->E = E; c->n_slots = n_slots; c->step = 0;
    c->slot_expert = (int32_t *)malloc(sizeof(int32_t) * (size_t)n_slots);
    c->expert_slot = (int32_t *)malloc(sizeof(int32_t) * (size_t)E);
    c->stamp = (int64_t *)calloc((size_t)E, sizeof(int64_t));
    for (int s = 0; s < n_slots; s++) c->slot_expert[s] = -1;
    for (int e = 0; e < E; e++) c->expert_slot[e] = -1;
    return c;
}

void orc_lru_free(void *p)
{
    orc_lru *c = (orc_lru *)p;
    if (!c) return;
    free(c->slot_expert); free(c->expert_slot); free(c->stamp); free(c);
}

int orc_lru_request(void *p, const int32_t *ids, int n, int32_t *slot,
                    int32_t *miss, int32_t *evicted)
{
    orc_lru *c = (orc_lru *)p;
    if (n > c->n_slots) return -2;
    for (int i = 0; i < n; i++) {
        if (ids[i] < 0 || ids[i] >= c->E) return -1;
        for (int j = 0; j < i; j++) if (ids[j] == ids[i]) return -1;
    }
    c->step++;
    char *wanted = (char *)calloc((size_t)c->E, 1);
    for (int i = 0; i < n; i++) wanted[ids[i]] = 1;
    int misses = 0;
    for (int i = 0; i < n; i++) {
        int e = ids[i];
        evicted[i] = -1;
        if (c->expert_slot[e] >= 0) {
            slot[i] = c->expert_slot[e];
            miss[i] = 0;
        } else {
            int s = -1;
            for (int q = 0; q < c->n_slots; q++)
                if (c->slot_expert[q] < 0) { s = q; break; }
            if (s < 0) {
                int victim = -1;
                for (int v = 0; v < c->E; v++) {
                    if (c->expert_slot[v] < 0 || wanted[v]) continue;
                    if (victim < 0 || c->stamp[v] < c->stamp[victim]) victim = v;
                }
                s = c->expert_slot[victim];
                c->expert_slot[victim] = -1;
                evicted[i] = victim;
            }
            c->slot_expert[s] = e;
            c->expert_slot[e] = s;
            slot[i] = s;
            miss[i] = 1;
            misses++;
        }
        c->stamp[e] = c->step;
    }
    free(wanted);
    return misses;
}

/* ------------------------------------------------------------------------
 * Expert-cache LRU simulation, global across layers, with run-time resize
 * (FreeToken fork README, "About": global LRU expert caching, and
 * "Elastic Memory Management": run-time re-allocation of the expert cache's
 * VRAM; FreeToken wiki explainer: shared LRU expert caching, elastic cache
 * resizing; kongchang article, "Dynamic Cache Adjustment Experiments").
 *
 * Rules (the pages name a global LRU and resizing only; these fill in the
 * rest, and reduce to orc_lru_request when there is one layer):
 *  - one pool of max_slots device slots shared by every layer; the first
 *    `cap` of them are in use (the capacity), all empty at start;
 *  - an entry is (layer, expert), keyed layer * E + expert;
 *  - a request is a list of distinct expert ids of one layer for one step;
 *    it fails (returns -2) if it holds more ids than the capacity, -1 on a
 *    bad id or layer; one step counter serves every layer;
 *  - every requested entry is stamped with the step number;
 *  - ids are served in the order given; a resident entry is a hit;
 *  - a missing entry takes the empty slot of lowest index below cap if
 *    there is one, otherwise evicts the resident entry with the oldest stamp
 *    among all layers that is not requested in this step (entries of the
 *    same layer and id), the lower key on equal stamps;
 *  - resize to a capacity c (1 <= c <= max_slots): a larger c only adds
 *    empty slots; a smaller c first evicts, oldest stamp first (lower key on
 *    equal stamps), until at most c entries are resident, then moves every
 *    entry held in a slot >= c, in increasing slot order, to the empty slot
 *    of lowest index below c.
 * Outputs of a request per id: slot[i], miss[i], evicted[i] (key of the
 * entry evicted to make room, or -1); returns the number of misses.
 * Outputs of a resize: the keys evicted (in order, *n_evicted of them) and
 * the moves as (from, to) slot pairs (in order, *n_moves of them).
 * ------------------------------------------------------------------------ */
typedef struct {
    int n_layers, E, max_slots, cap;
    int64_t step;
    int32_t *slot_key;      /* [max_slots], -1 = empty */
    int32_t *key_slot;      /* [n_layers * E], -1 = not resident */
    int64_t *stamp;         /* [n_layers * E] */
} orc_glru;

void *orc_glru_new(int n_layers, int E, int max_slots, int cap)
{
    if (n_layers <= 0 || E <= 0 || max_slots <= 0 || cap <= 0 || cap > max_slots) return NULL;
    orc_glru *c = (orc_glru *)calloc(1, sizeof(orc_glru));
    size_t nk = (size_t)n_layers * (size_t)E;
    c->n_layers = n_layers; c->E = E; c->max_slots = max_slots; c->cap = cap; c->step = 0;
    c->slot_key = (int32_t *)malloc(sizeof(int32_t) * (size_t)max_slots);
    c->key_slot = (int32_t *)malloc(sizeof(int32_t) * nk);
    c->stamp = (int64_t *)calloc(nk, sizeof(int64_t));
    for (int s = 0; s < max_slots; s++) c->slot_key[s] = -1;
    for (size_t k = 0; k < nk; k++) c->key_slot[k] = -1;
    return c;
}

void orc_glru_free(void *p)
{
    orc_glru *c = (orc_glru *)p;
    if (!c) return;
    free(c->slot_key); free(c->key_slot); free(c->stamp); free(c);
}

/* The resident entry with the oldest stamp (lower key on equal stamps),
 * skipping entries of `layer` whose id is marked in `wanted` (NULL: none). */
static int glru_oldest(const orc_glru *c, int layer, const char *wanted)
{
    int best = -1;
    int nk = c->n_layers * c->E;
    for (int k = 0; k < nk; k++) {
        if (c->key_slot[k] < 0) continue;
        if (wanted && k / c->E == layer && wanted[k % c->E]) continue;
        if (best < 0 || c->stamp[k] < c->stamp[best]) best = k;
    }
    return best;
}

int orc_glru_request(void *p, int layer, const int32_t *ids, int n, int32_t *slot,
                     int32_t *miss, int32_t *evicted)
{
    orc_glru *c = (orc_glru *)p;
    if (layer < 0 || layer >= c->n_layers) return -1;
    if (n > c->cap) return -2;
    for (int i = 0; i < n; i++) {
        if (ids[i] < 0 || ids[i] >= c->E) return -1;
        for (int j = 0; j < i; j++) if (ids[j] == ids[i]) return -1;
    }
    c->step++;
    char *wanted = (char *)calloc((size_t)c->E, 1);
    for (int i = 0; i < n; i++) wanted[ids[i]] = 1;
    int misses = 0;
    for (int i = 0; i < n; i++) {
        int key = layer * c->E + ids[i];
        evicted[i] = -1;
        if (c->key_slot[key] >= 0) {
            slot[i] = c->key_slot[key];
            miss[i] = 0;
        } else {
            int s = -1;
            for (int q = 0; q < c->cap; q++)
                if (c->slot_key[q] < 0) { s = q; break; }
            if (s < 0) {
                int victim = glru_oldest(c, layer, wanted);
                s = c->key_slot[victim];
                c->key_slot[victim] = -1;
                evicted[i] = victim;
            }
            c->slot_key[s] = key;
            c->key_slot[key] = s;
            slot[i] = s;
            miss[i] = 1;
            misses++;
        }
        c->stamp[key] = c->step;
    }
    free(wanted);
    return misses;
}

int orc_glru_resize(void *p, int cap, int32_t *evicted, int *n_evicted, int32_t *moves,
                    int *n_moves)
{
    orc_glru *c = (orc_glru *)p;
    *n_evicted = 0;
    *n_moves = 0;
    if (cap < 1 || cap > c->max_slots) return -1;
    if (cap < c->cap) {
        int resident = 0;
        for (int s = 0; s < c->cap; s++) if (c->slot_key[s] >= 0) resident++;
        while (resident > cap) {
            int victim = glru_oldest(c, -1, NULL);
            c->slot_key[c->key_slot[victim]] = -1;
            c->key_slot[victim] = -1;
            evicted[(*n_evicted)++] = victim;
            resident--;
        }
        for (int s = cap; s < c->cap; s++) {
            int key = c->slot_key[s];
            if (key < 0) continue;
            int d = -1;
            for (int q = 0; q < cap; q++)
                if (c->slot_key[q] < 0) { d = q; break; }
            c->slot_key[d] = key;
            c->slot_key[s] = -1;
            c->key_slot[key] = d;
            moves[2 * *n_moves] = s;
            moves[2 * *n_moves + 1] = d;
            (*n_moves)++;
        }
    }
    c->cap = cap;
    return 0;
}
