/*
 * CSA2 sparse global attention over an NVFP4 main-KV cache -- CPU ORACLE.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the slow, plain, obviously-correct
 * statement of what the hot path computes.  Only the tests, the package's
 * smoke check and the CPU-baseline leg of the benchmark may load it.  It shares
 * no code, header, table or helper with the CUDA library, and the product path
 * never calls it.
 *
 * Sources (titles of the pages and the section each step follows):
 *  [P1] "DeepSeek lanca V4.1-Flash com contexto de um milhao de tokens..."
 *       (conexaotc.com.br), untitled paragraphs 5-6: CSA2 modes Full /
 *       Reindex / Reuse, Top-512, the hierarchical indexer of up to 2048
 *       blocks of 8 (16,384 positions), and the main KV stored as E2M1 with
 *       one E4M3 scale per 16 channels, NVFP4 without its global scale.
 *  [P4] "O que os autores propoem" / "Como funciona" (e-cogni.com.br):
 *       Reindex re-scores the shared indexer K with its own indexer Q; Reuse
 *       re-uses the global KV and the Top-K indices and runs sparse attention
 *       directly; every layer keeps its own global Q and its own SWA KV.
 *  [P5] "Atencion escasa comprimida 2 (CSA2)" and "FP4 KV, repeticion
 *       limitada..." (7minutos.es): same facts; 128-token SWA window in every
 *       layer ("Codificador-decodificador causal").
 *
 * The pages fix neither the score function, the head sizes, the softmax scale,
 * rounding, nor tie-breaking.  The workload statement fixes: 16 query heads of
 * dim 128 sharing one 128-d K and one 128-d V (MQA); indexer 4 heads x 64 with
 * score = sum_h w_h * ReLU(q_h . k); ratio 2 = mean of adjacent token pairs;
 * mean-pooled indexer K per 8-token block; log-sum-exp merge with the bf16
 * 128-token SWA; ties to the lower index.  Everything else is a stated reading:
 *
 *   R1  E4M3 is the OCP "e4m3fn" format (bias 7, no inf, 0x7F/0xFF NaN, max
 *       448); E2M1 has magnitudes {0,.5,1,1.5,2,3,4,6}, sign in bit 3.
 *   R2  block scale s = E4M3_RNE_satfinite(amax / 6) with an fp32 division;
 *       code = E2M1_RNE_satfinite(x / s), fp32 division, sign bit copied from
 *       x (so small negatives encode -0 = 0x8); if s decodes to 0 every code is
 *       0x0.
 *   R3  byte j of an entry packs channel 2j in the low nibble, 2j+1 high.
 *   R4  ratio 2: y = (x_2j + x_2j+1) * 0.5f, then R2.
 *   R5  pooled indexer K of block j = bf16_RNE(fp32 sequential sum of the
 *       rows present / n), n = rows present (8, or fewer in the last block).
 *   R6  dot_h = sequential fp32 fused multiply-add over d = 0..63;
 *       score = sequential fp32 FMA over h of w_h * max(dot_h, 0).  No scale.
 *   R7  Top-K by (score desc, index asc), output ascending, -1 padded.
 *   R8  decoder: if ceil(L/8) <= 2048 every block is a candidate, else the
 *       Top-2048 blocks; Reindex scores the Full layer's candidates of the
 *       same step with its own indexer Q (no new block selection).
 *   R9  attention logits (q . k) / sqrt(128); no RoPE, no sink; the selected
 *       set and the window are NOT de-duplicated; two branches merged by LSE.
 *   R10 decode window = last min(128, L) tokens including the current one;
 *       prefill window of the query at p = tokens [max(0, p-127), p]; entry j
 *       is visible to query p iff (j+1)*ratio - 1 <= p.
 *   R12 SWA Bounded Replay: a layer's window K|V row of a token is bf16(h . W)
 *       with h the token's hidden state and W the layer's K|V projection
 *       (synthetic here: the pages' weights are not available).
 *   R11 the pages place the hierarchical indexer in the decoder only; the
 *       encoder's Full layers (ratio 2) select their Top-512 over every entry
 *       of the context ("flat"), as its prefill does.  A decode step with
 *       keep = 0 has no block level: a Full (or Reindex) layer takes the
 *       Top-K over all L entries.
 *
 * Floating point: where a float decides an integer (codes, scales, pooled
 * bf16, scores deciding Top-K membership) the oracle works in fp32, the
 * precision the kernels decide in; the attention outputs are computed in fp64.
 * Build: gcc -O2 -ffp-contract=off -fopenmp (no fast-math).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------ */
/* Number formats (R1)                                                */
/* ------------------------------------------------------------------ */

float orc_bf16_to_f32(uint16_t h) {
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

/* Round-to-nearest-even fp32 -> bf16 (textbook: add 0x7FFF + lsb, truncate). */
uint16_t orc_f32_to_bf16(float x) {
    uint32_t u;
    memcpy(&u, &x, 4);
    if ((u & 0x7FFFFFFFu) > 0x7F800000u) return (uint16_t)((u >> 16) | 0x40u);
    u += 0x7FFFu + ((u >> 16) & 1u);
    return (uint16_t)(u >> 16);
}

/* E4M3 (fn): sign | 4-bit exponent, bias 7 | 3-bit mantissa. */
double orc_e4m3_value(uint8_t b) {
    int sign = (b >> 7) & 1;
    int e = (b >> 3) & 0xF;
    int m = b & 7;
    double v;
    if (e == 0xF && m == 7) return NAN;
    if (e == 0) v = ldexp((double)m / 8.0, -6);
    else v = ldexp(1.0 + (double)m / 8.0, e - 7);
    return sign ? -v : v;
}

/* Nearest E4M3 value, ties to even mantissa, saturating at 448. */
uint8_t orc_e4m3_encode(float xf) {
    if (isnan(xf)) return 0x7F;
    uint8_t sign = signbit(xf) ? 0x80 : 0x00;
    double a = fabs((double)xf);
    if (a >= 448.0) return sign | 0x7E;
    int e2;
    frexp(a, &e2);
    int E = e2 - 1;            /* a in [2^E, 2^(E+1)) */
    if (a == 0.0 || E < -6) E = -6; /* subnormals share the quantum 2^-9 */
    double quantum = ldexp(1.0, E - 3);
    double n = nearbyint(a / quantum); /* exact quotient; ties to even */
    double v = n * quantum;
    if (v == 0.0) return sign;
    frexp(v, &e2);
    E = e2 - 1;
    if (E < -6) {                      /* subnormal: v = m * 2^-9 */
        int m = (int)(v / ldexp(1.0, -9));
        return sign | (uint8_t)m;
    }
    int m = (int)(v / ldexp(1.0, E) * 8.0) - 8;
    return sign | (uint8_t)(((E + 7) << 3) | m);
}

/* E2M1: sign bit 3 | 2-bit exponent, bias 1 | 1-bit mantissa. */
double orc_e2m1_value(uint8_t c) {
    static const double mag[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};
    double v = mag[c & 7];
    return (c & 8) ? -v : v;
}

/* Nearest E2M1 value, ties to even code, saturating at 6, sign copied. */
uint8_t orc_e2m1_encode(float yf) {
    uint8_t sign = signbit(yf) ? 0x8 : 0x0;
    double a = fabs((double)yf);
    if (isnan(yf)) return sign | 0x7; /* not reached for finite inputs */
    double quantum = (a < 2.0) ? 0.5 : (a < 4.0 ? 1.0 : 2.0);
    double v = nearbyint(a / quantum) * quantum;
    if (v > 6.0) v = 6.0;
    uint8_t code;
    if (v == 0.0) code = 0;
    else if (v == 0.5) code = 1;
    else if (v == 1.0) code = 2;
    else if (v == 1.5) code = 3;
    else if (v == 2.0) code = 4;
    else if (v == 3.0) code = 5;
    else if (v == 4.0) code = 6;
    else code = 7; /* 6.0 */
    return sign | code;
}

/* vectorised forms (for exhaustive pins) */
void orc_e4m3_encode_n(const float* x, uint8_t* out, int64_t n) {
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) out[i] = orc_e4m3_encode(x[i]);
}
void orc_e2m1_encode_n(const float* x, uint8_t* out, int64_t n) {
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) out[i] = orc_e2m1_encode(x[i]);
}
void orc_f32_to_bf16_n(const float* x, uint16_t* out, int64_t n) {
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) out[i] = orc_f32_to_bf16(x[i]);
}

/* ------------------------------------------------------------------ */
/* FP4 main-KV entry: 256 channels (K = 0..127, V = 128..255)  (R2,R3) */
/* ------------------------------------------------------------------ */

#define ORC_CH 256
#define ORC_CODE_BYTES 128
#define ORC_SCALES 16

void orc_quant_entry(const float* x, uint8_t* codes, uint8_t* scales) {
    for (int b = 0; b < ORC_SCALES; ++b) {
        const float* xb = x + 16 * b;
        float amax = 0.0f;
        for (int i = 0; i < 16; ++i) {
            float a = fabsf(xb[i]);
            if (a > amax) amax = a;
        }
        uint8_t sb = orc_e4m3_encode(amax / 6.0f);
        scales[b] = sb;
        float s = (float)orc_e4m3_value(sb);
        uint8_t c[16];
        for (int i = 0; i < 16; ++i) c[i] = (s == 0.0f) ? 0 : orc_e2m1_encode(xb[i] / s);
        for (int j = 0; j < 8; ++j) codes[8 * b + j] = (uint8_t)(c[2 * j] | (c[2 * j + 1] << 4));
    }
}

/* x_hat = e2m1(code) * e4m3(scale), exact in double. */
void orc_dequant_entry(const uint8_t* codes, const uint8_t* scales, double* x) {
    for (int ch = 0; ch < ORC_CH; ++ch) {
        uint8_t byte = codes[ch >> 1];
        uint8_t c = (ch & 1) ? (byte >> 4) : (byte & 0xF);
        x[ch] = orc_e2m1_value(c) * orc_e4m3_value(scales[ch >> 4]);
    }
}

/* n entries from n*ratio fp32 source rows (R4).  Parallel over entries. */
void orc_quant_rows(const float* src, int64_t n, int ratio, uint8_t* codes, uint8_t* scales) {
#pragma omp parallel for schedule(static)
    for (int64_t e = 0; e < n; ++e) {
        float y[ORC_CH];
        if (ratio == 2) {
            const float* a = src + (2 * e) * ORC_CH;
            const float* b = src + (2 * e + 1) * ORC_CH;
            for (int ch = 0; ch < ORC_CH; ++ch) y[ch] = (a[ch] + b[ch]) * 0.5f;
        } else {
            memcpy(y, src + e * ORC_CH, sizeof(y));
        }
        orc_quant_entry(y, codes + e * ORC_CODE_BYTES, scales + e * ORC_SCALES);
    }
}

/* ------------------------------------------------------------------ */
/* Indexer (R5, R6)                                                   */
/* ------------------------------------------------------------------ */

#define ORC_IH 4
#define ORC_ID 64

/* Pooled indexer K of every block of a sequence of L rows: [ceil(L/8)][64]. */
void orc_pool_blocks(const uint16_t* idx_k, int64_t L, uint16_t* pooled) {
    int64_t nblk = (L + 7) / 8;
#pragma omp parallel for schedule(static)
    for (int64_t j = 0; j < nblk; ++j) {
        int64_t r0 = 8 * j;
        int n = (int)((L - r0) < 8 ? (L - r0) : 8);
        for (int d = 0; d < ORC_ID; ++d) {
            float acc = 0.0f;
            for (int r = 0; r < n; ++r) acc = acc + orc_bf16_to_f32(idx_k[(r0 + r) * ORC_ID + d]);
            pooled[j * ORC_ID + d] = orc_f32_to_bf16(acc / (float)n);
        }
    }
}

float orc_score(const uint16_t* q, const float* w, const uint16_t* k) {
    float s = 0.0f;
    for (int h = 0; h < ORC_IH; ++h) {
        float dot = 0.0f;
        for (int d = 0; d < ORC_ID; ++d)
            dot = fmaf(orc_bf16_to_f32(q[h * ORC_ID + d]), orc_bf16_to_f32(k[d]), dot);
        float r = dot > 0.0f ? dot : 0.0f;
        s = fmaf(w[h], r, s);
    }
    return s;
}

void orc_score_rows(const uint16_t* q, const float* w, const uint16_t* rows, int64_t n, float* out) {
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) out[i] = orc_score(q, w, rows + i * ORC_ID);
}

/* ------------------------------------------------------------------ */
/* Top-K (R7)                                                         */
/* ------------------------------------------------------------------ */

typedef struct { float s; int64_t i; } orc_pair;

static int orc_cmp_rank(const void* pa, const void* pb) {
    const orc_pair* a = (const orc_pair*)pa;
    const orc_pair* b = (const orc_pair*)pb;
    if (a->s > b->s) return -1;
    if (a->s < b->s) return 1;
    return (a->i < b->i) ? -1 : (a->i > b->i);
}

static int orc_cmp_i32(const void* pa, const void* pb) {
    int32_t a = *(const int32_t*)pa, b = *(const int32_t*)pb;
    return (a < b) ? -1 : (a > b);
}

/* ids[i] is the label of scores[i].  Writes the labels of the Top-k ranked
 * items, ascending, then -1 up to k_out. Returns the number selected. */
int64_t orc_topk_labels(const float* scores, const int32_t* ids, int64_t n, int64_t k, int32_t* out,
                        int64_t k_out) {
    orc_pair* p = (orc_pair*)malloc(sizeof(orc_pair) * (n > 0 ? n : 1));
    for (int64_t i = 0; i < n; ++i) {
        p[i].s = scores[i];
        p[i].i = ids ? ids[i] : i;
    }
    qsort(p, (size_t)n, sizeof(orc_pair), orc_cmp_rank);
    int64_t m = n < k ? n : k;
    for (int64_t i = 0; i < m; ++i) out[i] = (int32_t)p[i].i;
    qsort(out, (size_t)m, sizeof(int32_t), orc_cmp_i32);
    for (int64_t i = m; i < k_out; ++i) out[i] = -1;
    free(p);
    return m;
}

/* ------------------------------------------------------------------ */
/* Decoder indexer for one sequence (R8)                              */
/* ------------------------------------------------------------------ */

/* Candidate blocks of the Full layer: all blocks when ceil(L/8) <= keep, else
 * the Top-keep blocks by pooled score.  out_blocks[keep] ascending, -1 pad.
 * If block_scores is non-null it receives the ceil(L/8) pooled scores. */
int64_t orc_select_blocks(const uint16_t* pooled, int64_t L, const uint16_t* q, const float* w, int64_t keep,
                          int32_t* out_blocks, float* block_scores) {
    int64_t nblk = (L + 7) / 8;
    float* s = (float*)malloc(sizeof(float) * (nblk > 0 ? nblk : 1));
    orc_score_rows(q, w, pooled, nblk, s);
    if (block_scores) memcpy(block_scores, s, sizeof(float) * nblk);
    int64_t m;
    if (nblk <= keep) {
        for (int64_t j = 0; j < nblk; ++j) out_blocks[j] = (int32_t)j;
        for (int64_t j = nblk; j < keep; ++j) out_blocks[j] = -1;
        m = nblk;
    } else {
        m = orc_topk_labels(s, NULL, nblk, keep, out_blocks, keep);
    }
    free(s);
    return m;
}

/* Token Top-K among the candidate positions of the given blocks (ascending,
 * -1 terminated), or among all L positions when blocks is NULL. */
int64_t orc_select_tokens(const uint16_t* idx_k, int64_t L, const int32_t* blocks, int64_t nblocks,
                          const uint16_t* q, const float* w, int64_t topk, int32_t* out_idx,
                          float* cand_scores, int32_t* cand_pos, int64_t* n_cand) {
    int64_t cap = blocks ? 8 * nblocks : L;
    int32_t* pos = (int32_t*)malloc(sizeof(int32_t) * (cap > 0 ? cap : 1));
    int64_t c = 0;
    if (blocks) {
        for (int64_t b = 0; b < nblocks && blocks[b] >= 0; ++b)
            for (int64_t t = 8 * (int64_t)blocks[b]; t < 8 * (int64_t)blocks[b] + 8 && t < L; ++t)
                pos[c++] = (int32_t)t;
    } else {
        for (int64_t t = 0; t < L; ++t) pos[c++] = (int32_t)t;
    }
    float* s = (float*)malloc(sizeof(float) * (c > 0 ? c : 1));
    for (int64_t i = 0; i < c; ++i) s[i] = orc_score(q, w, idx_k + (int64_t)pos[i] * ORC_ID);
    int64_t m = orc_topk_labels(s, pos, c, topk, out_idx, topk);
    if (cand_scores) memcpy(cand_scores, s, sizeof(float) * c);
    if (cand_pos) memcpy(cand_pos, pos, sizeof(int32_t) * c);
    if (n_cand) *n_cand = c;
    free(s);
    free(pos);
    return m;
}

/* ------------------------------------------------------------------ */
/* Attention (R9, R10), fp64                                          */
/* ------------------------------------------------------------------ */

#define ORC_H 16
#define ORC_D 128

/* One softmax branch for all 16 heads over n keys (K, V as [n][128] double).
 * n == 0 gives lse = -inf and a zero output. */
static void orc_branch(const double* q, int64_t n, const double* K, const double* V, double* o, double* lse) {
    const double scale = 1.0 / sqrt((double)ORC_D);
    double* z = (double*)malloc(sizeof(double) * (n > 0 ? n : 1));
    for (int h = 0; h < ORC_H; ++h) {
        double m = -INFINITY;
        for (int64_t j = 0; j < n; ++j) {
            double dot = 0.0;
            for (int d = 0; d < ORC_D; ++d) dot += q[h * ORC_D + d] * K[j * ORC_D + d];
            z[j] = dot * scale;
            if (z[j] > m) m = z[j];
        }
        double l = 0.0;
        for (int d = 0; d < ORC_D; ++d) o[h * ORC_D + d] = 0.0;
        if (n == 0) { lse[h] = -INFINITY; continue; }
        for (int64_t j = 0; j < n; ++j) {
            double p = exp(z[j] - m);
            l += p;
            for (int d = 0; d < ORC_D; ++d) o[h * ORC_D + d] += p * V[j * ORC_D + d];
        }
        for (int d = 0; d < ORC_D; ++d) o[h * ORC_D + d] /= l;
        lse[h] = m + log(l);
    }
    free(z);
}

/* o = (e^l1 o1 + e^l2 o2) / (e^l1 + e^l2),  lse = log(e^l1 + e^l2). */
static void orc_lse_merge(const double* o1, const double* l1, const double* o2, const double* l2, float* out,
                          float* lse) {
    for (int h = 0; h < ORC_H; ++h) {
        double m = l1[h] > l2[h] ? l1[h] : l2[h];
        double a = (l1[h] == -INFINITY) ? 0.0 : exp(l1[h] - m);
        double b = (l2[h] == -INFINITY) ? 0.0 : exp(l2[h] - m);
        for (int d = 0; d < ORC_D; ++d)
            out[h * ORC_D + d] = (float)((a * o1[h * ORC_D + d] + b * o2[h * ORC_D + d]) / (a + b));
        lse[h] = (float)(m + log(a + b));
    }
}

/* Sparse branch over the selected entries (idx -1 skipped) plus the SWA
 * branch over n_swa bf16 tokens [n_swa][256] (K = 0..127, V = 128..255).
 * codes/scales are indexed by entry position. */
void orc_attend(const uint16_t* q_bf16, const int32_t* idx, int64_t k, const uint8_t* codes,
                const uint8_t* scales, const uint16_t* swa, int64_t n_swa, float* out, float* lse) {
    double q[ORC_H * ORC_D];
    for (int i = 0; i < ORC_H * ORC_D; ++i) q[i] = orc_bf16_to_f32(q_bf16[i]);
    int64_t n = 0;
    for (int64_t i = 0; i < k; ++i) n += idx[i] >= 0;
    double* K1 = (double*)malloc(sizeof(double) * ORC_D * (n > 0 ? n : 1));
    double* V1 = (double*)malloc(sizeof(double) * ORC_D * (n > 0 ? n : 1));
    double row[ORC_CH];
    int64_t r = 0;
    for (int64_t i = 0; i < k; ++i) {
        if (idx[i] < 0) continue;
        orc_dequant_entry(codes + (int64_t)idx[i] * ORC_CODE_BYTES, scales + (int64_t)idx[i] * ORC_SCALES, row);
        memcpy(K1 + r * ORC_D, row, sizeof(double) * ORC_D);
        memcpy(V1 + r * ORC_D, row + ORC_D, sizeof(double) * ORC_D);
        ++r;
    }
    double* K2 = (double*)malloc(sizeof(double) * ORC_D * (n_swa > 0 ? n_swa : 1));
    double* V2 = (double*)malloc(sizeof(double) * ORC_D * (n_swa > 0 ? n_swa : 1));
    for (int64_t j = 0; j < n_swa; ++j)
        for (int d = 0; d < ORC_D; ++d) {
            K2[j * ORC_D + d] = orc_bf16_to_f32(swa[j * ORC_CH + d]);
            V2[j * ORC_D + d] = orc_bf16_to_f32(swa[j * ORC_CH + ORC_D + d]);
        }
    double o1[ORC_H * ORC_D], o2[ORC_H * ORC_D], l1[ORC_H], l2[ORC_H];
    orc_branch(q, n, K1, V1, o1, l1);
    orc_branch(q, n_swa, K2, V2, o2, l2);
    orc_lse_merge(o1, l1, o2, l2, out, lse);
    free(K1); free(V1); free(K2); free(V2);
}

/* ------------------------------------------------------------------ */
/* Schedule (P1 paragraph 6, P4 "Como funciona")                      */
/* ------------------------------------------------------------------ */

enum { ORC_FULL = 0, ORC_REINDEX = 1, ORC_REUSE = 2 };

/* Decoder: 20 layers, 5 groups of 4: Full+3 Reuse, then (Reindex+3 Reuse) x4.
 * Encoder: 18 CSA2 layers, 3 groups of 6: Full + 5 Reuse each. */
int orc_schedule(int decoder, int32_t* modes) {
    int n = decoder ? 20 : 18, g = decoder ? 4 : 6;
    for (int l = 0; l < n; ++l) {
        if (l % g) modes[l] = ORC_REUSE;
        else modes[l] = (decoder && l > 0) ? ORC_REINDEX : ORC_FULL;
    }
    return n;
}

/* One decode step of one sequence through n_layers layers of the given modes.
 * The cache (codes, scales, idx_k, pooled) already holds the L entries,
 * including the current token.  keep = 0 selects the flat indexer (R11):
 * pooled and blocks are not used.  Per layer l: q[l] [16][128] bf16, swa[l]
 * [n_swa][256] bf16 (n_swa = min(window, L)); indexer layers also read
 * q_idx[l] [4][64] bf16 and w[l] [4].  Outputs: idx_sets[l] [topk],
 * out[l] [16][128], lse[l] [16], blocks [keep] (the Full layer's set). */
void orc_decode_step(int n_layers, const int32_t* modes, int64_t L, const uint8_t* codes, const uint8_t* scales,
                     const uint16_t* idx_k, const uint16_t* pooled, const uint16_t* q_idx, const float* w,
                     const uint16_t* q, const uint16_t* swa, int64_t window, int64_t keep, int64_t topk,
                     int32_t* blocks, int32_t* idx_sets, float* out, float* lse) {
    int64_t n_swa = L < window ? L : window;
    int32_t* cur = NULL;
    int have_blocks = 0;
    for (int l = 0; l < n_layers; ++l) {
        int32_t* set = idx_sets + (int64_t)l * topk;
        const uint16_t* qi = q_idx + (int64_t)l * ORC_IH * ORC_ID;
        const float* wl = w + (int64_t)l * ORC_IH;
        if (modes[l] != ORC_REUSE && keep == 0) {
            orc_select_tokens(idx_k, L, NULL, 0, qi, wl, topk, set, NULL, NULL, NULL);
        } else if (modes[l] == ORC_FULL) {
            orc_select_blocks(pooled, L, qi, wl, keep, blocks, NULL);
            have_blocks = 1;
            orc_select_tokens(idx_k, L, blocks, keep, qi, wl, topk, set, NULL, NULL, NULL);
        } else if (modes[l] == ORC_REINDEX) {
            if (!have_blocks) return; /* a Reindex layer needs a preceding Full layer */
            orc_select_tokens(idx_k, L, blocks, keep, qi, wl, topk, set, NULL, NULL, NULL);
        } else {
            if (!cur) return;         /* a Reuse layer needs a preceding index set */
            memcpy(set, cur, sizeof(int32_t) * topk);
        }
        cur = set;
        orc_attend(q + (int64_t)l * ORC_H * ORC_D, set, topk, codes, scales,
                   swa + (int64_t)l * window * ORC_CH, n_swa, out + (int64_t)l * ORC_H * ORC_D,
                   lse + (int64_t)l * ORC_H);
    }
}

/* Decode steps of n_seq independent sequences in parallel (for timing).
 * Per-sequence arrays are strided by the given element counts. */
void orc_decode_batch(int n_seq, int n_layers, const int32_t* modes, const int64_t* L, const uint8_t* const* codes,
                      const uint8_t* const* scales, const uint16_t* const* idx_k, const uint16_t* const* pooled,
                      const uint16_t* q_idx, const float* w, const uint16_t* q, const uint16_t* swa,
                      int64_t window, int64_t keep, int64_t topk, int32_t* blocks, int32_t* idx_sets,
                      float* out, float* lse) {
#pragma omp parallel for schedule(dynamic, 1)
    for (int b = 0; b < n_seq; ++b) {
        orc_decode_step(n_layers, modes, L[b], codes[b], scales[b], idx_k[b], pooled[b],
                        q_idx + (int64_t)b * n_layers * ORC_IH * ORC_ID, w + (int64_t)b * n_layers * ORC_IH,
                        q + (int64_t)b * n_layers * ORC_H * ORC_D, swa + (int64_t)b * n_layers * window * ORC_CH,
                        window, keep, topk, blocks + (int64_t)b * keep, idx_sets + (int64_t)b * n_layers * topk,
                        out + (int64_t)b * n_layers * ORC_H * ORC_D, lse + (int64_t)b * n_layers * ORC_H);
    }
}

/* ------------------------------------------------------------------ */
/* Prefill (flat indexer, causal visibility R10)                      */
/* ------------------------------------------------------------------ */

/* Number of entries visible to the query at absolute token position p. */
int64_t orc_visible_entries(int64_t p, int ratio, int64_t n_entries) {
    int64_t v = (p + 1) / ratio; /* largest j with (j+1)*ratio - 1 <= p, plus one */
    return v < n_entries ? v : n_entries;
}

/* Token Top-K of each query over its visible entries: q_idx [T][4][64],
 * w [T][4], out [T][topk]. */
void orc_prefill_indexer(int64_t T, const int32_t* q_pos, int ratio, int64_t n_entries, const uint16_t* idx_k,
                         const uint16_t* q_idx, const float* w, int64_t topk, int32_t* out) {
#pragma omp parallel for schedule(dynamic, 4)
    for (int64_t t = 0; t < T; ++t) {
        int64_t v = orc_visible_entries(q_pos[t], ratio, n_entries);
        orc_select_tokens(idx_k, v, NULL, 0, q_idx + t * ORC_IH * ORC_ID, w + t * ORC_IH, topk,
                          out + t * topk, NULL, NULL, NULL);
    }
}

/* Attention of each query: q [T][16][128]; idx [T][topk]; swa holds tokens
 * swa_start .. swa_start + n_swa_rows - 1 as [n_swa_rows][256]; the window
 * of the query at p is tokens [max(0, p - window + 1), p]. */
void orc_prefill_attn(int64_t T, const int32_t* q_pos, const uint16_t* q, const int32_t* idx, int64_t topk,
                      const uint8_t* codes, const uint8_t* scales, const uint16_t* swa, int64_t swa_start,
                      int64_t window, float* out, float* lse) {
#pragma omp parallel for schedule(dynamic, 4)
    for (int64_t t = 0; t < T; ++t) {
        int64_t p = q_pos[t];
        int64_t lo = p - window + 1;
        if (lo < 0) lo = 0;
        orc_attend(q + t * ORC_H * ORC_D, idx + t * topk, topk, codes, scales, swa + (lo - swa_start) * ORC_CH,
                   p - lo + 1, out + t * ORC_H * ORC_D, lse + t * ORC_H);
    }
}

/* ------------------------------------------------------------------ */
/* SWA Bounded Replay, attention part ([P5] "FP4 KV, repeticion        */
/* limitada...": on a miss only 128 tokens are recomputed; [P4] "Como   */
/* funciona": the replay avoids persisting the SWA cache)              */
/* ------------------------------------------------------------------ */

/* R12 (reading): a layer's SWA K|V row of a token is its hidden state h
 * (bf16, d_model values) times the layer's K|V projection w (bf16, 256 output
 * channels x d_model), rounded to bf16: out[t][c] = bf16_RNE(sum_k h[t][k] *
 * w[c][k]).  The sum is taken in fp64 (it decides no integer), rounded to fp32
 * and then to bf16.  h [n][d], w [256][d], out [n][256]. */
void orc_swa_replay(const uint16_t* h, const uint16_t* w, int64_t n, int64_t d, uint16_t* out) {
    for (int64_t t = 0; t < n; ++t)
        for (int c = 0; c < ORC_CH; ++c) {
            double acc = 0.0;
            for (int64_t k = 0; k < d; ++k)
                acc += (double)orc_bf16_to_f32(h[t * d + k]) * (double)orc_bf16_to_f32(w[(int64_t)c * d + k]);
            out[t * ORC_CH + c] = orc_f32_to_bf16((float)acc);
        }
}

/* ------------------------------------------------------------------ */
/* Cache accounting                                                   */
/* ------------------------------------------------------------------ */

/* Global KV bytes per token: sum over Full layers of (main-entry bytes +
 * indexer-K bytes) / ratio; Reindex and Reuse layers store nothing new. */
double orc_cache_bytes_per_token(int n_full, const int32_t* ratios, double main_entry_bytes, double idx_entry_bytes) {
    double t = 0.0;
    for (int i = 0; i < n_full; ++i) t += (main_entry_bytes + idx_entry_bytes) / (double)ratios[i];
    return t;
}
