/*
 * CPU oracle of the HiFA4-style 4-bit FlashAttention forward.
 *
 * TEST INFRASTRUCTURE ONLY. Only the tests, the smoke check and the
 * benchmark's CPU-baseline leg may load this library. The product path never
 * does, and this file shares no code, header or table with the CUDA library.
 *
 * Source of the method: "HiFA4: Training-Free 4-bit FlashAttention on Ascend
 * HIF4 NPUs for LLM Inference" (abstract, as printed on the scholarfeed,
 * hf.space, thelatestinai, fugumt and mlsanity pages). The abstract fixes the
 * shape of the method:
 *   - QK^T and PV both run as 4-bit GEMMs inside FlashAttention;
 *   - the online-softmax state is kept in a wider float format;
 *   - Smooth-QK: a calibration-static per-channel rescale, Q*s and K/s, applied
 *     after RoPE and before quantization;
 *   - P-Reordering: the softmax normalizer is accumulated from the same
 *     quantized probabilities P_hat that feed the PV GEMM, instead of from the
 *     unquantized probabilities ("high-precision reconstruction").
 * The HIF4 encoding is not on the pages. The substitute format is E2M1
 * elements with one E4M3 scale per 16 elements along the contraction
 * dimension, round-to-nearest-even, no per-tensor scale.
 *
 * Readings taken where the pages are silent (each one is listed with its
 * reason in the design notes):
 *   scale      sf = E4M3_rne_satfinite(amax * RN(1/6)), S = decode(sf)
 *   elements   r = RN(1/S) (r = 0 when S = 0), code = E2M1_rne_satfinite(RN(x*r)),
 *              the sign of x is kept, also when the code is zero
 *   smoothing  s = aK^a / aQ^(1-a) per (kv head, channel), a = 0.5 -> sqrt(aK/aQ),
 *              s = 1 when either amax is 0; Q' = RN(Q*s), K' = RN(K*RN(1/s))
 *   tiling     one pass over 128-key tiles in ascending order, running max
 *              updated every tile, P relative to the current running max
 *   softmax    c = RN(sm_scale*log2 e); mc = RN(m*c); P = RN(2^fma(S,c,-mc));
 *              P is quantized per 16 keys of its row with the element rule
 *   causal     key j is visible to query i iff j <= i + Nkv - Nq
 *   output     O = O_acc / l, LSE = mc*ln 2 + ln l (natural log)
 *   split kv   (inference option, flash-decoding) the kv tiles are cut into
 *              n_splits contiguous ranges [floor(s*T/n), floor((s+1)*T/n)); each
 *              range runs the online softmax above from its own start (its own
 *              running max, so its P_hat is relative to the range's max), and
 *              the ranges are merged with their log-sum-exp weights:
 *              O = sum_s 2^(mc_s - M) O_acc_s / sum_s 2^(mc_s - M) l_s,
 *              M = max mc_s over ranges with mass; n_splits = 1 is the plain pass
 * Every quantization decision is taken in fp32, the precision the GPU takes
 * it in. Sums and the online-softmax state are kept in fp64, which is exact for
 * the per-tile sums (all decoded operands are multiples of 2^-10 bounded by
 * 2688, so a 256-term QK sum or a 128-term PV sum needs at most 52 bits).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define TILE_KV 128

/* ---------------------------------------------------------------- E2M1 */

/* Magnitudes of the eight 3-bit E2M1 codes (1 sign bit above them). */
static const double kE2M1[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};

double ora_e2m1_decode(uint8_t code) {
    double m = kE2M1[code & 7];
    return (code & 8) ? -m : m;
}

/* Round-to-nearest-even onto the E2M1 grid, saturating at 6, sign kept.
 * The thresholds are the midpoints between neighbouring values; at an exact
 * midpoint the neighbour with an even code (mantissa bit 0) wins. */
uint8_t ora_e2m1_encode(float x) {
    uint8_t sign = signbit(x) ? 8 : 0;
    double a = fabs((double)x);
    uint8_t m;
    if (isnan(x))       m = 7;
    else if (a <= 0.25) m = 0;   /* 0.25 ties to 0   */
    else if (a < 0.75)  m = 1;   /* 0.75 ties to 1.0 */
    else if (a <= 1.25) m = 2;   /* 1.25 ties to 1.0 */
    else if (a < 1.75)  m = 3;   /* 1.75 ties to 2.0 */
    else if (a <= 2.5)  m = 4;   /* 2.5 ties to 2.0  */
    else if (a < 3.5)   m = 5;   /* 3.5 ties to 4.0  */
    else if (a <= 5.0)  m = 6;   /* 5 ties to 4.0    */
    else                m = 7;
    return (uint8_t)(sign | m);
}

/* ---------------------------------------------------------------- E4M3 */

/* E4M3 ("fn" variant): bias 7, no infinities, 0x7F/0xFF are NaN, max 448,
 * subnormals m * 2^-9. */
double ora_e4m3_decode(uint8_t code) {
    int e = (code >> 3) & 15, m = code & 7;
    double v;
    if ((code & 0x7F) == 0x7F) return NAN;
    if (e == 0) v = ldexp((double)m, -9);
    else        v = ldexp(1.0 + m / 8.0, e - 7);
    return (code & 0x80) ? -v : v;
}

uint8_t ora_e4m3_encode(float x) {
    uint8_t sign = signbit(x) ? 0x80 : 0;
    double a = fabs((double)x);
    if (isnan(x)) return 0x7F;
    if (a >= 448.0) return (uint8_t)(sign | 0x7E);          /* satfinite */
    if (a == 0.0) return sign;
    int e2;
    frexp(a, &e2);                                          /* a in [2^(e2-1), 2^e2) */
    int E = e2 - 1;
    if (E < -6) {                                           /* subnormal: quantum 2^-9 */
        double q = nearbyint(a * 512.0);                    /* ties to even */
        return (uint8_t)(sign | (uint8_t)q);                /* q = 8 is the smallest normal */
    }
    double q = nearbyint(ldexp(a, 3 - E));                  /* in [8, 16] */
    if (q == 16.0) { q = 8.0; E += 1; }
    int code = ((E + 7) << 3) | ((int)q - 8);
    if (code > 0x7E) code = 0x7E;
    return (uint8_t)(sign | code);
}

/* ------------------------------------------------- block quantization */

/* RN(1/6) in fp32 = 0x3E2AAAAB. */
static float one_sixth(void) { return (float)(1.0 / 6.0); }

static float mul_f32(float a, float b) { return (float)((double)a * (double)b); }

/* Scale code of a 16-element block from its absolute maximum. */
uint8_t ora_scale_code(float amax) {
    return ora_e4m3_encode(mul_f32(amax, one_sixth()));
}

/* Element codes of one block given its scale code (nibble codes, unpacked). */
static void encode_block(const float* x, int n, uint8_t sf, uint8_t* codes) {
    double S = ora_e4m3_decode(sf);
    float r = (S == 0.0) ? 0.0f : (float)(1.0 / S);       /* RN(1/S) */
    for (int i = 0; i < n; ++i) codes[i] = ora_e2m1_encode(mul_f32(x[i], r));
}

/* Quantize one 16-element block: scale code + 16 nibble codes. */
void ora_quant_block16(const float* x, uint8_t* codes, uint8_t* sf) {
    float amax = 0.0f;
    for (int i = 0; i < 16; ++i) {
        float a = fabsf(x[i]);
        if (a > amax) amax = a;
    }
    *sf = ora_scale_code(amax);
    encode_block(x, 16, *sf, codes);
}

/* ------------------------------------------------------- calibration */

/* Smooth-QK factors per (kv head g, channel c). q: [B,Hq,N,D], k: [B,Hkv,N,D]. */
void ora_calibrate(const float* q, const float* k, int B, int Hq, int Hkv, int N, int D,
                   float alpha, float* s, float* s_inv) {
    int G = Hq / Hkv;
    for (int g = 0; g < Hkv; ++g) {
        for (int c = 0; c < D; ++c) {
            float aq = 0.0f, ak = 0.0f;
            for (int b = 0; b < B; ++b) {
                for (int hh = 0; hh < G; ++hh) {
                    const float* qp = q + (((size_t)b * Hq + (size_t)g * G + hh) * N) * D + c;
                    for (int i = 0; i < N; ++i) {
                        float a = fabsf(qp[(size_t)i * D]);
                        if (a > aq) aq = a;
                    }
                }
                const float* kp = k + (((size_t)b * Hkv + g) * N) * D + c;
                for (int i = 0; i < N; ++i) {
                    float a = fabsf(kp[(size_t)i * D]);
                    if (a > ak) ak = a;
                }
            }
            float sv;
            if (aq == 0.0f || ak == 0.0f) sv = 1.0f;
            else if (alpha == 0.5f) sv = (float)sqrt((double)(float)((double)ak / (double)aq));
            else sv = (float)(pow((double)ak, (double)alpha) / pow((double)aq, 1.0 - (double)alpha));
            s[(size_t)g * D + c] = sv;
            s_inv[(size_t)g * D + c] = (float)(1.0 / (double)sv);
        }
    }
}

/* ------------------------------------------------------ quantization */

/* Q or K: x [B,H,N,D] -> codes [B,H,N,D/2] (element 2i in the low nibble),
 * scales [B,H,N,D/16]. scale: [H/group, D] fp32 multiplier per (kv head,
 * channel), or NULL for no smoothing. group = number of heads per kv head
 * (Hq/Hkv for Q, 1 for K). */
void ora_quantize_rows(const float* x, int B, int H, int N, int D, int group,
                       const float* scale, uint8_t* codes, uint8_t* sf) {
    int nb = D / 16;
#pragma omp parallel for schedule(static)
    for (long long row = 0; row < (long long)B * H * N; ++row) {
        int h = (int)((row / N) % H);
        const float* xr = x + (size_t)row * D;
        float buf[16];
        uint8_t c16[16];
        for (int blk = 0; blk < nb; ++blk) {
            for (int i = 0; i < 16; ++i) {
                int d = blk * 16 + i;
                buf[i] = scale ? mul_f32(xr[d], scale[(size_t)(h / group) * D + d]) : xr[d];
            }
            ora_quant_block16(buf, c16, &sf[(size_t)row * nb + blk]);
            for (int i = 0; i < 8; ++i)
                codes[(size_t)row * (D / 2) + blk * 8 + i] = (uint8_t)(c16[2 * i] | (c16[2 * i + 1] << 4));
        }
    }
}

/* V quantized along tokens: v [B,Hkv,N,D] -> vtc [B,Hkv,D,N/2], vts [B,Hkv,D,N/16]. */
void ora_quantize_v(const float* v, int B, int Hkv, int N, int D, uint8_t* vtc, uint8_t* vts) {
    int nb = N / 16;
#pragma omp parallel for schedule(static)
    for (long long bgd = 0; bgd < (long long)B * Hkv * D; ++bgd) {
        long long bg = bgd / D;
        int d = (int)(bgd % D);
        const float* vp = v + (size_t)bg * N * D + d;
        float buf[16];
        uint8_t c16[16];
        for (int blk = 0; blk < nb; ++blk) {
            for (int i = 0; i < 16; ++i) buf[i] = vp[(size_t)(blk * 16 + i) * D];
            ora_quant_block16(buf, c16, &vts[(size_t)bgd * nb + blk]);
            for (int i = 0; i < 8; ++i)
                vtc[(size_t)bgd * (N / 2) + blk * 8 + i] = (uint8_t)(c16[2 * i] | (c16[2 * i + 1] << 4));
        }
    }
}

/* ----------------------------------------- steps before quantization */

/* Rotary position embedding, rotate-half pairing: channel d < D/2 pairs with
 * channel d + D/2 (the abstract applies Smooth-QK "after RoPE"; RoPE itself
 * is the standard rotation of the RoFormer paper in this pairing). In place on
 * x [rows, D], with c = cos_t[pos[row], d] and s = sin_t[pos[row], d]
 * (tables [*, D/2]):
 *   x[d]       <- RN(RN(x[d]*c) - RN(x[d+D/2]*s))
 *   x[d+D/2]   <- RN(RN(x[d+D/2]*c) + RN(x[d]*s))
 * each product and sum rounded to fp32 (no fused multiply-add). */
void ora_rope_neox(float* x, long long rows, int D, const float* cos_t, const float* sin_t, const int* pos) {
    int H2 = D / 2;
    for (long long r = 0; r < rows; ++r) {
        float* xr = x + (size_t)r * D;
        const float* cr = cos_t + (size_t)pos[r] * H2;
        const float* sr = sin_t + (size_t)pos[r] * H2;
        for (int d = 0; d < H2; ++d) {
            float a = xr[d], b = xr[d + H2];
            float ac = a * cr[d], bs = b * sr[d], bc = b * cr[d], as = a * sr[d];
            xr[d] = ac - bs;
            xr[d + H2] = bc + as;
        }
    }
}

/* Smooth-QK multiply in place: x[b,h,i,d] <- RN(x * scale[h/group, d])
 * (the same product ora_quantize_rows takes when given a scale). */
void ora_smooth_rows(float* x, int B, int H, int N, int D, int group, const float* scale) {
    for (long long row = 0; row < (long long)B * H * N; ++row) {
        int h = (int)((row / N) % H);
        float* xr = x + (size_t)row * D;
        for (int d = 0; d < D; ++d) xr[d] = mul_f32(xr[d], scale[(size_t)(h / group) * D + d]);
    }
}

/* Q-Mean auxiliary, first half: the per-(batch, head, channel) mean of the
 * pre-quantization Q over its N tokens, mean[bh, d] = RN_fp32(sum_i x / N),
 * with the sum accumulated in fp64 and divided in fp64 (x [BH, N, D]). */
void ora_q_mean(const float* x, long long BH, int N, int D, float* mean) {
    for (long long bh = 0; bh < BH; ++bh) {
        for (int d = 0; d < D; ++d) {
            double sum = 0.0;
            for (int i = 0; i < N; ++i) sum += (double)x[((size_t)bh * N + i) * D + d];
            mean[(size_t)bh * D + d] = (float)(sum / (double)N);
        }
    }
}

/* x[bh, i, d] <- RN(x - mean[bh, d]): the residual that is quantized. */
void ora_sub_mean(float* x, long long BH, int N, int D, const float* mean) {
    for (long long bh = 0; bh < BH; ++bh)
        for (int i = 0; i < N; ++i)
            for (int d = 0; d < D; ++d) x[((size_t)bh * N + i) * D + d] -= mean[(size_t)bh * D + d];
}

/* Q-Mean auxiliary, second half: the rank-one score term the residual leaves
 * out, bias[b,h,j] = sum_d mean[b,h,d] * K'[b,g,j,d] (g = h / (Hq/Hkv)), with
 * K' the keys as they enter quantization (after RoPE and smoothing, before
 * 4-bit rounding: the term is kept at full precision), accumulated in fp64.
 * kf [B,Hkv,Nkv,D]; bias [B,Hq,Nkv]. */
void ora_q_mean_bias(const float* mean, const float* kf, int B, int Hq, int Hkv, int Nkv, int D, double* bias) {
    int G = Hq / Hkv;
    for (long long bh = 0; bh < (long long)B * Hq; ++bh) {
        long long b = bh / Hq;
        int g = (int)(bh % Hq) / G;
        for (int j = 0; j < Nkv; ++j) {
            const float* kr = kf + (((size_t)b * Hkv + g) * (size_t)Nkv + j) * D;
            double acc = 0.0;
            for (int d = 0; d < D; ++d) acc += (double)mean[(size_t)bh * D + d] * (double)kr[d];
            bias[(size_t)bh * Nkv + j] = acc;
        }
    }
}

/* Decode helpers over the canonical packed layouts. */
static double dec_row(const uint8_t* codes, const uint8_t* sf, int idx) {
    uint8_t byte = codes[idx >> 1];
    uint8_t nib = (idx & 1) ? (byte >> 4) : (byte & 15);
    return ora_e2m1_decode(nib) * ora_e4m3_decode(sf[idx >> 4]);
}

/* ------------------------------------------------------- QK scores */

/* One row of unmasked scores S[n] = sum_d Qhat[row,d]*Khat[n,d], rounded once
 * to fp32. Exposed for the exact-sum pin. */
void ora_qk_row(const uint8_t* qc, const uint8_t* qs, const uint8_t* kc, const uint8_t* ks,
                int Hq, int Hkv, int Nq, int Nkv, int D, long long row, float* S) {
    int G = Hq / Hkv;
    long long bh = row / Nq;
    int b = (int)(bh / Hq), h = (int)(bh % Hq), g = h / G;
    const uint8_t* qcr = qc + (size_t)row * (D / 2);
    const uint8_t* qsr = qs + (size_t)row * (D / 16);
    double qd[256];
    for (int d = 0; d < D; ++d) qd[d] = dec_row(qcr, qsr, d);
    size_t kbase = ((size_t)b * Hkv + g) * (size_t)Nkv;
    for (int n = 0; n < Nkv; ++n) {
        const uint8_t* kcr = kc + (kbase + n) * (D / 2);
        const uint8_t* ksr = ks + (kbase + n) * (D / 16);
        double acc = 0.0;
        for (int d = 0; d < D; ++d) acc += qd[d] * dec_row(kcr, ksr, d);
        S[n] = (float)acc;
    }
}

/* ------------------------------------------------------- attention */

/* norm_mode: 0 = P-Reordering (l from P_hat), 1 = high-precision l (from P).
 * n_splits >= 1: kv split count (see the header; 1 = one pass).
 * s_bias: NULL, or a per-(b, h, key) score term [B,Hq,Nkv] added to the fp64
 * dot product before its one rounding, S = RN_fp32(Q_hat K_hat^T + s_bias)
 * (the Q-Mean auxiliary: ora_q_mean_bias; 4-bit path only).
 * quant: 1 = 4-bit path on the packed operands; 0 = the same online softmax
 * on the fp32 operands qf/kf/vf ([B,H,N,D], already smoothed) with P unquantized.
 * rows: flat query-row ids (b*Hq + h)*Nq + i. Outputs are per requested row.
 * Optional outputs may be NULL: l_hat/l_hp [n_rows]; eps_tile [n_rows, Nkv/128]
 * (sum P_hat / sum P - 1 per tile, NAN where the tile has no mass for the row);
 * p_codes [n_rows, Nkv/2], p_sf [n_rows, Nkv/16] (P_hat in canonical layout,
 * zero for tiles not visited). Returns 0, or -1 on unsupported arguments. */
int ora_attention_rows(const uint8_t* qc, const uint8_t* qs, const uint8_t* kc, const uint8_t* ks,
                       const uint8_t* vtc, const uint8_t* vts,
                       const float* qf, const float* kf, const float* vf,
                       int B, int Hq, int Hkv, int Nq, int Nkv, int D,
                       float sm_scale, int causal, int norm_mode, int quant, int n_splits,
                       const double* s_bias, const long long* rows, long long n_rows,
                       double* O, double* lse, double* l_hat_out, double* l_hp_out,
                       double* eps_tile, uint8_t* p_codes, uint8_t* p_sf, int n_threads) {
    if (D > 256 || D % 16 || Nkv % TILE_KV || Hq % Hkv || n_splits < 1) return -1;
    (void)B;
    int G = Hq / Hkv;
    int n_tiles = Nkv / TILE_KV;
    float c = (float)((double)sm_scale * 1.4426950408889634074);   /* RN(sm_scale*log2 e) */
#ifdef _OPENMP
    if (n_threads > 0) omp_set_num_threads(n_threads);
#else
    (void)n_threads;
#endif
#pragma omp parallel for schedule(dynamic, 4)
    for (long long r = 0; r < n_rows; ++r) {
        long long row = rows[r];
        long long bh = row / Nq;
        int i = (int)(row % Nq);
        int b = (int)(bh / Hq), h = (int)(bh % Hq), g = h / G;
        size_t kvbase = ((size_t)b * Hkv + g) * (size_t)Nkv;     /* row of K[b,g,0] */
        size_t vtbase = ((size_t)b * Hkv + g) * (size_t)D;       /* row of Vt[b,g,0] */
        long long last = causal ? (long long)i + Nkv - Nq : (long long)Nkv - 1;

        double qd[256];
        if (quant) {
            for (int d = 0; d < D; ++d) qd[d] = dec_row(qc + (size_t)row * (D / 2), qs + (size_t)row * (D / 16), d);
        } else {
            for (int d = 0; d < D; ++d) qd[d] = qf[(size_t)row * D + d];
        }
        double Oacc[256], L_out = 0.0, Lhat_out = 0.0, Lhp_out = 0.0;
        float M = -INFINITY;                       /* largest mc over the splits with mass */
        for (int d = 0; d < D; ++d) Oacc[d] = 0.0;
        float S[TILE_KV], P[TILE_KV];
        double Ph[TILE_KV];
        if (eps_tile) for (int t = 0; t < n_tiles; ++t) eps_tile[r * n_tiles + t] = NAN;
        if (p_codes) memset(p_codes + (size_t)r * (Nkv / 2), 0, (size_t)Nkv / 2);
        if (p_sf) memset(p_sf + (size_t)r * (Nkv / 16), 0, (size_t)Nkv / 16);

        for (int sp = 0; sp < n_splits; ++sp) {
        const int t_begin = (int)(((long long)sp * n_tiles) / n_splits);
        const int t_end = (int)(((long long)(sp + 1) * n_tiles) / n_splits);
        double oacc[256];
        for (int d = 0; d < D; ++d) oacc[d] = 0.0;
        double l_hat = 0.0, l_hp = 0.0;
        float m = -INFINITY, mc = 0.0f;
        for (int t = t_begin; t < t_end && (long long)t * TILE_KV <= last; ++t) {
            /* scores of this tile, masked keys at -inf */
            float rowmax = -INFINITY;
            for (int j = 0; j < TILE_KV; ++j) {
                long long n = (long long)t * TILE_KV + j;
                if (n > last) { S[j] = -INFINITY; continue; }
                double acc = 0.0;
                if (quant) {
                    const uint8_t* kcr = kc + (kvbase + n) * (D / 2);
                    const uint8_t* ksr = ks + (kvbase + n) * (D / 16);
                    for (int d = 0; d < D; ++d) acc += qd[d] * dec_row(kcr, ksr, d);
                    if (s_bias) acc += s_bias[(size_t)bh * Nkv + n];     /* bh = b*Hq + h */
                } else {
                    const float* kr = kf + (kvbase + n) * D;
                    for (int d = 0; d < D; ++d) acc += qd[d] * (double)kr[d];
                }
                S[j] = (float)acc;
                if (S[j] > rowmax) rowmax = S[j];
            }
            /* online softmax: running max, rescale factor, probabilities */
            float m_new = rowmax > m ? rowmax : m;
            float mc_new = (float)((double)m_new * (double)c);
            double alpha = (m == -INFINITY) ? 0.0 : exp2((double)mc - (double)mc_new);
            double sumP = 0.0, sumPh = 0.0;
            for (int j = 0; j < TILE_KV; ++j) {
                P[j] = (S[j] == -INFINITY) ? 0.0f : (float)exp2((double)fmaf(S[j], c, -mc_new));
                sumP += P[j];
            }
            /* quantized probabilities, 16 keys per scale */
            if (quant) {
                for (int blk = 0; blk < TILE_KV / 16; ++blk) {
                    uint8_t c16[16], sf;
                    ora_quant_block16(P + blk * 16, c16, &sf);
                    double Sd = ora_e4m3_decode(sf);
                    for (int e = 0; e < 16; ++e) Ph[blk * 16 + e] = ora_e2m1_decode(c16[e]) * Sd;
                    long long kv0 = (long long)t * TILE_KV + blk * 16;
                    if (p_sf) p_sf[(size_t)r * (Nkv / 16) + kv0 / 16] = sf;
                    if (p_codes)
                        for (int e = 0; e < 8; ++e)
                            p_codes[(size_t)r * (Nkv / 2) + kv0 / 2 + e] = (uint8_t)(c16[2 * e] | (c16[2 * e + 1] << 4));
                }
            } else {
                for (int j = 0; j < TILE_KV; ++j) Ph[j] = P[j];
            }
            for (int j = 0; j < TILE_KV; ++j) sumPh += Ph[j];
            /* O_acc <- alpha*O_acc + P_hat V_hat over this tile */
            for (int d = 0; d < D; ++d) {
                double acc = 0.0;
                for (int j = 0; j < TILE_KV; ++j) {
                    if (Ph[j] == 0.0) continue;
                    long long n = (long long)t * TILE_KV + j;
                    double vv = quant ? dec_row(vtc + (vtbase + d) * (size_t)(Nkv / 2),
                                                vts + (vtbase + d) * (size_t)(Nkv / 16), (int)n)
                                      : (double)vf[(kvbase + n) * D + d];
                    acc += Ph[j] * vv;
                }
                oacc[d] = alpha * oacc[d] + acc;
            }
            l_hat = alpha * l_hat + sumPh;
            l_hp = alpha * l_hp + sumP;
            if (eps_tile && sumP > 0.0) eps_tile[r * n_tiles + t] = sumPh / sumP - 1.0;
            m = m_new;
            mc = mc_new;
        }
        /* merge this split into the running result, in the frame of the
         * largest mc seen so far (with one split: weight 1, the plain pass) */
        double l = norm_mode == 0 ? l_hat : l_hp;
        if (l > 0.0) {
            double w_old = 1.0, w_new = 1.0;
            if (M == -INFINITY) {
                M = mc;
            } else if (mc > M) {
                w_old = exp2((double)M - (double)mc);
                M = mc;
            } else {
                w_new = exp2((double)mc - (double)M);
            }
            for (int d = 0; d < D; ++d) Oacc[d] = w_old * Oacc[d] + w_new * oacc[d];
            L_out = w_old * L_out + w_new * l;
            Lhat_out = w_old * Lhat_out + w_new * l_hat;
            Lhp_out = w_old * Lhp_out + w_new * l_hp;
        }
        }
        for (int d = 0; d < D; ++d) O[(size_t)r * D + d] = L_out > 0.0 ? Oacc[d] / L_out : 0.0;
        lse[r] = L_out > 0.0 ? (double)M * 0.69314718055994530942 + log(L_out) : -INFINITY;
        if (l_hat_out) l_hat_out[r] = Lhat_out;
        if (l_hp_out) l_hp_out[r] = Lhp_out;
    }
    return 0;
}
