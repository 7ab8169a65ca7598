/*
 * qattn_oracle.c -- plain, slow CPU oracle for quantized scaled-dot-product attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may link, load or call this file;
 * only the test suite, the package smoke check and the benchmark's CPU-baseline leg do.
 * It shares no code, header, table or helper with the CUDA library.
 *
 * What it computes follows the NVIDIA developer blog "Optimizing FLUX.1 Kontext for Image
 * Editing with Low-Precision Quantization", section "Workflow and quantization":
 *   - Q, K, V go through FakeQuantize nodes, per-tensor FP8 or per-block FP4 (bullet 1, Fig. 4);
 *   - BMM1 (Q K^T) runs in FP8 with higher-precision accumulation, after an extra FP8
 *     quantize of its inputs (bullet 2);
 *   - softmax runs in FP32, unquantized (bullet 3; Fig. 4 "softmax always in FP32");
 *   - BMM2 (P V) runs with per-tensor FP8 quantization (bullet 4; Fig. 4).
 * The pages do not spell out the number formats; E4M3 and E2M1 follow the OCP 8-bit / MX
 * definitions (E4M3 "fn": bias 7, no infinities, max 448; E2M1: bias 1, max 6).  Every
 * reading taken where the pages are silent is listed next to the function that takes it.
 *
 * Arithmetic: exact where a plain definition exists (amax, both BMM sums, which are exact in
 * FP64 for these operand widths), FP32 where the method says FP32 (scores, softmax), and
 * correctly rounded FP32 division for every scale application.  No blocking, no fusion, no
 * reordering beyond what the definitions state.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORC_OK 0
#define ORC_ERR_INVALID 1
#define ORC_ERR_NONFINITE 4

/* ------------------------------------------------------------------------------------------
 * Number formats (format definitions; the blog names FP8 and FP4 but not their encodings).
 * ---------------------------------------------------------------------------------------- */

/* bfloat16 bits -> float: the top 16 bits of an IEEE binary32. */
float orc_bf16_to_float(uint16_t b) {
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

/* E4M3 ("fn") code -> value.  sign | eeee | mmm, bias 7; e = 0 is subnormal (m/8 * 2^-6);
 * e = 15, m = 7 is NaN; there are no infinities. */
float orc_e4m3_to_float(uint8_t c) {
    int s = (c >> 7) & 1, e = (c >> 3) & 15, m = c & 7;
    double v;
    if (e == 15 && m == 7) return NAN;
    if (e == 0) v = ldexp((double)m / 8.0, -6);
    else v = ldexp(1.0 + (double)m / 8.0, e - 7);
    return (float)(s ? -v : v);
}

/* float -> E4M3 code, round to nearest with ties to even, saturating to +-448 (no infinity
 * in the format).  The sign is always kept, so -0 and negatives that round to zero give 0x80.
 * NaN input gives the NaN code 0x7F (callers reject non-finite tensors before this point). */
uint8_t orc_e4m3_from_float(float x) {
    uint8_t sign = signbit(x) ? 0x80 : 0x00;
    double a = fabs((double)x);
    if (isnan(x)) return 0x7F;
    if (a > 448.0) return sign | 0x7E;                 /* satfinite */
    if (a < ldexp(1.0, -6)) {                          /* subnormal range: step 2^-9 */
        double q = rint(a * 512.0);                    /* exact scaling, RNE */
        return sign | (uint8_t)q;                      /* q == 8 is the smallest normal, code 8 */
    }
    int E;
    double f = frexp(a, &E);                           /* a = f * 2^E, f in [0.5, 1) */
    int e = E - 1;                                     /* a = m * 2^e, m in [1, 2) */
    double m = f * 2.0;
    double q = rint((m - 1.0) * 8.0);                  /* 3 mantissa bits, RNE */
    if (q == 8.0) { q = 0.0; e += 1; }
    int code = ((e + 7) << 3) | (int)q;
    if (code > 0x7E) code = 0x7E;                      /* cannot trigger for a <= 448 */
    return sign | (uint8_t)code;
}

/* E2M1 code (4 bits) -> value.  s | ee | m, bias 1; grid {0, .5, 1, 1.5, 2, 3, 4, 6}. */
float orc_e2m1_to_float(uint8_t c) {
    int s = (c >> 3) & 1, e = (c >> 1) & 3, m = c & 1;
    double v = (e == 0) ? 0.5 * m : ldexp(1.0 + 0.5 * m, e - 1);
    return (float)(s ? -v : v);
}

/* float -> E2M1 code, RNE with ties to the even code, saturating to +-6, sign kept. */
uint8_t orc_e2m1_from_float(float x) {
    uint8_t sign = signbit(x) ? 0x8 : 0x0;
    double a = fabs((double)x);
    if (isnan(x)) return sign | 0x7;                   /* no NaN in E2M1; callers never pass one */
    if (a > 6.0) return sign | 0x7;                    /* satfinite */
    if (a < 1.0) {                                     /* subnormal range: step 0.5 */
        double q = rint(a * 2.0);                      /* q == 2 is the code of 1.0 */
        return sign | (uint8_t)q;
    }
    int E;
    double f = frexp(a, &E);
    int e = E - 1;                                     /* 0, 1 or 2 */
    double q = rint((f * 2.0 - 1.0) * 2.0);            /* 1 mantissa bit, RNE */
    if (q == 2.0) { q = 0.0; e += 1; }
    int code = ((e + 1) << 1) | (int)q;
    if (code > 7) code = 7;
    return sign | (uint8_t)code;
}

/* ------------------------------------------------------------------------------------------
 * Calibration and FakeQuantize (blog, "Workflow and quantization": per-tensor FP8 or
 * per-block FP4 quantization of Q, K, V; the post-training calibration step of the flow,
 * reduced here to the max-calibration of the tensor in hand).
 * ---------------------------------------------------------------------------------------- */

/* amax = max |x| over the whole tensor, exact.  Returns ORC_ERR_NONFINITE for inf/NaN. */
int orc_amax_bf16(const uint16_t *x, int64_t n, float *amax) {
    float m = 0.0f;
    int bad = 0;
    for (int64_t i = 0; i < n; ++i) {
        float v = fabsf(orc_bf16_to_float(x[i]));
        if (!isfinite(v)) bad = 1;
        else if (v > m) m = v;
    }
    *amax = bad ? INFINITY : m;
    return bad ? ORC_ERR_NONFINITE : ORC_OK;
}

/* Per-tensor FP8 FakeQuantize: s = fl32(amax / 448); code = e4m3(fl32(x / s)).
 * Reading: amax == 0 gives s = 1 (all codes are signed zeros).  The dequantized value is
 * fl32(val(code) * s). */
int orc_quantize_fp8(const uint16_t *x, int64_t n, float amax, uint8_t *codes, float *scale) {
    if (!isfinite(amax) || amax < 0.0f) return ORC_ERR_NONFINITE;
    float s = (amax == 0.0f) ? 1.0f : amax / 448.0f;   /* binary32 division, correctly rounded */
    for (int64_t i = 0; i < n; ++i) {
        float q = orc_bf16_to_float(x[i]) / s;
        codes[i] = orc_e4m3_from_float(q);
    }
    *scale = s;
    return ORC_OK;
}

/* Per-block FP4 FakeQuantize followed by the per-tensor FP8 quantize of BMM1's inputs.
 * Blocks are 16 consecutive elements (along D in a [..., D] tensor), E2M1 values, one E4M3
 * scale per block and one FP32 tensor scale:
 *   s_g  = fl32(amax / 2688)                   (2688 = 6 * 448: E2M1 max times E4M3 max)
 *   s_b  = e4m3(fl32(amax_b / fl32(6 * s_g)))  (block scale, an E4M3 code)
 *   eff  = fl32(val(s_b) * s_g)
 *   c    = e2m1(fl32(x / eff))                  (eff == 0: the block's codes are 0)
 *   xhat = fl32(fl32(val(c) * val(s_b)) * s_g)  (the dequantized FP4 value)
 * then the extra FP8 quantize the blog puts in front of BMM1:
 *   s8   = fl32(max|xhat| / 448),  c8 = e4m3(fl32(xhat / s8)).
 * Packing: element 2i in the low nibble of byte i, element 2i+1 in the high nibble.
 * max|xhat| is found by brute force over all xhat.  codes8/scale8 may be NULL. */
int orc_quantize_fp4_block(const uint16_t *x, int64_t n, float amax, uint8_t *packed,
                           uint8_t *bscale, float *gscale, uint8_t *codes8, float *scale8) {
    if (n % 16 != 0) return ORC_ERR_INVALID;
    if (!isfinite(amax) || amax < 0.0f) return ORC_ERR_NONFINITE;
    float sg = (amax == 0.0f) ? 1.0f : amax / 2688.0f;
    float six_sg = 6.0f * sg;
    float *xhat = codes8 ? (float *)malloc(sizeof(float) * (size_t)n) : NULL;
    float xhat_max = 0.0f;
    for (int64_t b = 0; b < n / 16; ++b) {
        const uint16_t *xb = x + b * 16;
        float amax_b = 0.0f;
        for (int i = 0; i < 16; ++i) {
            float v = fabsf(orc_bf16_to_float(xb[i]));
            if (v > amax_b) amax_b = v;
        }
        uint8_t sb = orc_e4m3_from_float(amax_b / six_sg);
        bscale[b] = sb;
        float eff = orc_e4m3_to_float(sb) * sg;
        uint8_t c[16];
        for (int i = 0; i < 16; ++i) {
            c[i] = (eff == 0.0f) ? 0 : orc_e2m1_from_float(orc_bf16_to_float(xb[i]) / eff);
        }
        for (int i = 0; i < 8; ++i) packed[b * 8 + i] = (uint8_t)(c[2 * i] | (c[2 * i + 1] << 4));
        if (xhat) {
            for (int i = 0; i < 16; ++i) {
                float t = orc_e2m1_to_float(c[i]) * orc_e4m3_to_float(sb);
                float v = t * sg;
                xhat[b * 16 + i] = v;
                if (fabsf(v) > xhat_max) xhat_max = fabsf(v);
            }
        }
    }
    *gscale = sg;
    if (codes8) {
        float s8 = (xhat_max == 0.0f) ? 1.0f : xhat_max / 448.0f;
        for (int64_t i = 0; i < n; ++i) codes8[i] = orc_e4m3_from_float(xhat[i] / s8);
        if (scale8) *scale8 = s8;
        free(xhat);
    }
    return ORC_OK;
}

/* Dequantize packed FP4 (for tests): xhat as defined above. */
void orc_dequant_fp4_block(const uint8_t *packed, const uint8_t *bscale, float sg, int64_t n,
                           float *out) {
    for (int64_t i = 0; i < n; ++i) {
        uint8_t byte = packed[i / 2];
        uint8_t c = (i % 2 == 0) ? (byte & 0xF) : (byte >> 4);
        float t = orc_e2m1_to_float(c) * orc_e4m3_to_float(bscale[i / 16]);
        out[i] = t * sg;
    }
}

/* ------------------------------------------------------------------------------------------
 * Attention (blog, "Workflow and quantization", bullets 2-4 and Fig. 4).
 *
 * Tensors are [B, H, T, D] (T tokens per batch row).  Along T, every batch row holds the
 * sequences [cu[s], cu[s+1]) for s < nseq; attention is full (non-causal) inside a sequence
 * and absent across sequences (a dense [B, H, L, D] call is nseq = 1, cu = {0, L}).
 *
 * Inputs are VALUES without their per-tensor scale: val(code) for quantized tensors, or
 * arbitrary doubles.  Per query row i of a sequence with keys j:
 *   acc_j = sum_d q_d k_jd                               exact in FP64 for E4M3 operands
 *   FP32 softmax (flag ORC_FP32):  S'_j = fl32(acc_j * c),  c = fl32(s_q s_k sm_scale log2 e)
 *   otherwise (exact):             S'_j = acc_j * s_q s_k sm_scale log2 e   (FP64)
 *   M   = ceil(max_j S'_j)                                power-of-two row max (reading below)
 *   p_j = 2^(S'_j - M)               (ORC_FP32: fl32(2^fl32(S'_j - M)))
 *   l   = sum_j p_j                  (ORC_FP32: FP64 sum rounded once to FP32)
 *   P quantization (flag ORC_QUANT_P): P8_j = e4m3(fl32(p_j * 448)), i.e. per-tensor scale 1/448
 *   O_d = (sum_j val(P8_j) v_jd) * s_v / 448 / l          (ORC_QUANT_P)
 *   O_d = (sum_j p_j v_jd) * s_v / l                      (otherwise)
 * Flag ORC_FIG4_LITERAL quantizes the normalized probability instead:
 *   P8_j = e4m3(fl32(fl32(p_j / l) * 448)),  O_d = (sum_j val(P8_j) v_jd) * s_v / 448.
 *
 * Readings where the blog is silent: (1) P is quantized before normalization with the fixed
 * scale 1/448 (amax of the unnormalized p is exactly 1 at the row max), and the FP32 row sum
 * divides the BMM2 result; (2) the subtracted row max is rounded up to an integer in base-2
 * units, so every p lies in (0, 1] and the result does not depend on how keys are tiled.
 *
 * rows: NULL for every row, else nrows row ids r = (b * H + h) * T + t.  out: [nrows, D].
 * amb (optional, [nrows, D]): per output, the largest change of O that choosing the other code
 * of an ambiguous P decision (see attend_row) can make, summed over keys.
 * ---------------------------------------------------------------------------------------- */
#define ORC_FP32 1
#define ORC_QUANT_P 2
#define ORC_FIG4_LITERAL 4

/* Ambiguity of a P code (flag ORC_QUANT_P with ORC_FP32, `amb` != NULL).  The blog fixes the
 * accumulation of BMM1 only as "higher precision"; an FP32 accumulator that rounds in another
 * order than this oracle's exact sum changes S' by up to about kappa * u * sum_d |q_d k_d| * c
 * (u = 2^-24, kappa = 16 roundings), the FP32 steps of the softmax add a few ulps of S', and a
 * hardware exp2 a few ulps of p.  When that interval of S' - M straddles an E4M3 rounding
 * boundary of p * 448, both codes are correct results of the method; amb[j] records how far the
 * other code's value lies from this one's (0 when the code is unique). */
#define ORC_AMB_KAPPA 16.0

static double e4m3_val_of(double p448) {
    return (double)orc_e4m3_to_float(orc_e4m3_from_float((float)p448));
}

static void attend_row(const double *q, const double *K, const double *V, int64_t nkeys, int D,
                       double c64, float c32, double s_v, int flags, double *S, double *P,
                       double *W, double *out, double *amb_out) {
    /* scores */
    double smax = -INFINITY;
    for (int64_t j = 0; j < nkeys; ++j) {
        const double *k = K + j * D;
        double acc = 0.0, absacc = 0.0;
        for (int d = 0; d < D; ++d) {
            acc += q[d] * k[d];
            absacc += fabs(q[d] * k[d]);
        }
        double s = (flags & ORC_FP32) ? (double)(float)((float)acc * c32) : acc * c64;
        S[j] = s;
        W[j] = absacc;
        if (s > smax) smax = s;
    }
    double M = ceil(smax);
    /* unnormalized probabilities and their sum */
    double lsum = 0.0;
    for (int64_t j = 0; j < nkeys; ++j) {
        double p;
        if (flags & ORC_FP32) p = (double)(float)exp2((double)(float)(S[j] - M));
        else p = exp2(S[j] - M);
        P[j] = p;
        lsum += p;
    }
    double l = (flags & ORC_FP32) ? (double)(float)lsum : lsum;
    /* P quantization */
    double post = s_v / l;
    if (flags & ORC_FIG4_LITERAL) {
        for (int64_t j = 0; j < nkeys; ++j) {
            float pn = (float)P[j] / (float)l;
            P[j] = (double)orc_e4m3_to_float(orc_e4m3_from_float(pn * 448.0f));
        }
        post = s_v / 448.0;
    } else if (flags & ORC_QUANT_P) {
        for (int64_t j = 0; j < nkeys; ++j) {
            double code_val = (double)orc_e4m3_to_float(orc_e4m3_from_float((float)P[j] * 448.0f));
            if (amb_out) {
                double x = S[j] - M;
                double delta = ORC_AMB_KAPPA * ldexp(W[j] * c64, -24)
                             + 4.0 * ldexp(fabs(S[j]) + fabs(M) + 1.0, -23) + ldexp(1.0, -20);
                double lo = e4m3_val_of(exp2(x - delta) * 448.0);
                double hi = e4m3_val_of(exp2(x + delta) * 448.0);
                double a = fabs(lo - code_val), b = fabs(hi - code_val);
                W[j] = a > b ? a : b;     /* W is reused as the ambiguity of code j */
            }
            P[j] = code_val;
        }
        post = s_v / 448.0 / l;
    }
    /* BMM2 */
    for (int d = 0; d < D; ++d) out[d] = 0.0;
    for (int64_t j = 0; j < nkeys; ++j) {
        const double *v = V + j * D;
        double p = P[j];
        for (int d = 0; d < D; ++d) out[d] += p * v[d];
    }
    for (int d = 0; d < D; ++d) out[d] *= post;
    if (amb_out) {
        for (int d = 0; d < D; ++d) amb_out[d] = 0.0;
        if ((flags & ORC_QUANT_P) && !(flags & ORC_FIG4_LITERAL)) {
            for (int64_t j = 0; j < nkeys; ++j) {
                if (W[j] == 0.0) continue;
                const double *v = V + j * D;
                for (int d = 0; d < D; ++d) amb_out[d] += W[j] * fabs(v[d]) * post;
            }
        }
    }
}

typedef struct { int64_t row; int64_t slot; } row_ref;

static int cmp_row_ref(const void *a, const void *b) {
    int64_t x = ((const row_ref *)a)->row, y = ((const row_ref *)b)->row;
    return (x > y) - (x < y);
}

/* Core over values (doubles).  See the block comment above for the definition. */
int orc_attention_values(const double *q, const double *k, const double *v, int B, int H,
                         int64_t T, int D, const int64_t *cu, int nseq, double s_q, double s_k,
                         double s_v, double sm_scale, int flags, const int64_t *rows,
                         int64_t nrows, double *out, double *amb) {
    if (B < 1 || H < 1 || T < 1 || D < 1 || nseq < 1) return ORC_ERR_INVALID;
    if (cu[0] != 0 || cu[nseq] != T) return ORC_ERR_INVALID;
    for (int s = 0; s < nseq; ++s) if (cu[s + 1] <= cu[s]) return ORC_ERR_INVALID;
    const double log2e = 1.4426950408889634;   /* log2(e) to double precision */
    double c64 = s_q * s_k * sm_scale * log2e;
    float c32 = (float)c64;
    int64_t total = rows ? nrows : (int64_t)B * H * T;
    row_ref *refs = (row_ref *)malloc(sizeof(row_ref) * (size_t)(total > 0 ? total : 1));
    for (int64_t i = 0; i < total; ++i) {
        refs[i].row = rows ? rows[i] : i;
        refs[i].slot = i;
        if (refs[i].row < 0 || refs[i].row >= (int64_t)B * H * T) { free(refs); return ORC_ERR_INVALID; }
    }
    qsort(refs, (size_t)total, sizeof(row_ref), cmp_row_ref);
    /* group rows by (b, h, sequence) and run each group's rows in parallel */
    int64_t g0 = 0;
    while (g0 < total) {
        int64_t bh = refs[g0].row / T, t0 = refs[g0].row % T;
        int s = 0;
        while (!(cu[s] <= t0 && t0 < cu[s + 1])) ++s;
        int64_t g1 = g0;
        while (g1 < total && refs[g1].row / T == bh && refs[g1].row % T < cu[s + 1]) ++g1;
        int64_t base = bh * T + cu[s], nkeys = cu[s + 1] - cu[s];
        const double *Kb = k + base * D, *Vb = v + base * D;
#pragma omp parallel
        {
            double *S = (double *)malloc(sizeof(double) * (size_t)nkeys);
            double *P = (double *)malloc(sizeof(double) * (size_t)nkeys);
            double *W = (double *)malloc(sizeof(double) * (size_t)nkeys);
#pragma omp for schedule(dynamic, 8)
            for (int64_t i = g0; i < g1; ++i) {
                attend_row(q + refs[i].row * D, Kb, Vb, nkeys, D, c64, c32, s_v, flags, S, P, W,
                           out + refs[i].slot * D, amb ? amb + refs[i].slot * D : NULL);
            }
            free(S);
            free(P);
            free(W);
        }
        g0 = g1;
    }
    free(refs);
    return ORC_OK;
}

/* Same, over E4M3 codes: values are val(code) (the scales are passed separately). */
int orc_attention_e4m3(const uint8_t *q8, const uint8_t *k8, const uint8_t *v8, int B, int H,
                       int64_t T, int D, const int64_t *cu, int nseq, double s_q, double s_k,
                       double s_v, double sm_scale, int flags, const int64_t *rows,
                       int64_t nrows, double *out, double *amb) {
    int64_t n = (int64_t)B * H * T * D;
    double tbl[256];
    for (int c = 0; c < 256; ++c) tbl[c] = (double)orc_e4m3_to_float((uint8_t)c);
    double *q = (double *)malloc(sizeof(double) * (size_t)n);
    double *k = (double *)malloc(sizeof(double) * (size_t)n);
    double *v = (double *)malloc(sizeof(double) * (size_t)n);
    if (!q || !k || !v) { free(q); free(k); free(v); return ORC_ERR_INVALID; }
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) {
        q[i] = tbl[q8[i]];
        k[i] = tbl[k8[i]];
        v[i] = tbl[v8[i]];
    }
    int rc = orc_attention_values(q, k, v, B, H, T, D, cu, nseq, s_q, s_k, s_v, sm_scale, flags,
                                  rows, nrows, out, amb);
    free(q);
    free(k);
    free(v);
    return rc;
}

/* One query row's P decisions, for comparing the P codes of an implementation key by key
 * (flags ORC_FP32 | ORC_QUANT_P, the method's steps as in attend_row).  row = (b * H + h) * T + t.
 * For each key j of the row's sequence: code[j] = e4m3(fl32(2^fl32(S'_j - M)) * 448), x[j] = S'_j - M
 * (S'_j the FP32 base-2 score), delta[j] = the accumulation-order radius of S'_j defined above
 * (ORC_AMB_KAPPA), and lo[j], hi[j] = the E4M3 codes of 2^(x[j] - delta[j]) * 448 and
 * 2^(x[j] + delta[j]) * 448: a method with another FP32 summation order may produce any code from
 * lo[j] to hi[j] for key j.  *M_out = M, *l_out = the FP32 row sum of the unquantized p.
 * Returns the number of keys, or a negative status. */
int64_t orc_p_row_detail(const uint8_t *q8, const uint8_t *k8, int B, int H, int64_t T, int D,
                         const int64_t *cu, int nseq, double s_q, double s_k, double sm_scale,
                         int64_t row, uint8_t *code, double *x, double *delta, uint8_t *lo,
                         uint8_t *hi, double *M_out, double *l_out) {
    if (B < 1 || H < 1 || T < 1 || D < 1 || nseq < 1 || row < 0 || row >= (int64_t)B * H * T)
        return ORC_ERR_INVALID;
    if (cu[0] != 0 || cu[nseq] != T) return ORC_ERR_INVALID;
    const int64_t bh = row / T, t = row % T;
    int s = 0;
    while (!(cu[s] <= t && t < cu[s + 1])) ++s;
    const int64_t nkeys = cu[s + 1] - cu[s], base = bh * T + cu[s];
    const double log2e = 1.4426950408889634;
    const double c64 = s_q * s_k * sm_scale * log2e;
    const float c32 = (float)c64;
    double *S = (double *)malloc(sizeof(double) * (size_t)nkeys);
    double *W = (double *)malloc(sizeof(double) * (size_t)nkeys);
    if (!S || !W) { free(S); free(W); return ORC_ERR_INVALID; }
    const uint8_t *q = q8 + row * D;
    double smax = -INFINITY;
    for (int64_t j = 0; j < nkeys; ++j) {
        const uint8_t *k = k8 + (base + j) * D;
        double acc = 0.0, absacc = 0.0;
        for (int d = 0; d < D; ++d) {
            const double prod = (double)orc_e4m3_to_float(q[d]) * (double)orc_e4m3_to_float(k[d]);
            acc += prod;
            absacc += fabs(prod);
        }
        S[j] = (double)(float)((float)acc * c32);
        W[j] = absacc;
        if (S[j] > smax) smax = S[j];
    }
    const double M = ceil(smax);
    double lsum = 0.0;
    for (int64_t j = 0; j < nkeys; ++j) {
        const double p = (double)(float)exp2((double)(float)(S[j] - M));
        lsum += p;
        code[j] = orc_e4m3_from_float((float)p * 448.0f);
        x[j] = S[j] - M;
        delta[j] = ORC_AMB_KAPPA * ldexp(W[j] * c64, -24) + 4.0 * ldexp(fabs(S[j]) + fabs(M) + 1.0, -23) +
                   ldexp(1.0, -20);
        lo[j] = orc_e4m3_from_float((float)(exp2(x[j] - delta[j]) * 448.0));
        hi[j] = orc_e4m3_from_float((float)(exp2(x[j] + delta[j]) * 448.0));
    }
    *M_out = M;
    *l_out = (double)(float)lsum;
    free(S);
    free(W);
    return nkeys;
}

int orc_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
