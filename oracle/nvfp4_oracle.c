/*
 * nvfp4_oracle.c -- plain, slow CPU oracle (TEST INFRASTRUCTURE ONLY).
 *
 * Only tests, the smoke check and the benchmark's CPU-baseline leg may load
 * this file's shared library.  It shares nothing with the CUDA library.
 *
 * Build: gcc -O2 -std=c11 -fno-fast-math -ffp-contract=off -fPIC -shared
 * (no x87: float expressions are evaluated in float, as FLT_EVAL_METHOD == 0
 * on x86-64 and aarch64).  No threads here; a caller may run disjoint row
 * ranges concurrently because every function is re-entrant.
 *
 * Sources (page title, section):
 *   H-Scale summary, sec. 3 "NVFP4 quantization", "Hessian-guided objective",
 *     "Group-wise scale selection", "Efficient scale search"; sec. B
 *     "Implementation", "HScaleGroupQuantize".
 *   ScaleSweep summary, sec. 1 "Optimization Objectives", sec. 2 "Theoretical
 *     Bounds", sec. 3 "Implementation".
 */
#include "nvfp4_oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>

/* ---- number formats --------------------------------------------------- */

/* E4M3 (FP8, bias 7, no infinities, 0x7F = NaN).  Bit pattern order equals
 * value order for the positive codes, which is why the pages can speak of a
 * "+7 offset in bit-pattern space" (ScaleSweep sec. 2). */
double orc_e4m3_value(int code) {
    if (code < 0 || code > 126) return -1.0;
    int e = code >> 3, m = code & 7;
    if (e == 0) return ldexp((double)m, -9);          /* subnormal: m * 2^-9 */
    return ldexp(1.0 + m / 8.0, e - 7);                /* (1 + m/8) * 2^(e-7) */
}

int orc_e4m3_nearest(double f) {
    if (!(f >= 0.0)) return -1;                        /* NaN or negative */
    int best = 0;
    double bd = fabs(f - 0.0);
    for (int c = 1; c <= 126; ++c) {
        double d = fabs(f - orc_e4m3_value(c));        /* exact: both <= 2^9, f is a float */
        if (d < bd || (d == bd && (c & 1) == 0)) { bd = d; best = c; }
    }
    return best;                                       /* f > 448 lands on 126 */
}

/* E2M1 magnitudes; the index is also the 3-bit magnitude code. */
static const double kGrid[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};
/* midpoint between grid[i] and grid[i+1] */
static const double kMid[7] = {0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0};

int orc_e2m1_index(double a, double vS) {
    int k = 0;
    for (int i = 0; i < 7; ++i) {
        double t = kMid[i] * vS;                       /* exact (<= 31 significant bits) */
        if (a > t) k = i + 1;
        else if (a == t) { k = ((i & 1) == 0) ? i : i + 1; break; }  /* tie: even index */
        else break;
    }
    return k;
}

static double bf16_to_double(uint16_t b) {
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

static int bf16_is_finite(uint16_t b) { return (b & 0x7F80u) != 0x7F80u; }

/* ---- objective ---------------------------------------------------------- */

/* The loss of a group given its 16 magnitudes a[j] (exact doubles of bf16 or
 * FP32 values). */
static double group_loss_abs(const double* a, const float* h, float S, int code) {
    double v = orc_e4m3_value(code);
    if (v < 0.0) return NAN;
    double vS = v * (double)S;                         /* exact: 4 x 24 bits */
    double L = 0.0;
    for (int j = 0; j < 16; ++j) {
        double q = (vS > 0.0) ? kGrid[orc_e2m1_index(a[j], vS)] : 0.0;
        double d = a[j] - q * vS;                      /* exact: a and q*vS within a factor 2 */
        double hj = h ? (double)h[j] : 1.0;
        L += hj * (d * d);
    }
    return L;
}

static void abs_bf16(const uint16_t* w, double* a, int* neg) {
    for (int j = 0; j < 16; ++j) {
        a[j] = fabs(bf16_to_double(w[j]));
        neg[j] = (w[j] & 0x8000u) != 0;
    }
}

static void abs_f32(const float* w, double* a, int* neg) {
    for (int j = 0; j < 16; ++j) {
        a[j] = fabs((double)w[j]);
        neg[j] = signbit(w[j]) != 0;
    }
}

double orc_group_loss(const uint16_t* w, const float* h, float S, int code) {
    double a[16];
    int neg[16];
    abs_bf16(w, a, neg);
    return group_loss_abs(a, h, S, code);
}

double orc_group_loss_f32(const float* w, const float* h, float S, int code) {
    double a[16];
    int neg[16];
    abs_f32(w, a, neg);
    return group_loss_abs(a, h, S, code);
}

/* ---- calibration statistic: diagonal Hessian ----------------------------- */

void orc_diag_hessian(const uint16_t* X, int64_t tokens, int64_t in, int64_t ldx,
                      float* h, int accumulate) {
    /* acc_j = sum over t in increasing order of x_tj^2, in double.  The loops
     * run row by row only so that memory is read in order; each column's sum
     * still adds its terms in token order. */
    double* acc = (double*)calloc((size_t)(in > 0 ? in : 1), sizeof(double));
    if (!acc) return;
    for (int64_t t = 0; t < tokens; ++t) {
        const uint16_t* row = X + t * ldx;
        for (int64_t j = 0; j < in; ++j) {
            double x = bf16_to_double(row[j]);
            acc[j] += x * x;                           /* x*x exact: 16 significant bits */
        }
    }
    for (int64_t j = 0; j < in; ++j) {
        double s = accumulate ? (double)h[j] : 0.0;
        h[j] = (float)(s + acc[j]);
    }
    free(acc);
}

/* ---- global scale -------------------------------------------------------- */

int orc_global_scale(const uint16_t* W, int64_t out, int64_t in, int64_t ldw,
                     float q_max, float* S, float* amax) {
    double m = 0.0;
    for (int64_t r = 0; r < out; ++r)
        for (int64_t j = 0; j < in; ++j) {
            uint16_t b = W[r * ldw + j];
            if (!bf16_is_finite(b)) { *S = NAN; if (amax) *amax = NAN; return -5; }
            double a = fabs(bf16_to_double(b));
            if (a > m) m = a;
        }
    float fm = (float)m;                               /* exact: a bf16 value */
    float denom = q_max * 6.0f;                        /* fl32(Q * 6) */
    *S = (fm == 0.0f) ? 0.0f : fm / denom;             /* one IEEE float division */
    if (amax) *amax = fm;
    return 0;
}

/* ---- the windowed scale sweep ------------------------------------------- */

/* Base code from the group's magnitudes; a[j] are exact values of FP32 (or
 * bf16) numbers, so their maximum is an FP32 value. */
static int base_code_abs(const double* a16, float S) {
    double a = 0.0;
    for (int j = 0; j < 16; ++j)
        if (a16[j] > a) a = a16[j];
    if (a == 0.0) return 0;
    float t = (float)a / 6.0f;                         /* fl32(a / 6) */
    float u = t / S;                                   /* fl32(. / S) */
    int b = orc_e4m3_nearest((double)u);
    if (b < 1) b = 1;
    if (b > 126) b = 126;
    return b;
}

int orc_base_code(const uint16_t* w, float S) {
    double a[16];
    int neg[16];
    abs_bf16(w, a, neg);
    return base_code_abs(a, S);
}

int orc_base_code_f32(const float* w, float S) {
    double a[16];
    int neg[16];
    abs_f32(w, a, neg);
    return base_code_abs(a, S);
}

static int clamp_code(int c) { return c < 1 ? 1 : (c > 126 ? 126 : c); }

static void sweep_group_abs(const double* a, const int* neg, const float* h, float S, int lo,
                            int hi, uint8_t* codes8, uint8_t* scale, int8_t* offset, double* loss) {
    int b = base_code_abs(a, S);
    uint8_t nib[16];
    if (b == 0) {                                      /* all-zero group */
        if (codes8) memset(codes8, 0, 8);
        if (scale) *scale = 0;
        if (offset) *offset = 0;
        if (loss) *loss = 0.0;
        return;
    }
    double best = INFINITY;
    int bc = b, bk = 0;
    for (int k = lo; k <= hi; ++k) {                   /* ascending offsets */
        int c = clamp_code(b + k);
        double L = group_loss_abs(a, h, S, c);
        if (L < best) { best = L; bc = c; bk = k; }    /* strict: ties keep lowest offset */
    }
    double vS = orc_e4m3_value(bc) * (double)S;
    for (int j = 0; j < 16; ++j) {
        int k = orc_e2m1_index(a[j], vS);
        nib[j] = (uint8_t)((k != 0 && neg[j]) ? (8 | k) : k);
    }
    if (codes8)
        for (int i = 0; i < 8; ++i) codes8[i] = (uint8_t)(nib[2 * i] | (nib[2 * i + 1] << 4));
    if (scale) *scale = (uint8_t)bc;
    if (offset) *offset = (int8_t)bk;
    if (loss) *loss = best;
}

void orc_sweep_group(const uint16_t* w, const float* h, float S, int lo, int hi,
                     uint8_t* codes8, uint8_t* scale, int8_t* offset, double* loss) {
    double a[16];
    int neg[16];
    abs_bf16(w, a, neg);
    sweep_group_abs(a, neg, h, S, lo, hi, codes8, scale, offset, loss);
}

void orc_sweep_group_f32(const float* w, const float* h, float S, int lo, int hi,
                         uint8_t* codes8, uint8_t* scale, int8_t* offset, double* loss) {
    double a[16];
    int neg[16];
    abs_f32(w, a, neg);
    sweep_group_abs(a, neg, h, S, lo, hi, codes8, scale, offset, loss);
}

void orc_sweep_group_f32_list(const float* w, const float* h, int64_t n, float S, int lo, int hi,
                              uint8_t* codes, uint8_t* scales, int8_t* offsets, double* losses) {
    for (int64_t i = 0; i < n; ++i)
        orc_sweep_group_f32(w + 16 * i, h ? h + 16 * i : NULL, S, lo, hi, codes + 8 * i,
                            scales + i, offsets ? offsets + i : NULL, losses ? losses + i : NULL);
}

/* E2M1 nibbles (sign << 3 | magnitude index; +0 for a zero magnitude) of n FP32
 * values w[i], each at its own scale vS[i] > 0 (an exact double); vS[i] == 0
 * gives nibble 0.  The quantization step of a quantizer that has already chosen
 * its scales, e.g. inside GPTQ's column loop. */
void orc_e2m1_quantize_list(const float* w, const double* vS, int64_t n, uint8_t* nib) {
    for (int64_t i = 0; i < n; ++i) {
        if (!(vS[i] > 0.0)) { nib[i] = 0; continue; }
        int k = orc_e2m1_index(fabs((double)w[i]), vS[i]);
        nib[i] = (uint8_t)((k != 0 && signbit(w[i])) ? (8 | k) : k);
    }
}

void orc_sweep_quantize(const uint16_t* W, int64_t out, int64_t in, int64_t ldw,
                        const float* h, float S, int lo, int hi,
                        uint8_t* codes, uint8_t* scales, int8_t* offsets) {
    int64_t G = in / 16;
    for (int64_t r = 0; r < out; ++r)
        for (int64_t g = 0; g < G; ++g)
            orc_sweep_group(W + r * ldw + g * 16, h ? h + g * 16 : NULL, S, lo, hi,
                            codes + r * (in / 2) + g * 8, scales + r * G + g,
                            offsets ? offsets + r * G + g : NULL, NULL);
}

/* ---- activations, quantized online ---------------------------------------
 * [ScaleSweep] sec. 1-3 and "Experimental Results": in the W+A settings the
 * activations are NVFP4 too, with the MSE objective (no Hessian) and the
 * [-3, +7] window.  Reading taken where the page is silent: the global scale
 * is dynamic, one per token (row), by the same formula as for a weight tensor,
 * and each row is then swept as a one-row matrix. */
int orc_quantize_activations(const uint16_t* A, int64_t tokens, int64_t in, int64_t lda,
                             float q_max, int lo, int hi, float* S, uint8_t* codes,
                             uint8_t* scales, int8_t* offsets) {
    int64_t G = in / 16;
    int rc = 0;
    for (int64_t t = 0; t < tokens; ++t) {
        const uint16_t* row = A + t * lda;
        uint8_t* crow = codes + t * (in / 2);
        uint8_t* srow = scales + t * G;
        int8_t* orow = offsets ? offsets + t * G : NULL;
        if (orc_global_scale(row, 1, in, lda, q_max, &S[t], NULL) != 0) {
            rc = -5;                                   /* S[t] is NaN; outputs zero */
            memset(crow, 0, (size_t)(in / 2));
            memset(srow, 0, (size_t)G);
            if (orow) memset(orow, 0, (size_t)G);
            continue;
        }
        orc_sweep_quantize(row, 1, in, lda, NULL, S[t], lo, hi, crow, srow, orow);
    }
    return rc;
}

void orc_sweep_group_list(const uint16_t* w, const float* h, int64_t n, float S,
                          int lo, int hi, uint8_t* codes, uint8_t* scales,
                          int8_t* offsets, double* losses) {
    for (int64_t i = 0; i < n; ++i)
        orc_sweep_group(w + 16 * i, h ? h + 16 * i : NULL, S, lo, hi, codes + 8 * i,
                        scales + i, offsets ? offsets + i : NULL, losses ? losses + i : NULL);
}

void orc_group_loss_list(const uint16_t* w, const float* h, int64_t n, float S,
                         const uint8_t* code, double* losses) {
    for (int64_t i = 0; i < n; ++i)
        losses[i] = orc_group_loss(w + 16 * i, h ? h + 16 * i : NULL, S, code[i]);  /* code 0: all zero */
}

void orc_packed_loss_list(const uint16_t* w, const float* h, int64_t n, float S,
                          const uint8_t* codes, const uint8_t* scale, double* losses) {
    for (int64_t i = 0; i < n; ++i) {
        double v = orc_e4m3_value(scale[i]);
        if (v < 0.0) { losses[i] = NAN; continue; }
        double vS = v * (double)S;
        double L = 0.0;
        for (int j = 0; j < 16; ++j) {
            uint8_t byte = codes[8 * i + j / 2];
            uint8_t nib = (j & 1) ? (byte >> 4) : (byte & 15);
            double r = kGrid[nib & 7] * vS;                /* exact */
            if (nib & 8) r = -r;
            double d = bf16_to_double(w[16 * i + j]) - r;  /* exact */
            double hj = h ? (double)h[16 * i + j] : 1.0;
            L += hj * (d * d);
        }
        losses[i] = L;
    }
}

/* ---- dequantize ----------------------------------------------------------- */

void orc_dequantize(const uint8_t* codes, const uint8_t* scales, float S,
                    int64_t out, int64_t in, float* W_out) {
    int64_t G = in / 16;
    for (int64_t r = 0; r < out; ++r)
        for (int64_t j = 0; j < in; ++j) {
            uint8_t byte = codes[r * (in / 2) + j / 2];
            uint8_t nib = (j & 1) ? (byte >> 4) : (byte & 15);
            double v = orc_e4m3_value(scales[r * G + j / 16]);
            if (v < 0.0) v = NAN;
            double mag = kGrid[nib & 7] * v * (double)S;   /* exact (<= 30 bits) */
            float f = (float)mag;                          /* one rounding to float */
            W_out[r * in + j] = (nib & 8) ? -f : f;
        }
}
