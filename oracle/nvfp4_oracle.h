/*
 * nvfp4_oracle.h -- plain, slow CPU oracle for Hessian-weighted NVFP4
 * block-scale selection.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may include, link
 * or call this code: it exists so that tests, the smoke check and the CPU
 * baseline of the benchmark can check the CUDA library against an
 * independent, obviously-correct definition.  It shares no source, header,
 * table or helper with the CUDA library.
 *
 * Every decision is taken exactly (in exact real arithmetic, realised with
 * IEEE double where every product involved is exactly representable); the
 * reconstruction loss is accumulated in double.  Each function cites the
 * passage of the method it follows:
 *   [H-Scale]    "H-Scale: Hessian-Guided Scale Refinement for NVFP4 Sub-Byte
 *                LLM Inference" (paperlayer.ai summary), sections 3 and B.
 *   [ScaleSweep] "Technical Summary: ScaleSweep" (gist.science), sections 2
 *                and 3.
 *   [SchurRep]   "Replay the Curvature" (paperlayer.ai summary), section 1
 *                (4.5 bits per value).
 *
 * Parity status: every function below is pinned by tests under tests/
 * (closed forms, library conversions, brute force, invariants) except the
 * page's calibration microcase, whose inputs are not printed ("parity
 * unpinned" for that example only).
 */
#ifndef NVFP4_ORACLE_H
#define NVFP4_ORACLE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Value of E4M3 code `code` (0..126), exactly, as a double.  Code 127 (NaN)
 * and anything outside 0..126 returns -1.  [ScaleSweep] sec. 2: the 126
 * positive finite FP8 scales. */
double orc_e4m3_value(int code);

/* Nearest E4M3 code to f >= 0 (ties to the even code), saturating to 126
 * (value 448) for f above the largest finite value.  Returns -1 for NaN or
 * negative input.  [ScaleSweep] sec. 2: s_base is the FP8-rounded maximum. */
int orc_e4m3_nearest(double f);

/* E2M1 magnitude index k in 0..7 (grid 0,0.5,1,1.5,2,3,4,6) nearest to the
 * exact real a / vS, ties to the even index, saturating at 6.  a >= 0 and
 * vS > 0 must be exact doubles whose products with the midpoints are exact
 * (true for |bf16| and E4M3 x FP32).  [H-Scale] sec. 3: E2M1 values with an
 * E4M3 scale; round to nearest. */
int orc_e2m1_index(double a, double vS);

/* Weighted reconstruction loss of one 16-element group at E4M3 code `code`:
 *   L = sum_j h_j (|w_j| - g[k_j] * v(code) * S)^2,
 * h == NULL meaning h_j = 1 (plain MSE).  [H-Scale] sec. 3 (diagonal-Hessian
 * weighted objective); [ScaleSweep] sec. 1 (MSE / WMSE). */
double orc_group_loss(const uint16_t* w_bf16, const float* h, float S, int code);

/* h_j (+)= sum_t x_tj^2 over X[tokens, in] (bf16, row stride ldx elements);
 * summed in double over exact bf16 values and rounded once to float.  With
 * accumulate != 0 the old h_j is added (in double) before that rounding.
 * [H-Scale] sec. B: h = diag(X^T X). */
void orc_diag_hessian(const uint16_t* X, int64_t tokens, int64_t in, int64_t ldx,
                      float* h, int accumulate);

/* amax = max |w| over W[out, in] (row stride ldw); S = fl32(amax / fl32(q_max*6)).
 * amax == 0 gives S == 0.  Returns 0, or -5 if a non-finite value is present
 * (S and amax are then written as NaN).  [ScaleSweep] sec. 2: global scale
 * S = max|x| / (Q * 6). */
int orc_global_scale(const uint16_t* W, int64_t out, int64_t in, int64_t ldw,
                     float q_max, float* S, float* amax);

/* Base code of one group: b = clamp(nearest(fl32(fl32(a/6)/S)), 1, 126) for
 * group absmax a > 0; returns 0 for an all-zero group. */
int orc_base_code(const uint16_t* w_bf16, float S);

/* Sweep one group: for k = lo..hi (ascending), c = clamp(b+k, 1, 126), keep the
 * strictly smallest loss (ties to the lowest offset); then quantize and pack.
 * codes8[i] holds element 2i in its low nibble and 2i+1 in its high nibble;
 * nibble = sign<<3 | k with sign set only for a negative nonzero code.
 * Writes the chosen code to *scale, the winning offset to *offset and its loss
 * to *loss (any output pointer may be NULL).  An all-zero group gives scale 0,
 * zero codes, offset 0 and loss 0.  [H-Scale] sec. 3 and B. */
void orc_sweep_group(const uint16_t* w_bf16, const float* h, float S, int lo, int hi,
                     uint8_t* codes8, uint8_t* scale, int8_t* offset, double* loss);

/* FP32-input forms, for quantizers whose weights are FP32 values rather than
 * bf16 -- GPTQ's error-updated columns ([H-Scale] sec. B "GPTQ Integration":
 * H-Scale replaces GPTQ's local quantization call).  The same definitions with
 * w_j an FP32 number: exact E2M1 decisions, base code from fl32(fl32(a/6)/S),
 * loss in double. */
double orc_group_loss_f32(const float* w, const float* h, float S, int code);
int orc_base_code_f32(const float* w, float S);
void orc_sweep_group_f32(const float* w, const float* h, float S, int lo, int hi,
                         uint8_t* codes8, uint8_t* scale, int8_t* offset, double* loss);
void orc_sweep_group_f32_list(const float* w, const float* h, int64_t n, float S, int lo, int hi,
                              uint8_t* codes, uint8_t* scales, int8_t* offsets, double* losses);
/* Nibbles of n FP32 values, each at an already chosen scale vS[i] (exact
 * double; 0 gives nibble 0). */
void orc_e2m1_quantize_list(const float* w, const double* vS, int64_t n, uint8_t* nib);

/* Whole matrix: W[out, in] bf16 row stride ldw, h[in] or NULL.
 * codes[out, in/2], scales[out, in/16], offsets[out, in/16] (NULL allowed). */
void orc_sweep_quantize(const uint16_t* W, int64_t out, int64_t in, int64_t ldw,
                        const float* h, float S, int lo, int hi,
                        uint8_t* codes, uint8_t* scales, int8_t* offsets);

/* Activations quantized online ([ScaleSweep] W+A settings: the MSE sweep
 * applied to activations).  Per token t (row of A[tokens, in], row stride lda):
 *   S[t] = fl32(amax_t / fl32(q_max * 6))   (0 for an all-zero row), then the
 * row is swept as orc_sweep_quantize does with h == NULL and window [lo, hi].
 * A row holding Inf or NaN gets S[t] = NaN and zero codes, scales and offsets;
 * the return is -5 if any row did, else 0.  codes[tokens, in/2],
 * scales[tokens, in/16], offsets[tokens, in/16] (NULL allowed). */
int orc_quantize_activations(const uint16_t* A, int64_t tokens, int64_t in, int64_t lda,
                             float q_max, int lo, int hi, float* S, uint8_t* codes,
                             uint8_t* scales, int8_t* offsets);

/* List form used for sampled checks: n groups, w[n,16], h[n,16] or NULL. */
void orc_sweep_group_list(const uint16_t* w, const float* h, int64_t n, float S,
                          int lo, int hi, uint8_t* codes, uint8_t* scales,
                          int8_t* offsets, double* losses);

/* Loss of n groups at given codes: w[n,16], h[n,16] or NULL, code[n]. */
void orc_group_loss_list(const uint16_t* w, const float* h, int64_t n, float S,
                         const uint8_t* code, double* losses);

/* Loss of n groups as packed: w[n,16], h[n,16] or NULL, codes[n,8] (nibbles as
 * in orc_sweep_group), scale[n] E4M3 codes.  The reconstruction of element j
 * is decoded from its nibble (not re-derived), so this scores any packer's
 * actual output: L = sum_j h_j (w_j - sign_j g[k_j] v S)^2. */
void orc_packed_loss_list(const uint16_t* w, const float* h, int64_t n, float S,
                          const uint8_t* codes, const uint8_t* scale, double* losses);

/* W_out[r, j] = sign * fl32(g[k] * v(scale)) * S, float32 [out, in]. */
void orc_dequantize(const uint8_t* codes, const uint8_t* scales, float S,
                    int64_t out, int64_t in, float* W_out);

#ifdef __cplusplus
}
#endif
#endif
