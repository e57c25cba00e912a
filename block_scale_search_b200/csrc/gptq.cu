// gptq.cu -- H-Scale as the local quantizer inside GPTQ.
//
// H-Scale summary, sec. B "Implementation" and "GPTQ Integration": in GPTQ,
// H-Scale replaces only the local quantization call; the inverse-Cholesky
// processing, the error computation and its propagation stay GPTQ's own.  The
// GPTQ steps are the standard algorithm in the given column order:
//   H = X^T X; a column whose diagonal is 0 gets H_jj = 1 and zero weights;
//   H += damp * mean(diag H) * I; U = the upper Cholesky factor of H^-1;
//   column by column: quantize w_j, err_j = (w_j - q_j) / U_jj, and every later
//   column k takes w_k -= err_j U_jk.
// The local call: at the first column of each 16-column group, every row's
// E4M3 scale code for the group is chosen by the windowed sweep on the group's
// current (error-updated) FP32 weights, with h = diag(X^T X) and the global
// scale S of the original weights; each column of the group is then quantized
// at its turn with that scale (exact E2M1 round-to-nearest-even).
//
// On the device:
//   * h and S: this library's diagonal-Hessian and global-scale kernels;
//   * H = X^T X: cuBLAS GEMMs (bf16 in, FP32 accumulate), only the lower
//     blocks of a 4 x 4 split for in >= 4096 (the factorization reads one
//     triangle);
//   * the dead-column rule, the damping and the FP16 scales: gptq_prep_kernel;
//   * no inverse is formed.  With J the order-reversing permutation, the lower
//     Cholesky factor L' of J H J (cuSOLVER potrf, FP32) gives H = R R^T with
//     R = J L' J upper, and U = R^-1.  Reflecting the n x n array about its
//     anti-diagonal in place, before (J H J, H symmetric) and after, turns the
//     column-major L' into R row-major: R[j][k] at j * in + k, k >= j;
//   * the column loop runs in the R form of GPTQ's recurrence.  Quantizing
//     column j at its turn and propagating err_j = (w_j - q_j) / U_jj gives,
//     by induction over the columns, W - Q = Err U, so Err = (W - Q) R.  Then,
//     with D = W - Q and a 16-column group starting at column g0, the group's
//     current weights are  W_grp + (D[:, <g0] R[<g0, grp]) U_grp,  where
//     U_grp = R_grp^-1 is the inverse of the group's 16 x 16 diagonal block of
//     R (U is block upper triangular); inside the group the updates use U_grp
//     and err_j = (w_j - q_j) R_jj.  gptq_udiag_kernel inverts the diagonal
//     blocks (FP64);
//   * GPTQ's lazy batches, 512 columns each, in four parts of 128:
//     gptq_rblock_kernel runs the columns of one part, two threads per row --
//     each group's sums from the earlier groups of the part, its current
//     weights, the local call, the exact quantization and the in-group
//     updates -- and writes the part's D.  After each part a small GEMM adds
//     the batch's parts so far to the next part's sums; after the batch one
//     GEMM adds the batch to every later column's sums:
//     P[:, >] += D[:, batch] R[batch, >].  The GEMMs run
//     on the tensor cores as three FP16 products with FP32 accumulation,
//     D_hi R_hi + D_hi R_lo + D_lo R_hi: each FP32 operand, scaled by a power
//     of two that keeps it inside FP16's range, is split into its FP16
//     rounding and the FP16 rounding of the remainder (gptq_rsplit_kernel for
//     R; the batch kernel writes D's parts); the GEMM's alpha undoes the
//     scales exactly.  Each P element is read and written once per 512
//     columns, and the GEMM's K (3 x 512) keeps its FP32 read-modify-write of
//     P shorter than its products.
// Rows are independent in GPTQ (R is shared), so the batch kernel needs no
// communication between rows.  The device arithmetic is FP32 (the update GEMM
// about 2^-21 relative per product): results drift from the FP64 oracle's
// after a quantization decision flips, which a row then carries through its
// later columns.
#include <cublas_v2.h>
#include <cusolverDn.h>

#include <mutex>
#include <vector>

#include "nvfp4_kernels.cuh"
#include "nvfp4hs.h"
#include "sweep_core.cuh"

namespace nvfp4 {

namespace {

constexpr int kGB = 128;        // columns per batch kernel launch
constexpr int kCat = 3 * kGB;   // K of the split update per 128 columns
constexpr int kSub = 4;         // batch-kernel launches per lazy batch (512 columns)
constexpr int kDs = kGB + 4;    // a row's D in shared memory (16-byte rows)
// R's blocks above the diagonal blocks of one part: for group b, the rows of
// the part's earlier groups (16 b of them) by the group's 16 columns.
constexpr int kRsFloats = 256 * (kGB / 16) * (kGB / 16 - 1) / 2;

size_t al256(size_t x) { return (x + 255) & ~size_t{255}; }

// ------------------------------------------------------------ the local call

// Scaled group weights h' (the sweep's power-of-two rescaling) from 16 h.
__device__ __forceinline__ void weights_from(const float* h16, f32x2_t (&h2)[8], float& hs,
                                             float& hsum) {
  float hmax = 0.0f;
#pragma unroll
  for (int j = 0; j < 16; ++j) hmax = fmaxf(hmax, h16[j]);
  hs = weight_scale(hmax);
  hsum = 0.0f;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    h2[i] = f2_pack(h16[2 * i] * hs, h16[2 * i + 1] * hs);
    hsum += h16[2 * i] * hs + h16[2 * i + 1] * hs;
  }
}

// The E4M3 scale code the windowed sweep picks for 16 FP32 weights w (0 for
// an all-zero group), one thread: the fast FP32 losses of the weight sweep
// (fast_candidate_loss), its near-tie threshold, and where that flags other
// candidates, their exact losses in FP64 with exact E2M1 decisions, summed in
// element order; the first strict minimum in offset order wins.  h16 NULL:
// plain MSE.
template <bool kWeighted, int kK>
__device__ int local_sweep_f32(const float* w, const float* h16, const ScaleConsts& sc,
                               const CandEntry* tab, int lo, int K) {
  float a = 0.0f;
#pragma unroll
  for (int j = 0; j < 16; ++j) a = fmaxf(a, fabsf(w[j]));
  if (!(a > 0.0f)) return 0;
  f32x2_t h2[8];
  float hs = 1.0f, hsum = 16.0f;
  if constexpr (kWeighted) {
    weights_from(h16, h2, hs, hsum);
  } else {
#pragma unroll
    for (int i = 0; i < 8; ++i) h2[i] = f2_pack(1.0f, 1.0f);
  }
  f32x2_t y2[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    f32x2_t a2 = f2_pack(w[2 * i], w[2 * i + 1]);
    if (sc.tiny_s) a2 = f2_mul(a2, f2_pack(sc.p, sc.p));
    y2[i] = f2_mul(a2, f2_pack(sc.inv_sp, sc.inv_sp));
  }
  const float S = sc.S;
  const int b = clamp_code(e4m3_code_rne_sat(__fdiv_rn(__fdiv_rn(a, 6.0f), S)));
  const CandEntry* ce = tab + (b + lo + kTabOffset);
  uint32_t kbest = 0xFFFFFFFFu, ksec = 0xFFFFFFFFu;
  auto cand = [&](int i) {
    const float Li = fast_candidate_loss<kWeighted>(y2, h2, ce[i]);
    const uint32_t key = (__float_as_uint(Li) & ~0xFu) | static_cast<uint32_t>(i);
    ksec = min(ksec, max(kbest, key));
    kbest = min(kbest, key);
  };
  if constexpr (kK > 0) {
#pragma unroll
    for (int i = 0; i < kK; ++i) cand(i);
  } else {
    for (int i = 0; i < K; ++i) cand(i);
  }
  int bi = static_cast<int>(kbest & 0xFu);
  const float best = __uint_as_float(kbest & ~0xFu) * (1.0f + 0x1p-18f);
  const float second = __uint_as_float(ksec & ~0xFu);
  constexpr float c1 = 0x1p-19f, c2 = 0x1p-15f;
  constexpr float k2 = 1.0f / (2.0f * (1.0f - c2));
  auto threshold = [&](float A) {
    const float ca = c1 * sqrt_approx(A);
    const float sr = (ca + sqrt_approx(fmaf(ca, ca, 4.0f * (1.0f - c2) * best))) * k2;
    return sr * sr * (1.0f + 0x1p-16f);
  };
  const float ymax = (sc.tiny_s ? a * sc.p : a) * sc.inv_sp;
  float T = threshold(hsum * ymax * ymax);
  bool flagged = second <= T;
  if (flagged) {
    f32x2_t A2 = f2_pack(0.0f, 0.0f);
#pragma unroll
    for (int i = 0; i < 8; ++i) A2 = f2_fma(kWeighted ? f2_mul(h2[i], y2[i]) : y2[i], y2[i], A2);
    float A0, A1;
    f2_unpack(A2, A0, A1);
    T = threshold(A0 + A1);
    flagged = second <= T;
  }
  if (flagged) {  // rare: the definition's own arithmetic decides among the near-ties
    double bestd = __longlong_as_double(0x7FF0000000000000ll);
    int bid = bi;
    for (int i = 0; i < K; ++i) {
      // the fast loss again (flagged groups are rare; no per-candidate array)
      if (fast_candidate_loss<kWeighted>(y2, h2, ce[i]) > T) continue;
      const CandEntry t = ce[i];
      const float ivl = t.iv * (1.0f - 0x1p-20f);
      const double vS = __dmul_rn(static_cast<double>(t.v), static_cast<double>(S));
      double Ld = 0.0;
      for (int j = 0; j < 16; ++j) {
        const float aj = fabsf(w[j]);
        const float yj = (sc.tiny_s ? aj * sc.p : aj) * sc.inv_sp;
        const uint32_t k = exact_e2m1_one(yj * ivl, aj, t.v, S);
        const double q = static_cast<double>(e2m1_nibble_value(k));
        const double d = fma(-q, vS, static_cast<double>(aj));  // exact
        const double hj = kWeighted ? static_cast<double>(h16[j]) : 1.0;
        Ld = __dadd_rn(Ld, __dmul_rn(hj, __dmul_rn(d, d)));
      }
      if (Ld < bestd) { bestd = Ld; bid = i; }
    }
    bi = bid;
  }
  return clamp_code(b + lo + bi);
}

// local_sweep_f32 shared by the two lanes of a pair (lanes 2k and 2k + 1 of a
// warp, both holding the same 16 weights w): lane `half` scores candidates
// half, half + 2, ..., and the pair's smallest and second-smallest keys are
// combined by shuffles, so both lanes take the same decision as one lane
// scoring them all.  pm holds whole pairs and every lane in it must call this.
template <bool kWeighted, int kK>
__device__ int local_sweep_f32_pair(const float* w, const float* h16, const ScaleConsts& sc,
                                    const CandEntry* tab, int lo, int K, int half, unsigned pm) {
  float a = 0.0f;
#pragma unroll
  for (int j = 0; j < 16; ++j) a = fmaxf(a, fabsf(w[j]));
  f32x2_t h2[8];
  float hs = 1.0f, hsum = 16.0f;
  if constexpr (kWeighted) {
    weights_from(h16, h2, hs, hsum);
  } else {
#pragma unroll
    for (int i = 0; i < 8; ++i) h2[i] = f2_pack(1.0f, 1.0f);
  }
  f32x2_t y2[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    f32x2_t a2 = f2_pack(w[2 * i], w[2 * i + 1]);
    if (sc.tiny_s) a2 = f2_mul(a2, f2_pack(sc.p, sc.p));
    y2[i] = f2_mul(a2, f2_pack(sc.inv_sp, sc.inv_sp));
  }
  const float S = sc.S;
  const int b = clamp_code(e4m3_code_rne_sat(__fdiv_rn(__fdiv_rn(a, 6.0f), S)));
  const CandEntry* ce = tab + (b + lo + kTabOffset);
  uint32_t kbest = 0xFFFFFFFFu, ksec = 0xFFFFFFFFu;
  auto cand = [&](int i) {
    const float Li = fast_candidate_loss<kWeighted>(y2, h2, ce[i]);
    const uint32_t key = (__float_as_uint(Li) & ~0xFu) | static_cast<uint32_t>(i);
    ksec = min(ksec, max(kbest, key));
    kbest = min(kbest, key);
  };
  if constexpr (kK > 0) {
#pragma unroll
    for (int m = 0; m < kK; m += 2) cand(m + half);
  } else {
    for (int i = half; i < K; i += 2) cand(i);
  }
  {  // the pair's two smallest keys
    const uint32_t ob = __shfl_xor_sync(pm, kbest, 1), os = __shfl_xor_sync(pm, ksec, 1);
    ksec = min(min(ksec, os), max(kbest, ob));
    kbest = min(kbest, ob);
  }
  if (!(a > 0.0f)) return 0;
  int bi = static_cast<int>(kbest & 0xFu);
  const float best = __uint_as_float(kbest & ~0xFu) * (1.0f + 0x1p-18f);
  const float second = __uint_as_float(ksec & ~0xFu);
  constexpr float c1 = 0x1p-19f, c2 = 0x1p-15f;
  constexpr float k2 = 1.0f / (2.0f * (1.0f - c2));
  auto threshold = [&](float A) {
    const float ca = c1 * sqrt_approx(A);
    const float sr = (ca + sqrt_approx(fmaf(ca, ca, 4.0f * (1.0f - c2) * best))) * k2;
    return sr * sr * (1.0f + 0x1p-16f);
  };
  const float ymax = (sc.tiny_s ? a * sc.p : a) * sc.inv_sp;
  float T = threshold(hsum * ymax * ymax);
  bool flagged = second <= T;
  if (flagged) {
    f32x2_t A2 = f2_pack(0.0f, 0.0f);
#pragma unroll
    for (int i = 0; i < 8; ++i) A2 = f2_fma(kWeighted ? f2_mul(h2[i], y2[i]) : y2[i], y2[i], A2);
    float A0, A1;
    f2_unpack(A2, A0, A1);
    T = threshold(A0 + A1);
    flagged = second <= T;
  }
  if (flagged) {  // rare: both lanes run the definition's own arithmetic on every candidate
    double bestd = __longlong_as_double(0x7FF0000000000000ll);
    int bid = bi;
    for (int i = 0; i < K; ++i) {
      if (fast_candidate_loss<kWeighted>(y2, h2, ce[i]) > T) continue;
      const CandEntry t = ce[i];
      const float ivl = t.iv * (1.0f - 0x1p-20f);
      const double vS = __dmul_rn(static_cast<double>(t.v), static_cast<double>(S));
      double Ld = 0.0;
      for (int j = 0; j < 16; ++j) {
        const float aj = fabsf(w[j]);
        const float yj = (sc.tiny_s ? aj * sc.p : aj) * sc.inv_sp;
        const uint32_t k = exact_e2m1_one(yj * ivl, aj, t.v, S);
        const double q = static_cast<double>(e2m1_nibble_value(k));
        const double d = fma(-q, vS, static_cast<double>(aj));  // exact
        const double hj = kWeighted ? static_cast<double>(h16[j]) : 1.0;
        Ld = __dadd_rn(Ld, __dmul_rn(hj, __dmul_rn(d, d)));
      }
      if (Ld < bestd) { bestd = Ld; bid = i; }
    }
    bi = bid;
  }
  return clamp_code(b + lo + bi);
}

// One FP32 weight quantized at E4M3 code `code` (0: the group is all zero):
// its nibble (sign << 3 | E2M1 index, +0 for a zero magnitude) and its
// reconstruction sign * g * v * S (one rounding).  The E2M1 decision is exact
// (the bracketed quotient; fma(m v, S, -|w|) where a midpoint lies inside).
__device__ __forceinline__ uint32_t quantize_one(float w, int code, const ScaleConsts& sc,
                                                 const CandEntry* tab, float& q) {
  if (code == 0) {
    q = 0.0f;
    return 0u;
  }
  const CandEntry t = tab[code + kTabOffset];
  const float aw = fabsf(w);
  const float y = (sc.tiny_s ? aw * sc.p : aw) * sc.inv_sp;
  const uint32_t k = exact_e2m1_one(y * (t.iv * (1.0f - 0x1p-20f)), aw, t.v, sc.S);
  const float mag = (e2m1_nibble_value(k) * t.v) * sc.S;
  const bool neg = signbit(w) && k != 0u;
  q = neg ? -mag : mag;
  return neg ? (k | 8u) : k;
}

// --------------------------------------------------------------- kernels

// The windowed sweep of an FP32 matrix, one thread per group: the local call
// and the quantization of the 16 weights at the chosen scale, no propagation.
template <bool kWeighted, int kK>
__global__ void __launch_bounds__(128)
sweep_f32_kernel(const float* __restrict__ W, int64_t out, int64_t G, int64_t ldw,
                 const float* __restrict__ h, const float* __restrict__ Sp, int lo, int hi,
                 uint8_t* __restrict__ codes, uint8_t* __restrict__ scales) {
  __shared__ CandEntry tab[kTabSize];
  fill_candidate_table(tab);
  __syncthreads();
  const ScaleConsts sc = scale_consts(*Sp);
  const int K = hi - lo + 1;
  for (int64_t gi = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; gi < out * G;
       gi += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t r = gi / G, g = gi - r * G;
    float w[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) w[j] = W[r * ldw + g * 16 + j];
    const int code = local_sweep_f32<kWeighted, kK>(w, kWeighted ? h + g * 16 : nullptr, sc, tab,
                                                    lo, K);
    uint32_t packed[2] = {0u, 0u};
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      float q;
      packed[j >> 3] |= quantize_one(w[j], code, sc, tab, q) << (4 * (j & 7));
    }
    *reinterpret_cast<uint2*>(codes + r * (G * 8) + g * 8) = make_uint2(packed[0], packed[1]);
    scales[gi] = static_cast<uint8_t>(code);
  }
}

// Dead columns, damping: one CTA.  H is symmetric (row- or column-major alike).
// Also the FP16 scales of the split update GEMMs, gs = {s_D, s_R, alpha, 1, 0}:
// powers of two with |D| s_D <= 2^14 and |R| s_R <= 2^14, where |D| = |W - q|
// <= amax + 6 * 448 * S (amax ~ S * 6 q_max) and every entry of row i of R is
// at most sqrt(H_ii) (H = R R^T); alpha = 1 / (s_D s_R).
__device__ __forceinline__ int pow2_floor_exp(float ratio) {
  if (!(ratio > 0.0f) || !isfinite(ratio)) return 0;
  int e;
  frexpf(ratio, &e);  // ratio in [2^(e-1), 2^e)
  return max(-60, min(60, e - 1));
}

__global__ void __launch_bounds__(256)
gptq_prep_kernel(float* __restrict__ H, int64_t in, float damp, uint8_t* __restrict__ dead,
                 const float* __restrict__ Sp, float q_max, float* __restrict__ gs) {
  __shared__ double part[256];
  __shared__ float mx[256];
  double s = 0.0;
  float m = 0.0f;
  for (int64_t j = threadIdx.x; j < in; j += blockDim.x) {
    float d = H[j * in + j];
    dead[j] = d == 0.0f ? 1 : 0;
    if (d == 0.0f) {
      d = 1.0f;
      H[j * in + j] = 1.0f;
    }
    s += static_cast<double>(d);
    m = fmaxf(m, d);
  }
  part[threadIdx.x] = s;
  mx[threadIdx.x] = m;
  __syncthreads();
  for (int o = 128; o > 0; o >>= 1) {
    if (threadIdx.x < o) {
      part[threadIdx.x] += part[threadIdx.x + o];
      mx[threadIdx.x] = fmaxf(mx[threadIdx.x], mx[threadIdx.x + o]);
    }
    __syncthreads();
  }
  const float lam = static_cast<float>(static_cast<double>(damp) * part[0] / static_cast<double>(in));
  for (int64_t j = threadIdx.x; j < in; j += blockDim.x) H[j * in + j] += lam;
  if (threadIdx.x == 0) {
    const float S = *Sp;
    const float dmax = S * (6.0f * q_max + 2688.0f) * (1.0f + 0x1p-10f);
    const float rmax = sqrtf(mx[0] + lam) * (1.0f + 0x1p-10f);
    const int kd = pow2_floor_exp(16384.0f / dmax), kr = pow2_floor_exp(16384.0f / rmax);
    gs[0] = ldexpf(1.0f, kd);
    gs[1] = ldexpf(1.0f, kr);
    gs[2] = ldexpf(1.0f, -kd - kr);
    gs[3] = 1.0f;
    gs[4] = 0.0f;
  }
}

// In place: a[r][c] <-> a[n-1-c][n-1-r] (reflection about the anti-diagonal;
// n a multiple of 16).  One 16 x 16 thread block per pair of 16 x 16 tiles:
// tile (bi, bj) pairs with tile (t-1-bj, t-1-bi), t = n / 16, so element
// (y, x) of the first is element (15-x, 15-y) of the second; blocks with
// bi + bj > t - 1 have nothing to do.  Both tiles are read and written in
// 16-float row segments through shared memory.
__global__ void __launch_bounds__(256)
antitranspose_kernel(float* __restrict__ a, int64_t n) {
  __shared__ float ta[16][17], tb[16][17];
  const int64_t t = n / 16;
  const int64_t bi = blockIdx.y, bj = blockIdx.x;
  if (bi + bj > t - 1) return;
  const int x = threadIdx.x & 15, y = threadIdx.x >> 4;
  float* A = a + (16 * bi + y) * n + 16 * bj + x;
  float* B = a + (16 * (t - 1 - bj) + y) * n + 16 * (t - 1 - bi) + x;
  ta[y][x] = *A;
  tb[y][x] = *B;
  __syncthreads();
  *A = tb[15 - x][15 - y];
  if (bi + bj < t - 1) *B = ta[15 - x][15 - y];
}

// A failed Cholesky factorization (devInfo != 0: the damped Hessian is not
// positive definite in FP32) is reported through the status word.
__global__ void gptq_status_kernel(const int* __restrict__ info, int n, int* status) {
  int bad = 0;
  for (int i = 0; i < n; ++i) bad |= info[i] != 0;
  if (bad && status) *status = -9;  // NVFP4_ERR_NUMERIC
}

// The inverses of R's 16 x 16 diagonal blocks (upper triangular), FP64 back
// substitution, one thread per column of an inverse: Ud[blk][i][k] =
// (R_blk^-1)[i][k], zero below the diagonal.  R row-major with stride in;
// entries below R's diagonal are not read.
__global__ void __launch_bounds__(128)
gptq_udiag_kernel(const float* __restrict__ R, int64_t in, float* __restrict__ Ud) {
  const int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (idx >= in) return;  // in / 16 blocks x 16 columns
  const int64_t blk = idx >> 4;
  const int k = static_cast<int>(idx & 15);
  const float* Rb = R + blk * 16 * in + blk * 16;
  double x[16];
#pragma unroll
  for (int i = 15; i >= 0; --i) {
    if (i > k) {
      x[i] = 0.0;
    } else {
      double s = i == k ? 1.0 : 0.0;
#pragma unroll
      for (int l = i + 1; l < 16; ++l)
        if (l <= k) s -= static_cast<double>(Rb[i * in + l]) * x[l];
      x[i] = s / static_cast<double>(Rb[i * in + i]);
    }
  }
  float* o = Ud + blk * 256 + k;
#pragma unroll
  for (int i = 0; i < 16; ++i) o[i * 16] = static_cast<float>(x[i]);
}

// x scaled by the power of two s, as its FP16 rounding and the FP16 rounding
// of the (exact FP32) remainder.
__device__ __forceinline__ void f16_split(float x, float s, __half& hi, __half& lo) {
  const float y = x * s;
  hi = __float2half_rn(y);
  lo = __float2half_rn(y - __half2float(hi));
}

// The B operand of a batch's split update GEMMs: for each part p of the batch
// (rows [r0 + kGB p, r0 + kGB (p + 1)) of R) and columns [c0, c0 + m), R scaled
// by s_R = gs[1], as [R_hi; R_lo; R_hi] in FP16 at rows kCat p .. of Rcat (row
// stride ldr).  blockIdx.y is the row of R within the batch.  Columns left of
// a row's diagonal are copied too and never read.
__global__ void __launch_bounds__(256)
gptq_rsplit_kernel(const float* __restrict__ R, int64_t in, int64_t r0, int64_t c0, int64_t m,
                   const float* __restrict__ gs, __half* __restrict__ Rcat, int64_t ldr) {
  const int64_t part = blockIdx.y / kGB, rr = blockIdx.y % kGB;
  const float sr = gs[1];
  const float* src = R + (r0 + blockIdx.y) * in + c0;
  __half* dst = Rcat + (part * kCat + rr) * ldr;
  for (int64_t c = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; c < m;
       c += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    __half hi, lo;
    f16_split(src[c], sr, hi, lo);
    dst[c] = hi;
    dst[kGB * ldr + c] = lo;
    dst[2 * kGB * ldr + c] = hi;
  }
}

// One part [j0, j0 + nb) of a lazy batch of GPTQ's columns in the R form, two
// threads (a pair of adjacent lanes) per row, kR rows per CTA.  Per 16-column
// group at g0 the pair
//   * sums v = P[r, grp] + D[r, j0:g0] R[j0:g0, grp] (P holds the earlier
//     parts' sums, D the part's earlier groups, in shared memory), each lane
//     8 of the 16 columns, and swaps halves;
//   * forms the current weights w = W[r, grp] + v U_grp (both lanes);
//   * runs the local call on w, each lane half of the candidates
//     (local_sweep_f32_pair);
//   * quantizes each column at its turn -- exact E2M1 decision, D = W - q,
//     err = (w - q) R_jj -- and updates the group's later columns by
//     w_k -= err U_jk (both lanes, the same arithmetic);
// and each lane writes its 8 columns of D, scaled by s_D = gs[0], as
// [D_hi | D_hi | D_lo] in FP16 (kCat columns from Dcat, row stride ldd) for
// the split update GEMMs.  Every sum is taken in the order one lane alone
// would take it, so the bytes do not depend on the pairing.  p_zero: the
// part's sums are zero (the first part of the first batch) and P is not read.  Dynamic shared
// memory: R's blocks above the diagonal blocks (kRsFloats), the groups' U
// blocks (8 x 256), the rows' D (kR x kDs).
template <bool kWeighted, int kK, int kR>
__global__ void __launch_bounds__(2 * kR)
gptq_rblock_kernel(const uint16_t* __restrict__ W, int64_t ldw, const uint8_t* __restrict__ dead,
                   int64_t out, int64_t in, int64_t j0, int nb, const float* __restrict__ P,
                   const float* __restrict__ R, const float* __restrict__ Ud,
                   const float* __restrict__ h, const float* __restrict__ Sp, int lo, int hi,
                   uint8_t* __restrict__ codes, uint8_t* __restrict__ scales,
                   const float* __restrict__ gs, __half* __restrict__ Dcat, int64_t ldd,
                   bool p_zero) {
  constexpr int kT = 2 * kR;
  extern __shared__ __align__(16) float gsm[];
  __shared__ CandEntry tab[kTabSize];
  __shared__ float hb[kGB];
  __shared__ float rdiag[kGB];
  __shared__ uint8_t deadb[kGB];
  float* Rs = gsm;
  float* Us = gsm + kRsFloats;
  float* Ds = Us + (kGB / 16) * 256;
  fill_candidate_table(tab);
  const int t = threadIdx.x;
  const int ng = nb / 16;
  // group b's block: R[j0 + i][j0 + 16 b + k], i < 16 b, at Rs + 128 b (b - 1) + 16 i + k.
  // Every copy is a 16-byte cp.async (R's rows and Ud are 64-byte aligned:
  // in % 16 == 0, j0 % 128 == 0), all in flight before one wait.
  for (int b = 1; b < ng; ++b) {
    float* dst = Rs + 128 * b * (b - 1);
    for (int c = t; c < 64 * b; c += kT) {  // 16 b rows x 4 chunks
      const int i = c >> 2, q = c & 3;
      cp_async16(dst + 16 * i + 4 * q, R + (j0 + i) * in + j0 + 16 * b + 4 * q);
    }
  }
  for (int c = t; c < ng * 64; c += kT) cp_async16(Us + 4 * c, Ud + (j0 / 16) * 256 + 4 * c);
  cp_async_commit();
  for (int k = t; k < nb; k += kT) {
    rdiag[k] = R[(j0 + k) * in + j0 + k];
    deadb[k] = dead[j0 + k];
    if (kWeighted) hb[k] = h[j0 + k];
  }
  cp_async_wait<0>();
  __syncthreads();
  const int lr = t >> 1, half = t & 1;
  const int64_t r = static_cast<int64_t>(blockIdx.x) * kR + lr;
  if (r >= out) return;  // both lanes of a pair, after the kernel's only barrier
  const unsigned pm = __activemask();  // whole pairs
  const ScaleConsts sc = scale_consts(*Sp);
  const int K = hi - lo + 1;
  float* ds = Ds + lr * kDs;
  const float* prow = P + r * in + j0 + 8 * half;
  const uint16_t* wrow = W + r * ldw + j0;
  __half* dcat = Dcat + r * ldd + 8 * half;
  const float sd = gs[0];
  const int64_t G = in / 16;
  // A group's P (this lane's 8 floats) and W (16 bf16, as 8 pairs, two 16-byte
  // loads: W is 16-byte aligned and ldw % 8 == 0) are loaded one group ahead,
  // so their latency hides behind the previous group's column loop.
  float4 pn[2];
  uint32_t wn[8];
  auto load_group = [&](int g) {
#pragma unroll
    for (int q = 0; q < 2; ++q)
      pn[q] = p_zero ? make_float4(0.0f, 0.0f, 0.0f, 0.0f)
                     : reinterpret_cast<const float4*>(prow + 16 * g)[q];
    const uint4 a = reinterpret_cast<const uint4*>(wrow + 16 * g)[0];
    const uint4 b = reinterpret_cast<const uint4*>(wrow + 16 * g)[1];
    wn[0] = a.x; wn[1] = a.y; wn[2] = a.z; wn[3] = a.w;
    wn[4] = b.x; wn[5] = b.y; wn[6] = b.z; wn[7] = b.w;
  };
  load_group(0);
  for (int g = 0; g < ng; ++g) {
    f32x2_t v2[4];  // this lane's 8 columns, 8 * half .. 8 * half + 7
    uint32_t wc[8];
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      v2[2 * q] = f2_pack(pn[q].x, pn[q].y);
      v2[2 * q + 1] = f2_pack(pn[q].z, pn[q].w);
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) wc[i] = wn[i];
    const float* rs = Rs + 128 * g * (g - 1) + 8 * half;
    for (int i = 0; i < 16 * g; i += 4) {
      const float4 d4 = *reinterpret_cast<const float4*>(ds + i);
      const float dv[4] = {d4.x, d4.y, d4.z, d4.w};
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const f32x2_t d2 = f2_pack(dv[u], dv[u]);
        const float4* rr = reinterpret_cast<const float4*>(rs + (i + u) * 16);
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          const float4 x = rr[q];
          v2[2 * q] = f2_fma(d2, f2_pack(x.x, x.y), v2[2 * q]);
          v2[2 * q + 1] = f2_fma(d2, f2_pack(x.z, x.w), v2[2 * q + 1]);
        }
      }
    }
    float v[16], w[16];
    {
      float mine[8];
#pragma unroll
      for (int i = 0; i < 4; ++i) f2_unpack(v2[i], mine[2 * i], mine[2 * i + 1]);
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const float other = __shfl_xor_sync(pm, mine[k], 1);
        v[k] = half ? other : mine[k];
        v[8 + k] = half ? mine[k] : other;
      }
    }
    // the group's original weights (dead columns zero), kept as bf16 pairs
    auto w0 = [&](int j) {
      const float wj = (j & 1) ? bf16_hi(wc[j >> 1]) : bf16_lo(wc[j >> 1]);
      return deadb[16 * g + j] ? 0.0f : wj;
    };
#pragma unroll
    for (int j = 0; j < 16; ++j) w[j] = w0(j);
    const float* ug = Us + 256 * g;
    // row i of the group's U block, columns 4 * (i / 4) .. 15, as float4 loads
    auto urow = [&](int i, float (&u)[16]) {
#pragma unroll
      for (int q = i / 4; q < 4; ++q) {
        const float4 x = reinterpret_cast<const float4*>(ug + i * 16)[q];
        u[4 * q] = x.x;
        u[4 * q + 1] = x.y;
        u[4 * q + 2] = x.z;
        u[4 * q + 3] = x.w;
      }
    };
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      float u[16];
      urow(i, u);
#pragma unroll
      for (int k = i; k < 16; ++k) w[k] = fmaf(v[i], u[k], w[k]);
    }
    // w waits in the row's D slots of this group (written only after the
    // column loop) while the sweep runs, which frees 16 registers there;
    // each lane parks its half, both read all 16
    float* wpark = ds + 16 * g;
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      const float4 lo4 = make_float4(w[4 * q], w[4 * q + 1], w[4 * q + 2], w[4 * q + 3]);
      const float4 hi4 = make_float4(w[8 + 4 * q], w[9 + 4 * q], w[10 + 4 * q], w[11 + 4 * q]);
      reinterpret_cast<float4*>(wpark + 8 * half)[q] = half ? hi4 : lo4;
    }
    __syncwarp(pm);
    const int code = local_sweep_f32_pair<kWeighted, kK>(
        wpark, kWeighted ? hb + 16 * g : nullptr, sc, tab, lo, K, half, pm);
    if (g + 1 < ng) load_group(g + 1);  // in flight during the column loop
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float4 x = reinterpret_cast<const float4*>(wpark)[q];
      w[4 * q] = x.x;
      w[4 * q + 1] = x.y;
      w[4 * q + 2] = x.z;
      w[4 * q + 3] = x.w;
    }
    uint32_t packed[2] = {0u, 0u};
    float dl[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      float q;
      packed[j >> 3] |= quantize_one(w[j], code, sc, tab, q) << (4 * (j & 7));
      dl[j] = w0(j) - q;
      const float err = (w[j] - q) * rdiag[16 * g + j];
      float u[16];
      urow(j, u);
#pragma unroll
      for (int k = j + 1; k < 16; ++k) w[k] = fmaf(-err, u[k], w[k]);
    }
    __syncwarp(pm);  // both lanes have read the parked w before D overwrites it
    float dh[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) dh[k] = half ? dl[8 + k] : dl[k];
#pragma unroll
    for (int q = 0; q < 2; ++q)
      *reinterpret_cast<float4*>(ds + 16 * g + 8 * half + 4 * q) =
          make_float4(dh[4 * q], dh[4 * q + 1], dh[4 * q + 2], dh[4 * q + 3]);
    uint32_t hw[4], lw[4];  // FP16 pairs, element 2i in the low half
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      __half h0, l0, h1, l1;
      f16_split(dh[2 * i], sd, h0, l0);
      f16_split(dh[2 * i + 1], sd, h1, l1);
      hw[i] = static_cast<uint32_t>(__half_as_ushort(h0)) |
              (static_cast<uint32_t>(__half_as_ushort(h1)) << 16);
      lw[i] = static_cast<uint32_t>(__half_as_ushort(l0)) |
              (static_cast<uint32_t>(__half_as_ushort(l1)) << 16);
    }
    const uint4 hv = make_uint4(hw[0], hw[1], hw[2], hw[3]);
    const uint4 lv = make_uint4(lw[0], lw[1], lw[2], lw[3]);
    *reinterpret_cast<uint4*>(dcat + 16 * g) = hv;
    *reinterpret_cast<uint4*>(dcat + kGB + 16 * g) = hv;
    *reinterpret_cast<uint4*>(dcat + 2 * kGB + 16 * g) = lv;
    if (half == 0) {
      const int64_t gg = j0 / 16 + g;
      *reinterpret_cast<uint2*>(codes + r * (G * 8) + gg * 8) = make_uint2(packed[0], packed[1]);
      scales[r * G + gg] = static_cast<uint8_t>(code);
    }
    __syncwarp(pm);  // the next group reads the partner's D
  }
}

// ------------------------------------------------------- library handles

struct Handles {
  cublasHandle_t blas = nullptr;
  cusolverDnHandle_t solver = nullptr;
};

std::mutex g_handles_mutex;
Handles g_handles[128];

// The calling thread's device's handles (created on first use).
bool handles_for_current_device(Handles** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 128) {
    cudaGetLastError();
    return false;
  }
  Handles& h = g_handles[dev];
  if (h.blas == nullptr && cublasCreate(&h.blas) != CUBLAS_STATUS_SUCCESS) {
    h.blas = nullptr;
    return false;
  }
  if (h.solver == nullptr && cusolverDnCreate(&h.solver) != CUSOLVER_STATUS_SUCCESS) {
    h.solver = nullptr;
    return false;
  }
  *out = &h;
  return true;
}

// Opt-in phase timing: CUDA event pairs recorded on the call's stream around
// its phases, summed per phase when read.  Process-wide, guarded by the
// handles' mutex; events are created on the device of the first timed call,
// and calls on another device are not timed.
struct PhaseTimer {
  bool on = false;
  int device = -1;
  struct Pair {
    cudaEvent_t a = nullptr, b = nullptr;
    int phase = 0;
  };
  std::vector<Pair> pairs;
  size_t used = 0;
  bool overflow = false;
};
PhaseTimer g_timer;
constexpr size_t kTimerPairs = 8192;

// Starts interval `phase` on `s`; returns its index, or -1 when not timing.
int timer_begin(int phase, cudaStream_t s) {
  PhaseTimer& T = g_timer;
  if (!T.on) return -1;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev != T.device) return -1;
  if (T.used == T.pairs.size()) {
    if (T.pairs.size() >= kTimerPairs) {
      T.overflow = true;
      return -1;
    }
    PhaseTimer::Pair p;
    if (cudaEventCreate(&p.a) != cudaSuccess || cudaEventCreate(&p.b) != cudaSuccess) {
      cudaGetLastError();
      T.overflow = true;
      return -1;
    }
    T.pairs.push_back(p);
  }
  PhaseTimer::Pair& p = T.pairs[T.used];
  p.phase = phase;
  if (cudaEventRecord(p.a, s) != cudaSuccess) {
    cudaGetLastError();
    return -1;
  }
  return static_cast<int>(T.used++);
}

void timer_end(int idx, cudaStream_t s) {
  if (idx < 0) return;
  if (cudaEventRecord(g_timer.pairs[idx].b, s) != cudaSuccess) cudaGetLastError();
}

struct GptqLayout {
  size_t h_ws = 0, s_ws = 0, H = 0, P = 0, Dcat = 0, Rcat = 0, gs = 0, Ud = 0, dead = 0,
         info = 0, lapack = 0, blas = 0;
  size_t bytes = 0;
  int lwork = 0;
  LanePlan dplan, gplan;
};

constexpr size_t kBlasWorkspace = 32u << 20;

bool gptq_layout(int64_t out, int64_t in, int64_t tokens, int sms, Handles* hd, GptqLayout* L) {
  L->dplan = diag_hessian_plan(tokens, in, sms);
  L->gplan = global_scale_plan(out, in, sms);
  int lw = 0;
  if (cusolverDnSpotrf_bufferSize(hd->solver, CUBLAS_FILL_MODE_LOWER, static_cast<int>(in),
                                  nullptr, static_cast<int>(in), &lw) != CUSOLVER_STATUS_SUCCESS)
    return false;
  L->lwork = lw;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off = al256(off + std::max<size_t>(bytes, 4));
    return o;
  };
  const size_t n = static_cast<size_t>(in), o = static_cast<size_t>(out);
  L->h_ws = take(diag_hessian_workspace_bytes(L->dplan, in));
  L->s_ws = take(global_scale_workspace_bytes(L->gplan));
  L->H = take(n * n * sizeof(float));
  L->P = take(o * n * sizeof(float));
  L->Dcat = take(o * kCat * kSub * sizeof(__half));
  L->Rcat = take(static_cast<size_t>(kCat) * kSub * n * sizeof(__half));
  L->gs = take(5 * sizeof(float));
  L->Ud = take(n * 16 * sizeof(float));
  L->dead = take(n);
  L->info = take(sizeof(int));
  L->lapack = take(static_cast<size_t>(lw) * sizeof(float));
  L->blas = take(kBlasWorkspace);
  L->bytes = off;
  return true;
}

// Rows per CTA of the batch kernel (two threads each): 208 -- one CTA per SM,
// 416 threads, so that a 28672-row matrix fits in one wave of 138 CTAs --
// when that keeps at least two thirds of the SMs busy, else 32.
constexpr size_t rblock_smem(int rows) {
  return (static_cast<size_t>(kRsFloats) + (kGB / 16) * 256 + static_cast<size_t>(rows) * kDs) *
         sizeof(float);
}

template <bool kW, int kKK, int kR>
cudaError_t launch_rblock_t(const uint16_t* W, int64_t ldw, const uint8_t* dead, int64_t out,
                            int64_t in, int64_t j0, int nb, const float* P, const float* R,
                            const float* Ud, const float* h, const float* S, int lo, int hi,
                            uint8_t* codes, uint8_t* scales, const float* gs, __half* Dcat,
                            int64_t ldd, bool p_zero, cudaStream_t s) {
  constexpr size_t smem = rblock_smem(kR);
  static const cudaError_t attr = cudaFuncSetAttribute(
      reinterpret_cast<const void*>(&gptq_rblock_kernel<kW, kKK, kR>),
      cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (attr != cudaSuccess) return attr;
  const unsigned blocks = static_cast<unsigned>((out + kR - 1) / kR);
  gptq_rblock_kernel<kW, kKK, kR><<<blocks, 2 * kR, smem, s>>>(
      W, ldw, dead, out, in, j0, nb, P, R, Ud, h, S, lo, hi, codes, scales, gs, Dcat, ldd, p_zero);
  return cudaGetLastError();
}

template <bool kW, int kKK>
cudaError_t launch_rblock(const uint16_t* W, int64_t ldw, const uint8_t* dead, int64_t out,
                          int64_t in, int64_t j0, int nb, const float* P, const float* R,
                          const float* Ud, const float* h, const float* S, int lo, int hi,
                          uint8_t* codes, uint8_t* scales, const float* gs, __half* Dcat,
                          int64_t ldd, bool p_zero, int sms, cudaStream_t s) {
  if (3 * ((out + 207) / 208) >= 2 * static_cast<int64_t>(sms))
    return launch_rblock_t<kW, kKK, 208>(W, ldw, dead, out, in, j0, nb, P, R, Ud, h, S, lo, hi,
                                         codes, scales, gs, Dcat, ldd, p_zero, s);
  return launch_rblock_t<kW, kKK, 32>(W, ldw, dead, out, in, j0, nb, P, R, Ud, h, S, lo, hi, codes,
                                      scales, gs, Dcat, ldd, p_zero, s);
}

}  // namespace

cudaError_t launch_sweep_f32(const float* W, int64_t out, int64_t in, int64_t ldw, const float* h,
                             const float* S, int lo, int hi, uint8_t* codes, uint8_t* scales,
                             int num_sms, cudaStream_t stream) {
  const int64_t G = in / 16;
  if (out == 0 || G == 0) return cudaSuccess;
  const int K = hi - lo + 1;
  int64_t blocks = (out * G + 127) / 128;
  const int64_t cap = static_cast<int64_t>(num_sms) * 16;
  if (blocks > cap) blocks = cap;
  const unsigned nbk = static_cast<unsigned>(blocks);
  if (h) {
    if (K == 16) sweep_f32_kernel<true, 16><<<nbk, 128, 0, stream>>>(W, out, G, ldw, h, S, lo, hi, codes, scales);
    else sweep_f32_kernel<true, 0><<<nbk, 128, 0, stream>>>(W, out, G, ldw, h, S, lo, hi, codes, scales);
  } else {
    if (K == 16) sweep_f32_kernel<false, 16><<<nbk, 128, 0, stream>>>(W, out, G, ldw, h, S, lo, hi, codes, scales);
    else sweep_f32_kernel<false, 0><<<nbk, 128, 0, stream>>>(W, out, G, ldw, h, S, lo, hi, codes, scales);
  }
  return cudaGetLastError();
}

size_t gptq_workspace_bytes(int64_t out, int64_t in, int64_t tokens, int sms) {
  std::lock_guard<std::mutex> lock(g_handles_mutex);
  Handles* hd = nullptr;
  if (!handles_for_current_device(&hd)) return 0;
  GptqLayout L;
  if (!gptq_layout(out, in, tokens, sms, hd, &L)) return 0;
  return L.bytes;
}

// The whole GPTQ pass on `stream`; returns the first failing CUDA, cuBLAS or
// cuSOLVER status as a cudaError_t (library failures map to
// cudaErrorUnknown).
cudaError_t launch_gptq(const uint16_t* W, int64_t out, int64_t in, int64_t ldw, const uint16_t* X,
                        int64_t tokens, int64_t ldx, float q_max, int lo, int hi, float damp,
                        bool weighted, uint8_t* codes, uint8_t* scales, float* S, float* h,
                        int* status, void* workspace, size_t workspace_bytes, int sms,
                        cudaStream_t stream) {
  std::lock_guard<std::mutex> lock(g_handles_mutex);
  Handles* hd = nullptr;
  if (!handles_for_current_device(&hd)) return cudaErrorUnknown;
  GptqLayout L;
  if (!gptq_layout(out, in, tokens, sms, hd, &L)) return cudaErrorUnknown;
  if (workspace_bytes < L.bytes) return cudaErrorInvalidValue;
  char* ws = static_cast<char*>(workspace);
  float* H = reinterpret_cast<float*>(ws + L.H);
  float* P = reinterpret_cast<float*>(ws + L.P);
  __half* Dcat = reinterpret_cast<__half*>(ws + L.Dcat);
  __half* Rcat = reinterpret_cast<__half*>(ws + L.Rcat);
  float* gs = reinterpret_cast<float*>(ws + L.gs);
  float* Ud = reinterpret_cast<float*>(ws + L.Ud);
  uint8_t* dead = reinterpret_cast<uint8_t*>(ws + L.dead);
  int* info = reinterpret_cast<int*>(ws + L.info);
  float* lapack = reinterpret_cast<float*>(ws + L.lapack);
  cudaError_t e;
  auto blas_ok = [](cublasStatus_t s) { return s == CUBLAS_STATUS_SUCCESS; };
  auto lapack_ok = [](cusolverStatus_t s) { return s == CUSOLVER_STATUS_SUCCESS; };
  if (!blas_ok(cublasSetStream(hd->blas, stream)) ||
      !blas_ok(cublasSetWorkspace(hd->blas, ws + L.blas, kBlasWorkspace)) ||
      !lapack_ok(cusolverDnSetStream(hd->solver, stream)))
    return cudaErrorUnknown;
  // the compute types are given per call; the handle's math mode stays the default
  if (!blas_ok(cublasSetMathMode(hd->blas, CUBLAS_DEFAULT_MATH)) ||
      !blas_ok(cublasSetPointerMode(hd->blas, CUBLAS_POINTER_MODE_HOST)))
    return cudaErrorUnknown;
  // the update GEMMs take alpha and beta from device memory; host mode again
  // on every way out of this call
  struct PointerModeGuard {
    cublasHandle_t h;
    ~PointerModeGuard() { cublasSetPointerMode(h, CUBLAS_POINTER_MODE_HOST); }
  } pointer_mode_guard{hd->blas};
  // h and S with this library's kernels
  int tm = timer_begin(NVFP4_GPTQ_PHASE_REDUCTIONS, stream);
  if ((e = launch_diag_hessian(X, tokens, in, ldx, h, 0, reinterpret_cast<float*>(ws + L.h_ws),
                               L.dplan, stream)) != cudaSuccess)
    return e;
  if ((e = launch_global_scale(W, out, ldw, q_max, S, nullptr, status,
                               reinterpret_cast<uint32_t*>(ws + L.s_ws), L.gplan, stream)) !=
      cudaSuccess)
    return e;
  timer_end(tm, stream);
  tm = timer_begin(NVFP4_GPTQ_PHASE_GRAM, stream);
  // H = X^T X: X row-major [tokens, ldx] is column-major [ldx, tokens], so
  // H = X_cm X_cm^T, bf16 products exact, FP32 accumulation.  Only H's
  // column-major lower triangle is read later (the reflection keeps each
  // triangle in place and potrf reads the lower one), so for in >= 4096 H is
  // built from the 10 blocks (I, J), I >= J, of a 4 x 4 split -- 10/16 of the
  // products; the blocks above the diagonal are left unwritten.
  const float one = 1.0f, zero = 0.0f;
  if (tokens > 0) {
    const int nsplit = in >= 4096 ? 4 : 1;
    int64_t edge[5];
    for (int k = 0; k <= nsplit; ++k) edge[k] = (in * k / nsplit) / 16 * 16;
    edge[nsplit] = in;
    for (int bi = 0; bi < nsplit; ++bi)
      for (int bj = 0; bj <= bi; ++bj) {
        const int64_t i0 = edge[bi], j0 = edge[bj];
        if (!blas_ok(cublasGemmEx(hd->blas, CUBLAS_OP_N, CUBLAS_OP_T,
                                  static_cast<int>(edge[bi + 1] - i0),
                                  static_cast<int>(edge[bj + 1] - j0), static_cast<int>(tokens),
                                  &one, X + i0, CUDA_R_16BF, static_cast<int>(ldx), X + j0,
                                  CUDA_R_16BF, static_cast<int>(ldx), &zero, H + i0 + j0 * in,
                                  CUDA_R_32F, static_cast<int>(in), CUBLAS_COMPUTE_32F,
                                  CUBLAS_GEMM_DEFAULT)))
          return cudaErrorUnknown;
      }
  } else if ((e = cudaMemsetAsync(H, 0, static_cast<size_t>(in) * in * sizeof(float), stream)) !=
             cudaSuccess) {
    return e;
  }
  timer_end(tm, stream);
  tm = timer_begin(NVFP4_GPTQ_PHASE_FACTOR, stream);
  gptq_prep_kernel<<<1, 256, 0, stream>>>(H, in, damp, dead, S, q_max, gs);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  // R = J L' J row-major, L' the lower Cholesky factor of J H J (FP32)
  const int n = static_cast<int>(in);
  auto reflect = [&]() {
    const dim3 grid(static_cast<unsigned>(in / 16), static_cast<unsigned>(in / 16));
    antitranspose_kernel<<<grid, 256, 0, stream>>>(H, in);
    return cudaGetLastError();
  };
  if ((e = reflect()) != cudaSuccess) return e;
  if (!lapack_ok(cusolverDnSpotrf(hd->solver, CUBLAS_FILL_MODE_LOWER, n, H, n, lapack, L.lwork,
                                  info)))
    return cudaErrorUnknown;
  if ((e = reflect()) != cudaSuccess) return e;
  gptq_status_kernel<<<1, 1, 0, stream>>>(info, 1, status);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  const float* R = H;  // row-major R[j][k] for k >= j
  gptq_udiag_kernel<<<static_cast<unsigned>((in + 127) / 128), 128, 0, stream>>>(R, in, Ud);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  timer_end(tm, stream);
  const int K = hi - lo + 1;
  const uint8_t* dd = dead;
  const int64_t ldd = static_cast<int64_t>(kCat) * kSub;
  auto block_t = [&](int64_t c0, int nb, __half* dcat) {
    if (weighted)
      return K == 16 ? launch_rblock<true, 16>(W, ldw, dd, out, in, c0, nb, P, R, Ud, h, S, lo, hi, codes, scales, gs, dcat, ldd, c0 == 0, sms, stream)
                     : launch_rblock<true, 0>(W, ldw, dd, out, in, c0, nb, P, R, Ud, h, S, lo, hi, codes, scales, gs, dcat, ldd, c0 == 0, sms, stream);
    return K == 16 ? launch_rblock<false, 16>(W, ldw, dd, out, in, c0, nb, P, R, Ud, nullptr, S, lo, hi, codes, scales, gs, dcat, ldd, c0 == 0, sms, stream)
                   : launch_rblock<false, 0>(W, ldw, dd, out, in, c0, nb, P, R, Ud, nullptr, S, lo, hi, codes, scales, gs, dcat, ldd, c0 == 0, sms, stream);
  };
  auto block = [&](int64_t c0, int nb, __half* dcat) {
    const int t = timer_begin(NVFP4_GPTQ_PHASE_BATCH, stream);
    const cudaError_t r = block_t(c0, nb, dcat);
    timer_end(t, stream);
    return r;
  };
  // one split per batch: every full part's rows, columns [c0, in)
  auto split = [&](int64_t r0, int parts, int64_t c0) {
    const int t = timer_begin(NVFP4_GPTQ_PHASE_SPLIT, stream);
    const int64_t m = in - c0;
    const dim3 grid(static_cast<unsigned>(std::min<int64_t>((m + 255) / 256, 8)),
                    static_cast<unsigned>(kGB * parts));
    gptq_rsplit_kernel<<<grid, 256, 0, stream>>>(R, in, r0, c0, m, gs, Rcat, in);
    timer_end(t, stream);
    return cudaGetLastError();
  };
  // P[:, c0 : c0 + m] += Dcat[:, :k] Rcat[:k, :m], all row-major: in
  // column-major terms P^T (m x out) += Rcat^T (m x k) Dcat^T (k x out)
  // alpha = 1 / (s_D s_R) and beta are device scalars (gs[2]; gs[3] = 1, or
  // gs[4] = 0 where the GEMM writes its columns of P first: every update of
  // the first batch -- P is never cleared, and the first part reads none of it)
  auto update = [&](int64_t c0, int64_t m, int k, const __half* rcat, int64_t ldr, bool first) {
    const int t = timer_begin(NVFP4_GPTQ_PHASE_UPDATE, stream);
    const bool ok = blas_ok(cublasGemmEx(hd->blas, CUBLAS_OP_N, CUBLAS_OP_N, static_cast<int>(m),
                                static_cast<int>(out), k, gs + 2, rcat, CUDA_R_16F,
                                static_cast<int>(ldr), Dcat, CUDA_R_16F, static_cast<int>(ldd),
                                first ? gs + 4 : gs + 3, P + c0, CUDA_R_32F, n,
                                CUBLAS_COMPUTE_32F,
                                CUBLAS_GEMM_DEFAULT));
    timer_end(t, stream);
    return ok;
  };
  if (!blas_ok(cublasSetPointerMode(hd->blas, CUBLAS_POINTER_MODE_DEVICE)))
    return cudaErrorUnknown;
  constexpr int64_t kBatch = static_cast<int64_t>(kGB) * kSub;
  for (int64_t j0 = 0; j0 < in; j0 += kBatch) {
    const int64_t jend = std::min(j0 + kBatch, in);
    const int nsub = static_cast<int>((jend - j0 + kGB - 1) / kGB);
    // R's rows of the batch's full parts (only the last part can be narrower,
    // and its rows are never an operand), columns from the second part on
    const int64_t col0 = j0 + kGB;
    const int full = static_cast<int>((jend - j0) / kGB);
    if (col0 < in && full > 0 && (e = split(j0, full, col0)) != cudaSuccess) return e;
    for (int sb = 0; sb < nsub; ++sb) {
      const int64_t c0 = j0 + static_cast<int64_t>(kGB) * sb;
      const int nb = static_cast<int>(std::min<int64_t>(kGB, jend - c0));
      if ((e = block(c0, nb, Dcat + static_cast<int64_t>(kCat) * sb)) != cudaSuccess) return e;
      if (sb + 1 < nsub) {  // the next part takes the batch's parts so far
        const int64_t c1 = c0 + nb;  // nb == kGB: only a batch's last part can be narrower
        const int64_t m = std::min<int64_t>(kGB, jend - c1);
        if (!update(c1, m, kCat * (sb + 1), Rcat + (c1 - col0), in, j0 == 0))
          return cudaErrorUnknown;
      }
    }
    if (jend < in &&  // every later column takes the whole batch (all parts full)
        !update(jend, in - jend, kCat * nsub, Rcat + (jend - col0), in, j0 == 0))
      return cudaErrorUnknown;
  }
  return cudaSuccess;
}

void gptq_set_timing(bool on) {
  std::lock_guard<std::mutex> lock(g_handles_mutex);
  g_timer.on = on;
  g_timer.used = 0;
  g_timer.overflow = false;
  if (on && g_timer.device < 0 && cudaGetDevice(&g_timer.device) != cudaSuccess) {
    cudaGetLastError();
    g_timer.on = false;
  }
}

cudaError_t gptq_phase_times(float* ms, int n, bool* overflow) {
  std::lock_guard<std::mutex> lock(g_handles_mutex);
  for (int i = 0; i < n; ++i) ms[i] = 0.0f;
  *overflow = g_timer.overflow;
  for (size_t i = 0; i < g_timer.used; ++i) {
    const PhaseTimer::Pair& p = g_timer.pairs[i];
    cudaError_t e = cudaEventSynchronize(p.b);
    float t = 0.0f;
    if (e == cudaSuccess) e = cudaEventElapsedTime(&t, p.a, p.b);
    if (e != cudaSuccess) return e;
    if (p.phase >= 0 && p.phase < n) ms[p.phase] += t;
  }
  return cudaSuccess;
}

}  // namespace nvfp4
