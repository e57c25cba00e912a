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
//   * H = X^T X: one cuBLAS GEMM (bf16 in, FP32 accumulate; a plain GEMM);
//   * the dead-column rule and the damping: gptq_prep_kernel;
//   * U without forming H^-1: with J the order-reversing permutation, the
//     lower Cholesky factor L' of J H J gives H = R R^T with R = J L' J upper,
//     so H^-1 = (R^-1)^T R^-1 and U = R^-1 = J L'^-1 J.  cuSOLVER factors
//     (potrf) and inverts (trtri) in FP32 on the lower triangle; the
//     reflection of the n x n array about its anti-diagonal, done in place
//     before (J H J, H symmetric) and after, turns the column-major L'^-1
//     into U row-major: U[j][k] at j * in + k;
//   * GPTQ's lazy batches of 128 columns: gptq_block_kernel runs the columns of
//     one batch for 64 rows per CTA -- local call, quantization, in-batch
//     propagation -- with the batch's triangle of U and the rows' weights in
//     shared memory, and writes the batch's errors; one FP32 GEMM (cuBLAS)
//     then applies them to every later column: W[:, >] -= Err U[batch, >].
// Rows are independent in GPTQ (U is shared), so the batch kernel needs no
// communication between rows.  FP32 throughout on the device: its results
// drift from the FP64 oracle's after a quantization decision flips, which a
// row then carries through its later columns.
#include <cublas_v2.h>
#include <cusolverDn.h>

#include <mutex>
#include <vector>

#include "nvfp4_kernels.cuh"
#include "sweep_core.cuh"

namespace nvfp4 {

namespace {

constexpr int kGB = 128;  // columns per lazy batch
constexpr int kGT = 64;   // rows (threads) per CTA of the batch kernel

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
  float Lf[16];
  uint32_t kbest = 0xFFFFFFFFu, ksec = 0xFFFFFFFFu;
  auto cand = [&](int i) {
    const float Li = fast_candidate_loss<kWeighted>(y2, h2, ce[i]);
    Lf[i] = Li;
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
      if (Lf[i] > T) continue;
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
__global__ void __launch_bounds__(256)
gptq_prep_kernel(float* __restrict__ H, int64_t in, float damp, uint8_t* __restrict__ dead) {
  __shared__ double part[256];
  double s = 0.0;
  for (int64_t j = threadIdx.x; j < in; j += blockDim.x) {
    float d = H[j * in + j];
    dead[j] = d == 0.0f ? 1 : 0;
    if (d == 0.0f) {
      d = 1.0f;
      H[j * in + j] = 1.0f;
    }
    s += static_cast<double>(d);
  }
  part[threadIdx.x] = s;
  __syncthreads();
  for (int o = 128; o > 0; o >>= 1) {
    if (threadIdx.x < o) part[threadIdx.x] += part[threadIdx.x + o];
    __syncthreads();
  }
  const float lam = static_cast<float>(static_cast<double>(damp) * part[0] / static_cast<double>(in));
  for (int64_t j = threadIdx.x; j < in; j += blockDim.x) H[j * in + j] += lam;
}

// FP32 working copy of W (row stride in), dead columns zero.
__global__ void __launch_bounds__(256)
gptq_wcopy_kernel(const uint16_t* __restrict__ W, int64_t out, int64_t in, int64_t ldw,
                  const uint8_t* __restrict__ dead, float* __restrict__ Wf) {
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < out * in;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t r = i / in, j = i - r * in;
    Wf[i] = dead[j] ? 0.0f : bf16_lo(W[r * ldw + j]);
  }
}

// In place: a[r][c] <-> a[n-1-c][n-1-r] (reflection about the anti-diagonal),
// one thread per pair r + c < n - 1.
__global__ void __launch_bounds__(256)
antitranspose_kernel(float* __restrict__ a, int64_t n) {
  const int64_t total = n * n;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t r = i / n, c = i - r * n;
    if (r + c >= n - 1) continue;
    const int64_t o = (n - 1 - c) * n + (n - 1 - r);
    const float t = a[i];
    a[i] = a[o];
    a[o] = t;
  }
}

// A failed Cholesky or inverse (devInfo != 0: the damped Hessian is not
// positive definite in FP32) is reported through the status word.
__global__ void gptq_status_kernel(const int* __restrict__ info, int n, int* status) {
  int bad = 0;
  for (int i = 0; i < n; ++i) bad |= info[i] != 0;
  if (bad && status) *status = -9;  // NVFP4_ERR_NUMERIC
}

// One lazy batch [j0, j0 + nb) of GPTQ's columns for kGT rows per CTA.
// Dynamic shared memory: U's batch triangle [kGB][kGB] then the rows'
// weights [kGT][kGB + 1].
template <bool kWeighted, int kK>
__global__ void __launch_bounds__(kGT)
gptq_block_kernel(const float* __restrict__ Wf, int64_t out, int64_t in, int64_t j0, int nb,
                  const float* __restrict__ U, const float* __restrict__ h,
                  const float* __restrict__ Sp, int lo, int hi, uint8_t* __restrict__ codes,
                  uint8_t* __restrict__ scales, float* __restrict__ Err) {
  extern __shared__ __align__(16) float gsm[];
  __shared__ CandEntry tab[kTabSize];
  __shared__ float hb[kGB];
  float* Ub = gsm;
  float* wr = gsm + kGB * kGB;
  fill_candidate_table(tab);
  const int t = threadIdx.x;
  const int64_t r0 = static_cast<int64_t>(blockIdx.x) * kGT;
  for (int idx = t; idx < nb * nb; idx += kGT) {
    const int i = idx / nb, k = idx - i * nb;
    Ub[i * kGB + k] = k >= i ? U[(j0 + i) * in + j0 + k] : 0.0f;
  }
  for (int idx = t; idx < kGT * nb; idx += kGT) {
    const int rr = idx / nb, k = idx - rr * nb;
    const int64_t r = r0 + rr;
    wr[rr * (kGB + 1) + k] = r < out ? Wf[r * in + j0 + k] : 0.0f;
  }
  if (kWeighted)
    for (int k = t; k < nb; k += kGT) hb[k] = h[j0 + k];
  __syncthreads();
  const int64_t r = r0 + t;
  if (r >= out) return;  // after the kernel's only barrier
  const ScaleConsts sc = scale_consts(*Sp);
  const int K = hi - lo + 1;
  float* w = wr + t * (kGB + 1);
  const int64_t G = in / 16;
  for (int g = 0; g < nb / 16; ++g) {
    float wg[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) wg[j] = w[16 * g + j];
    const int code = local_sweep_f32<kWeighted, kK>(wg, kWeighted ? hb + 16 * g : nullptr, sc,
                                                    tab, lo, K);
    uint32_t packed[2] = {0u, 0u};
    for (int i = 0; i < 16; ++i) {
      const int j = 16 * g + i;
      const float wv = w[j];
      float q;
      packed[i >> 3] |= quantize_one(wv, code, sc, tab, q) << (4 * (i & 7));
      const float err = (wv - q) / Ub[j * kGB + j];
      Err[r * kGB + j] = err;
      for (int k = j + 1; k < nb; ++k) w[k] = fmaf(-err, Ub[j * kGB + k], w[k]);
    }
    const int64_t gg = j0 / 16 + g;
    *reinterpret_cast<uint2*>(codes + r * (G * 8) + gg * 8) = make_uint2(packed[0], packed[1]);
    scales[r * G + gg] = static_cast<uint8_t>(code);
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

struct GptqLayout {
  size_t h_ws = 0, s_ws = 0, H = 0, Wf = 0, Err = 0, dead = 0, info = 0, lapack = 0, blas = 0;
  size_t bytes = 0;
  size_t lapack_bytes = 0, host_bytes = 0;
  int lwork = 0;
  LanePlan dplan, gplan;
};

constexpr size_t kBlasWorkspace = 32u << 20;

bool gptq_layout(int64_t out, int64_t in, int64_t tokens, int sms, Handles* hd, GptqLayout* L) {
  L->dplan = diag_hessian_plan(tokens, in, sms);
  L->gplan = global_scale_plan(out, in, sms);
  int lw1 = 0;
  if (cusolverDnSpotrf_bufferSize(hd->solver, CUBLAS_FILL_MODE_LOWER, static_cast<int>(in),
                                  nullptr, static_cast<int>(in), &lw1) != CUSOLVER_STATUS_SUCCESS)
    return false;
  size_t dev_b = 0, host_b = 0;
  if (cusolverDnXtrtri_bufferSize(hd->solver, CUBLAS_FILL_MODE_LOWER, CUBLAS_DIAG_NON_UNIT, in,
                                  CUDA_R_32F, nullptr, in, &dev_b, &host_b) !=
      CUSOLVER_STATUS_SUCCESS)
    return false;
  L->lwork = lw1;
  L->lapack_bytes = std::max(static_cast<size_t>(lw1) * sizeof(float), dev_b);
  L->host_bytes = host_b;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off = al256(off + std::max<size_t>(bytes, 4));
    return o;
  };
  L->h_ws = take(diag_hessian_workspace_bytes(L->dplan, in));
  L->s_ws = take(global_scale_workspace_bytes(L->gplan));
  L->H = take(static_cast<size_t>(in) * static_cast<size_t>(in) * sizeof(float));
  L->Wf = take(static_cast<size_t>(out) * static_cast<size_t>(in) * sizeof(float));
  L->Err = take(static_cast<size_t>(out) * kGB * sizeof(float));
  L->dead = take(static_cast<size_t>(in));
  L->info = take(3 * sizeof(int));
  L->lapack = take(L->lapack_bytes);
  L->blas = take(kBlasWorkspace);
  L->bytes = off;
  return true;
}

template <bool kW, int kKK>
cudaError_t launch_block(const float* Wf, int64_t out, int64_t in, int64_t j0, int nb,
                         const float* U, const float* h, const float* S, int lo, int hi,
                         uint8_t* codes, uint8_t* scales, float* Err, cudaStream_t s) {
  constexpr size_t smem = (static_cast<size_t>(kGB) * kGB + static_cast<size_t>(kGT) * (kGB + 1)) *
                          sizeof(float);
  static const cudaError_t attr = cudaFuncSetAttribute(
      reinterpret_cast<const void*>(&gptq_block_kernel<kW, kKK>),
      cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (attr != cudaSuccess) return attr;
  const unsigned blocks = static_cast<unsigned>((out + kGT - 1) / kGT);
  gptq_block_kernel<kW, kKK><<<blocks, kGT, smem, s>>>(Wf, out, in, j0, nb, U, h, S, lo, hi, codes,
                                                       scales, Err);
  return cudaGetLastError();
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
  float* Wf = reinterpret_cast<float*>(ws + L.Wf);
  float* Err = reinterpret_cast<float*>(ws + L.Err);
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
  // plain FP32 GEMMs (no TF32 or emulated paths: the same arithmetic whichever
  // cuBLAS build the process has loaded)
  if (!blas_ok(cublasSetMathMode(hd->blas, CUBLAS_DEFAULT_MATH))) return cudaErrorUnknown;
  // h and S with this library's kernels
  if ((e = launch_diag_hessian(X, tokens, in, ldx, h, 0, reinterpret_cast<float*>(ws + L.h_ws),
                               L.dplan, stream)) != cudaSuccess)
    return e;
  if ((e = launch_global_scale(W, out, ldw, q_max, S, nullptr, status,
                               reinterpret_cast<uint32_t*>(ws + L.s_ws), L.gplan, stream)) !=
      cudaSuccess)
    return e;
  // H = X^T X: X row-major [tokens, ldx] is column-major [ldx, tokens], so
  // H = X_cm X_cm^T, bf16 products exact, FP32 accumulation
  const float one = 1.0f, zero = 0.0f;
  if (tokens > 0) {
    if (!blas_ok(cublasGemmEx(hd->blas, CUBLAS_OP_N, CUBLAS_OP_T, static_cast<int>(in),
                              static_cast<int>(in), static_cast<int>(tokens), &one, X, CUDA_R_16BF,
                              static_cast<int>(ldx), X, CUDA_R_16BF, static_cast<int>(ldx), &zero,
                              H, CUDA_R_32F, static_cast<int>(in), CUBLAS_COMPUTE_32F,
                              CUBLAS_GEMM_DEFAULT)))
      return cudaErrorUnknown;
  } else if ((e = cudaMemsetAsync(H, 0, static_cast<size_t>(in) * in * sizeof(float), stream)) !=
             cudaSuccess) {
    return e;
  }
  gptq_prep_kernel<<<1, 256, 0, stream>>>(H, in, damp, dead);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  {
    const int64_t n = out * in;
    int64_t blocks = (n + 255) / 256;
    if (blocks > static_cast<int64_t>(sms) * 16) blocks = static_cast<int64_t>(sms) * 16;
    gptq_wcopy_kernel<<<static_cast<unsigned>(blocks), 256, 0, stream>>>(W, out, in, ldw, dead, Wf);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  // U = J L'^-1 J, L' the lower Cholesky factor of J H J (FP32)
  const int n = static_cast<int>(in);
  auto reflect = [&]() {
    int64_t blocks = (in * in + 255) / 256;
    if (blocks > static_cast<int64_t>(sms) * 16) blocks = static_cast<int64_t>(sms) * 16;
    antitranspose_kernel<<<static_cast<unsigned>(blocks), 256, 0, stream>>>(H, in);
    return cudaGetLastError();
  };
  std::vector<char> host_scratch(L.host_bytes);
  if ((e = reflect()) != cudaSuccess) return e;
  if (!lapack_ok(cusolverDnSpotrf(hd->solver, CUBLAS_FILL_MODE_LOWER, n, H, n, lapack, L.lwork,
                                  info)) ||
      !lapack_ok(cusolverDnXtrtri(hd->solver, CUBLAS_FILL_MODE_LOWER, CUBLAS_DIAG_NON_UNIT, in,
                                  CUDA_R_32F, H, in, lapack, L.lapack_bytes,
                                  host_scratch.empty() ? nullptr : host_scratch.data(),
                                  L.host_bytes, info + 1)))
    return cudaErrorUnknown;
  if ((e = reflect()) != cudaSuccess) return e;
  gptq_status_kernel<<<1, 1, 0, stream>>>(info, 2, status);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  const float* U = H;  // row-major U[j][k] for k >= j (the reflected L'^-1)
  const int K = hi - lo + 1;
  const float minus_one = -1.0f;
  for (int64_t j0 = 0; j0 < in; j0 += kGB) {
    const int nb = static_cast<int>(std::min<int64_t>(kGB, in - j0));
    if (weighted)
      e = K == 16 ? launch_block<true, 16>(Wf, out, in, j0, nb, U, h, S, lo, hi, codes, scales, Err, stream)
                  : launch_block<true, 0>(Wf, out, in, j0, nb, U, h, S, lo, hi, codes, scales, Err, stream);
    else
      e = K == 16 ? launch_block<false, 16>(Wf, out, in, j0, nb, U, nullptr, S, lo, hi, codes, scales, Err, stream)
                  : launch_block<false, 0>(Wf, out, in, j0, nb, U, nullptr, S, lo, hi, codes, scales, Err, stream);
    if (e != cudaSuccess) return e;
    const int64_t j1 = j0 + nb;
    if (j1 < in) {
      // W[:, j1:] -= Err[:, :nb] U[j0:j1, j1:], all row-major: in column-major
      // terms C^T (n2 x out) -= U_blk^T (n2 x nb) Err^T (nb x out)
      if (!blas_ok(cublasSgemm(hd->blas, CUBLAS_OP_N, CUBLAS_OP_N, static_cast<int>(in - j1),
                               static_cast<int>(out), nb, &minus_one, U + j0 * in + j1, n, Err,
                               kGB, &one, Wf + j1, n)))
        return cudaErrorUnknown;
    }
  }
  return cudaSuccess;
}

}  // namespace nvfp4
