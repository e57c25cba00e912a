// diag_hessian.cu -- h_j = sum_t x_tj^2 over calibration activations.
//
// H-Scale summary, sec. B "Implementation": the diagonal weights come from
// diag(X^T X) of the calibration activations (sec. 3 "Hessian-guided
// objective": the diagonal keeps per-channel activation energy and drops the
// cross-channel terms).
//
// HBM-bound: 2 bytes read per element, one FFMA.  Layout of the work:
//   * a "vector" is 8 consecutive bf16 of one row (16 B, one LDG.128);
//   * thread lanes form a grid of R row-lanes x VL vector-lanes; lane (r, vl)
//     owns vector columns vl, vl+VL, ... and rows r, r+R, ..., so adjacent
//     threads read adjacent 16-byte vectors of the same row (coalesced);
//   * U rows are loaded before any is consumed (U x 16 B in flight per thread);
//   * each lane sums a run of U squares in FP32, adds the run into an FP32
//     per-lane accumulator, and writes it to partials[r, col];
//   * a second kernel adds the R partials of each column in FP64 in a fixed
//     order (deterministic) and rounds once to FP32.
#include "nvfp4_kernels.cuh"

namespace nvfp4 {

template <int U>
__global__ void __launch_bounds__(256)
diag_hessian_partial_kernel(const uint16_t* __restrict__ X, int64_t T, int64_t in, int64_t ldx,
                            int64_t V, int64_t VL, int64_t R, float* __restrict__ P) {
  const int64_t tid = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (tid >= R * VL) return;
  const int64_t r = tid / VL;
  const int64_t vl = tid - r * VL;
  for (int64_t v = vl; v < V; v += VL) {
    float acc[8];
#pragma unroll
    for (int c = 0; c < 8; ++c) acc[c] = 0.0f;
    const uint16_t* col = X + v * 8;
    int64_t t = r;
    for (; t + (U - 1) * R < T; t += U * R) {
      uint4 q[U];
#pragma unroll
      for (int u = 0; u < U; ++u) q[u] = ld_stream_v4(col + (t + u * R) * ldx);
      float s[8];
#pragma unroll
      for (int c = 0; c < 8; ++c) s[c] = 0.0f;
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const uint32_t w[4] = {q[u].x, q[u].y, q[u].z, q[u].w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const float a = bf16_lo(w[k]), b = bf16_hi(w[k]);
          s[2 * k] = fmaf(a, a, s[2 * k]);
          s[2 * k + 1] = fmaf(b, b, s[2 * k + 1]);
        }
      }
#pragma unroll
      for (int c = 0; c < 8; ++c) acc[c] += s[c];
    }
    for (; t < T; t += R) {
      const uint4 q = ld_stream_v4(col + t * ldx);
      const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float a = bf16_lo(w[k]), b = bf16_hi(w[k]);
        acc[2 * k] = fmaf(a, a, acc[2 * k]);
        acc[2 * k + 1] = fmaf(b, b, acc[2 * k + 1]);
      }
    }
    float4* dst = reinterpret_cast<float4*>(P + r * in + v * 8);
    dst[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
    dst[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
  }
}

__global__ void __launch_bounds__(256)
diag_hessian_finalize_kernel(const float* __restrict__ P, int64_t R, int64_t in, float* h,
                             int accumulate) {
  const int64_t j = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (j >= in) return;
  double s0 = 0.0, s1 = 0.0, s2 = 0.0, s3 = 0.0;
  int64_t r = 0;
  for (; r + 3 < R; r += 4) {
    s0 += P[(r + 0) * in + j];
    s1 += P[(r + 1) * in + j];
    s2 += P[(r + 2) * in + j];
    s3 += P[(r + 3) * in + j];
  }
  for (; r < R; ++r) s0 += P[r * in + j];
  const double base = accumulate ? static_cast<double>(h[j]) : 0.0;
  h[j] = static_cast<float>(base + ((s0 + s1) + (s2 + s3)));
}

// Lane plan shared by the host-side workspace query and the launch.
LanePlan diag_hessian_plan(int64_t tokens, int64_t in, int num_sms) {
  LanePlan p;
  p.V = in / 8;
  static const int ctas = resident_ctas(
      reinterpret_cast<const void*>(&diag_hessian_partial_kernel<8>), 256);
  const int64_t nt = static_cast<int64_t>(num_sms) * ctas * 256;
  p.VL = p.V < nt ? (p.V > 0 ? p.V : 1) : nt;
  int64_t R = nt / p.VL;
  if (R > tokens) R = tokens;
  if (R < 1) R = 1;
  p.R = R;
  p.threads = p.R * p.VL;
  return p;
}

size_t diag_hessian_workspace_bytes(const LanePlan& p, int64_t in) {
  return static_cast<size_t>(p.R) * static_cast<size_t>(in) * sizeof(float);
}

cudaError_t launch_diag_hessian(const uint16_t* X, int64_t T, int64_t in, int64_t ldx, float* h,
                                int accumulate, float* partials, const LanePlan& p,
                                cudaStream_t stream) {
  const int64_t blocks = (p.threads + 255) / 256;
  if (T > 0) {
    diag_hessian_partial_kernel<8><<<static_cast<unsigned>(blocks), 256, 0, stream>>>(
        X, T, in, ldx, p.V, p.VL, p.R, partials);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  const int64_t rows = T > 0 ? p.R : 0;  // no tokens: finalize adds nothing
  diag_hessian_finalize_kernel<<<static_cast<unsigned>((in + 255) / 256), 256, 0, stream>>>(
      partials, rows, in, h, accumulate);
  return cudaGetLastError();
}

}  // namespace nvfp4
