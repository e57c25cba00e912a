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
#include "checks.cuh"
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
  const int64_t xbytes = extent_bytes(T, in, ldx, 2);
  auto ldx16 = [&](const uint16_t* p) {
    return ld_stream_v4(checked(reinterpret_cast<const uint4*>(p), X, xbytes, kSiteDiagX));
  };
  for (int64_t v = vl; v < V; v += VL) {
    float acc[8];
#pragma unroll
    for (int c = 0; c < 8; ++c) acc[c] = 0.0f;
    const uint16_t* col = X + v * 8;
    int64_t t = r;
    for (; t + (U - 1) * R < T; t += U * R) {
      uint4 q[U];
#pragma unroll
      for (int u = 0; u < U; ++u) q[u] = ldx16(col + (t + u * R) * ldx);
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
      const uint4 q = ldx16(col + t * ldx);
      const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float a = bf16_lo(w[k]), b = bf16_hi(w[k]);
        acc[2 * k] = fmaf(a, a, acc[2 * k]);
        acc[2 * k + 1] = fmaf(b, b, acc[2 * k + 1]);
      }
    }
    float4* dst = reinterpret_cast<float4*>(P + r * in + v * 8);
    const int64_t pbytes = R * in * 4;
    *checked(dst, P, pbytes, kSiteDiagPartial) = make_float4(acc[0], acc[1], acc[2], acc[3]);
    *checked(dst + 1, P, pbytes, kSiteDiagPartial) = make_float4(acc[4], acc[5], acc[6], acc[7]);
  }
}

// Second pass: 8 threads per column, thread g adding partial rows g, g + 8,
// ... in FP64 in order; the eight sums are combined in a fixed tree, and the
// result is rounded once to FP32 (deterministic for a given R).  Block:
// 32 columns x 8 row groups.
__global__ void __launch_bounds__(256)
diag_hessian_finalize_kernel(const float* __restrict__ P, int64_t R, int64_t in, float* h,
                             int accumulate) {
  __shared__ double part[8][33];
  const int c = threadIdx.x & 31, g = threadIdx.x >> 5;
  const int64_t j = static_cast<int64_t>(blockIdx.x) * 32 + c;
  double s = 0.0;
  if (j < in)
    for (int64_t r = g; r < R; r += 8) s += *checked(&P[r * in + j], P, R * in * 4, kSiteDiagPartial);
  part[g][c] = s;
  __syncthreads();
  if (g == 0 && j < in) {
    const double t = ((part[0][c] + part[1][c]) + (part[2][c] + part[3][c])) +
                     ((part[4][c] + part[5][c]) + (part[6][c] + part[7][c]));
    float* hj = checked(&h[j], h, in * 4, kSiteDiagH);
    const double base = accumulate ? static_cast<double>(*hj) : 0.0;
    *hj = static_cast<float>(base + t);
  }
}

cudaError_t launch_diag_hessian_finalize(const float* partials, int64_t rows, int64_t in, float* h,
                                         int accumulate, cudaStream_t stream) {
  diag_hessian_finalize_kernel<<<static_cast<unsigned>((in + 31) / 32), 256, 0, stream>>>(
      partials, rows, in, h, accumulate);
  return cudaGetLastError();
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
  return launch_diag_hessian_finalize(partials, rows, in, h, accumulate, stream);
}

}  // namespace nvfp4

// ------------------------------------------------------------------------
// Grouped diagonal Hessian: X holds the calibration rows of E experts one
// after another (expert e owns rows row_offsets[e] .. row_offsets[e+1]) and
// h[e, :] is each expert's own sum of squares -- one launch for all experts.
// Rows are cut into slices of about equal length that never straddle two
// experts, about one wave of them (the plain kernel's shape: each CTA streams
// one long contiguous run of rows).  A CTA sums one slice for one strip of up
// to 256 16-byte column vectors (a fixed-order reduction of its row lanes in
// shared memory) and writes one partial row; the finalize kernel adds each
// expert's partial rows in slice order in FP64 (deterministic) and rounds once.
namespace nvfp4 {

// Plan, on the device since the row offsets live there: slices of about
// `target` rows (total rows / nt), cut at expert boundaries, so that the
// partial kernel's grid is one wave with long contiguous slices per CTA.
// cstart[e] is the first slice of expert e; cstart[E] the number of slices
// (at most nt + E = cap); cstart[E + 1] holds the target.
__global__ void grouped_plan_kernel(const int64_t* __restrict__ off, int64_t E, int64_t total,
                                    int64_t nt, int64_t cap, int64_t* __restrict__ cstart) {
  if (blockIdx.x != 0 || threadIdx.x != 0) return;
  int64_t rows = 0;
  for (int64_t e = 0; e < E; ++e) {
    int64_t a = off[e], b = off[e + 1];
    a = a < 0 ? 0 : (a > total ? total : a);   // out-of-range offsets are clamped:
    b = b < a ? a : (b > total ? total : b);   // no access can leave X
    rows += b - a;
  }
  int64_t target = (rows + nt - 1) / nt;
  if (target < 1) target = 1;
  // cap bounds the slices the workspace holds; monotone offsets stay within it
  // (sum of ceil(rows_e / target) <= nt + E), others cannot push past it
  int64_t acc = 0;
  for (int64_t e = 0; e < E; ++e) {
    cstart[e] = acc < cap ? acc : cap;
    int64_t a = off[e], b = off[e + 1];
    a = a < 0 ? 0 : (a > total ? total : a);
    b = b < a ? a : (b > total ? total : b);
    acc += (b - a + target - 1) / target;
  }
  cstart[E] = acc < cap ? acc : cap;
  cstart[E + 1] = target;
}

template <int U>
__global__ void __launch_bounds__(256)
diag_hessian_grouped_partial_kernel(const uint16_t* __restrict__ X, const int64_t* __restrict__ off,
                                    const int64_t* __restrict__ cstart, int64_t E, int64_t total,
                                    int64_t in, int64_t ldx, float* __restrict__ P) {
  const int64_t q = blockIdx.x;            // slice
  const int64_t strip = blockIdx.y;        // 256 vectors per strip
  if (q >= cstart[E]) return;
  const int64_t target = cstart[E + 1];
  int64_t a = 0, z = E - 1;                // expert: last e with cstart[e] <= q
  while (a < z) {
    const int64_t mid = (a + z + 1) >> 1;
    if (cstart[mid] <= q) a = mid; else z = mid - 1;
  }
  const int64_t e = a;
  int64_t r_lo = off[e], r_hi = off[e + 1];
  r_lo = r_lo < 0 ? 0 : (r_lo > total ? total : r_lo);
  r_hi = r_hi < r_lo ? r_lo : (r_hi > total ? total : r_hi);
  const int64_t rb = r_lo + (q - cstart[e]) * target;
  const int64_t re = (rb + target < r_hi) ? rb + target : r_hi;
  const int64_t V = in / 8;
  const int64_t v0 = strip * 256;
  const int VLc = static_cast<int>((V - v0) < 256 ? (V - v0) : 256);
  const int RL = static_cast<int>(blockDim.x) / VLc;   // the block is a multiple of the widest strip
  const int vl = threadIdx.x % VLc, rl = threadIdx.x / VLc;
  float acc[8];
#pragma unroll
  for (int c = 0; c < 8; ++c) acc[c] = 0.0f;
  if (rl < RL) {
    const uint16_t* col = X + (v0 + vl) * 8;
    int64_t t = rb + rl;
    for (; t + (U - 1) * RL < re; t += U * RL) {
      uint4 qv[U];
#pragma unroll
      for (int u = 0; u < U; ++u) qv[u] = ld_stream_v4(col + (t + u * RL) * ldx);
      float s[8];
#pragma unroll
      for (int c = 0; c < 8; ++c) s[c] = 0.0f;
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const uint32_t w[4] = {qv[u].x, qv[u].y, qv[u].z, qv[u].w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const float x0 = bf16_lo(w[k]), x1 = bf16_hi(w[k]);
          s[2 * k] = fmaf(x0, x0, s[2 * k]);
          s[2 * k + 1] = fmaf(x1, x1, s[2 * k + 1]);
        }
      }
#pragma unroll
      for (int c = 0; c < 8; ++c) acc[c] += s[c];
    }
    for (; t < re; t += RL) {
      const uint4 qv = ld_stream_v4(col + t * ldx);
      const uint32_t w[4] = {qv.x, qv.y, qv.z, qv.w};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float x0 = bf16_lo(w[k]), x1 = bf16_hi(w[k]);
        acc[2 * k] = fmaf(x0, x0, acc[2 * k]);
        acc[2 * k + 1] = fmaf(x1, x1, acc[2 * k + 1]);
      }
    }
  }
  // fixed-order reduction over the row lanes of this CTA
  __shared__ float red[256][9];
#pragma unroll
  for (int c = 0; c < 8; ++c) red[threadIdx.x][c] = acc[c];
  __syncthreads();
  if (rl == 0) {
    for (int r = 1; r < RL; ++r)
#pragma unroll
      for (int c = 0; c < 8; ++c) acc[c] += red[r * VLc + vl][c];
    float4* dst = reinterpret_cast<float4*>(P + q * in + (v0 + vl) * 8);
    dst[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
    dst[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
  }
}

__global__ void __launch_bounds__(256)
diag_hessian_grouped_finalize_kernel(const float* __restrict__ P, const int64_t* __restrict__ cstart,
                                     int64_t E, int64_t in, float* h, int accumulate) {
  const int64_t e = blockIdx.y;
  const int64_t j = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (j >= in || e >= E) return;
  double s = accumulate ? static_cast<double>(h[e * in + j]) : 0.0;
  double t = 0.0;
  for (int64_t q = cstart[e]; q < cstart[e + 1]; ++q) t += P[q * in + j];
  h[e * in + j] = static_cast<float>(s + t);
}

namespace {
// slices of the partial kernel: about one wave of it, less one per expert
// (the rounding at expert boundaries adds at most one slice per expert)
struct GroupedPlan {
  int64_t strips, nt, cap;
  int block;
};
GroupedPlan grouped_plan(int64_t E, int64_t in, int num_sms) {
  GroupedPlan p;
  p.strips = (in / 8 + 255) / 256;
  // threads: row lanes x the widest strip's vectors, so no thread of a
  // narrow row (e.g. 96 vectors for in = 768) idles
  const int64_t v0 = in / 8 < 256 ? in / 8 : 256;
  p.block = static_cast<int>(v0 > 0 ? v0 * (256 / v0) : 256);
  const int ctas = resident_ctas(
      reinterpret_cast<const void*>(&diag_hessian_grouped_partial_kernel<8>), p.block);
  const int64_t per_strip = static_cast<int64_t>(num_sms) * ctas / p.strips;
  p.nt = per_strip - E > 1 ? per_strip - E : 1;
  p.cap = p.nt + E;
  return p;
}
size_t grouped_head_bytes(int64_t E) {
  return ((static_cast<size_t>(E + 2) * sizeof(int64_t)) + 255) & ~size_t{255};
}
}  // namespace

size_t diag_hessian_grouped_workspace_bytes(int64_t total, int64_t E, int64_t in, int num_sms) {
  (void)total;
  const GroupedPlan p = grouped_plan(E, in, num_sms);
  return grouped_head_bytes(E) + static_cast<size_t>(p.cap) * static_cast<size_t>(in) * sizeof(float);
}

// The grouped kernel's plan and partials, for a caller that streams the
// partial pass elsewhere (side_reduce.cuh, kind 2): launch the plan, let the
// tasks (slice q < cap, vector v) write the partials, then the finalize.
GroupedSide grouped_diag_side(int64_t E, int64_t in, void* workspace, int num_sms) {
  const GroupedPlan p = grouped_plan(E, in, num_sms);
  GroupedSide g;
  g.cstart = static_cast<int64_t*>(workspace);
  g.P = reinterpret_cast<float*>(static_cast<char*>(workspace) + grouped_head_bytes(E));
  g.cap = p.cap;
  g.block = p.block;
  g.nt = p.nt;
  return g;
}

cudaError_t launch_grouped_diag_plan(const int64_t* off, int64_t E, int64_t total,
                                     const GroupedSide& g, cudaStream_t stream) {
  grouped_plan_kernel<<<1, 32, 0, stream>>>(off, E, total, g.nt, g.cap, g.cstart);
  return cudaGetLastError();
}

cudaError_t launch_grouped_diag_finalize(int64_t E, int64_t in, float* h, int accumulate,
                                         const GroupedSide& g, cudaStream_t stream) {
  diag_hessian_grouped_finalize_kernel<<<dim3(static_cast<unsigned>((in + 255) / 256),
                                              static_cast<unsigned>(E)),
                                         256, 0, stream>>>(g.P, g.cstart, E, in, h, accumulate);
  return cudaGetLastError();
}

cudaError_t launch_diag_hessian_grouped(const uint16_t* X, const int64_t* off, int64_t E,
                                        int64_t total, int64_t in, int64_t ldx, float* h,
                                        int accumulate, void* workspace, int num_sms,
                                        cudaStream_t stream) {
  const GroupedPlan p = grouped_plan(E, in, num_sms);
  int64_t* cstart = static_cast<int64_t*>(workspace);
  float* P = reinterpret_cast<float*>(static_cast<char*>(workspace) + grouped_head_bytes(E));
  grouped_plan_kernel<<<1, 32, 0, stream>>>(off, E, total, p.nt, p.cap, cstart);
  cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  if (total > 0) {
    diag_hessian_grouped_partial_kernel<8><<<dim3(static_cast<unsigned>(p.cap),
                                                  static_cast<unsigned>(p.strips)),
                                             p.block, 0, stream>>>(X, off, cstart, E, total, in,
                                                                   ldx, P);
    err = cudaGetLastError();
    if (err != cudaSuccess) return err;
  }
  diag_hessian_grouped_finalize_kernel<<<dim3(static_cast<unsigned>((in + 255) / 256),
                                              static_cast<unsigned>(E)),
                                         256, 0, stream>>>(P, cstart, E, in, h, accumulate);
  return cudaGetLastError();
}

}  // namespace nvfp4
