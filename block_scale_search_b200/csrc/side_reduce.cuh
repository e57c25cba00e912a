// side_reduce.cuh -- reductions a sweep launch streams beside its own work.
//
// The sweep is bound by FP32 arithmetic and leaves HBM nearly idle, while the
// diagonal Hessian and the absmax of a global scale are bound by HBM.  A sweep
// CTA can therefore carry one extra warp that streams other inputs' reductions
// for weights swept later.  The warp's lanes each own one task of the
// standalone kernels' lane grid -- R row lanes x V 16-byte column vectors; task
// (r, v) covers rows r, r + R, ... of vector v -- so a diagonal-Hessian task
// writes exactly the partial row the standalone kernel writes (same order of
// operations, bit for bit), and the standalone finalize applies.  An absmax
// task folds its maximum into one word with atomicMax (exact in any order).
//
// Loads go through a per-lane ring in shared memory with cp.async (four
// batches of eight rows in flight), so no registers wait on memory; squares
// are summed with the mixed-precision bf16 FMA, whose exact product and single
// rounding equal fmaf on the widened values.
#pragma once

#include "nvfp4_device.cuh"
#include "sweep_core.cuh"

namespace nvfp4 {

constexpr int kSideRows = 8;     // rows per batch (the standalone kernel's run length)
constexpr int kSideBatches = 4;  // batches in flight per lane
constexpr int kMaxSideJobs = 8;

// One reduction's share of tasks [t0, t1) of its task grid.
struct SideJob {
  const uint16_t* A;   // bf16 [rows, ld]
  int64_t rows, ld;
  int64_t cols;        // elements per row (a multiple of 8)
  int64_t R;           // kinds 0, 1: row lanes of the task grid (R x V tasks)
  int64_t t0, t1;      // task range
  float* P;            // kinds 0, 2: partials
  uint32_t* amax;      // kind 1: the max word (bf16 bit pattern of |a|)
  // kind 2: expert-contiguous rows, as the grouped diagonal-Hessian kernel
  // reads them: row offsets [E + 1], its slice plan (device), and its CTA size
  const int64_t* off;
  const int64_t* cstart;
  int64_t E;
  int block;
  int kind;            // 0: diagonal Hessian, 1: absmax, 2: grouped diagonal Hessian
};

struct SideWork {
  SideJob job[kMaxSideJobs];
  int n;
  int64_t tasks;       // sum of t1 - t0
};

// Ring of the side warp: [batch slot * rows][lane].
struct SideRing {
  uint4 v[kSideBatches * kSideRows][32];
};

// x^2 + s for the two bf16 halves of w, each with one rounding.
__device__ __forceinline__ void sq_acc_bf16x2(uint32_t w, float& s0, float& s1) {
  asm("{ .reg .b16 l, h; mov.b32 {l, h}, %2;\n\t"
      "fma.rn.f32.bf16 %0, l, l, %0;\n\t"
      "fma.rn.f32.bf16 %1, h, h, %1; }"
      : "+f"(s0), "+f"(s1) : "r"(w));
}

// x^2 + 0 for the two bf16 halves of w: the same single rounding as
// sq_acc_bf16x2 on zeroed sums, without registers to zero.
__device__ __forceinline__ void sq_first_bf16x2(uint32_t w, float& s0, float& s1) {
  asm("{ .reg .b16 l, h; mov.b32 {l, h}, %2;\n\t"
      "fma.rn.f32.bf16 %0, l, l, 0f00000000;\n\t"
      "fma.rn.f32.bf16 %1, h, h, 0f00000000; }"
      : "=f"(s0), "=f"(s1) : "r"(w));
}

// The running maximum of eight sign-cleared bf16 patterns (two per 32 bits).
__device__ __forceinline__ uint32_t absmax_bf16x8(uint32_t m, const uint4& q) {
  return __vmaxu2(__vmaxu2(m, q.x & 0x7FFF7FFFu),
                  __vmaxu2(__vmaxu2(q.y & 0x7FFF7FFFu, q.z & 0x7FFF7FFFu), q.w & 0x7FFF7FFFu));
}

// Rows t0, t0 + stride, ... below t_end of one 16-byte column (col; ld
// elements per row): full runs of kSideRows rows through the ring, then the
// remaining rows one by one, as the standalone kernels order them.  kSq: sums
// of squares added into acc (a run summed first, then added); otherwise the
// maximum of sign-cleared patterns into m.
template <bool kSq>
__device__ __forceinline__ void side_stream(const uint16_t* col, int64_t ld, int64_t t0,
                                            int64_t stride, int64_t t_end, SideRing& ring,
                                            int lane, float (&acc)[8], uint32_t& m) {
  const int64_t n = t_end > t0 ? (t_end - t0 + stride - 1) / stride : 0;
  const int64_t runs = n / kSideRows;
  // rows are issued in order: a running pointer advanced by one row stride
  const int64_t step = stride * ld;
  const uint16_t* next_row = col + t0 * ld;
  auto issue = [&](int64_t k) {
    const int slot = static_cast<int>(k % kSideBatches) * kSideRows;
#pragma unroll
    for (int u = 0; u < kSideRows; ++u) {
      cp_async16(&ring.v[slot + u][lane], next_row);
      next_row += step;
    }
  };
#pragma unroll
  for (int k = 0; k < kSideBatches; ++k) {
    if (k < runs) issue(k);
    cp_async_commit();
  }
  for (int64_t k = 0; k < runs; ++k) {
    cp_async_wait<kSideBatches - 1>();
    const int slot = static_cast<int>(k % kSideBatches) * kSideRows;
    if constexpr (kSq) {
      float s[8];
      {
        const uint4 q = ring.v[slot][lane];
        sq_first_bf16x2(q.x, s[0], s[1]);
        sq_first_bf16x2(q.y, s[2], s[3]);
        sq_first_bf16x2(q.z, s[4], s[5]);
        sq_first_bf16x2(q.w, s[6], s[7]);
      }
#pragma unroll
      for (int u = 1; u < kSideRows; ++u) {
        const uint4 q = ring.v[slot + u][lane];
        sq_acc_bf16x2(q.x, s[0], s[1]);
        sq_acc_bf16x2(q.y, s[2], s[3]);
        sq_acc_bf16x2(q.z, s[4], s[5]);
        sq_acc_bf16x2(q.w, s[6], s[7]);
      }
#pragma unroll
      for (int c = 0; c < 8; ++c) acc[c] += s[c];
    } else {
#pragma unroll
      for (int u = 0; u < kSideRows; ++u) m = absmax_bf16x8(m, ring.v[slot + u][lane]);
    }
    if (k + kSideBatches < runs) issue(k + kSideBatches);
    cp_async_commit();
  }
  cp_async_wait<0>();
  for (int64_t t = t0 + runs * kSideRows * stride; t < t_end; t += stride, next_row += step) {
    const uint4 q = ld_stream_v4(next_row);
    if constexpr (kSq) {
      sq_acc_bf16x2(q.x, acc[0], acc[1]);
      sq_acc_bf16x2(q.y, acc[2], acc[3]);
      sq_acc_bf16x2(q.z, acc[4], acc[5]);
      sq_acc_bf16x2(q.w, acc[6], acc[7]);
    } else {
      m = absmax_bf16x8(m, q);
    }
  }
}

__device__ __forceinline__ void store_partial(float* p, const float (&acc)[8]) {
  float4* dst = reinterpret_cast<float4*>(p);
  dst[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
  dst[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
}

// Task t of a job.  Kinds 0 and 1: t = r V + v covers rows r, r + R, ... of
// vector v.  Kind 2: t = q V + v is slice q of the grouped kernel's plan for
// vector v: the row lanes of that kernel's CTA one after another, each as that
// lane streams it, then added in lane order as its CTA does.
__device__ __forceinline__ void side_task(const SideJob& j, int64_t t, SideRing& ring, int lane) {
  const int64_t V = j.cols / 8;
  const int64_t q = t / V, v = t - q * V;
  const uint16_t* col = j.A + v * 8;
  float acc[8];
  uint32_t m = 0;
#pragma unroll
  for (int c = 0; c < 8; ++c) acc[c] = 0.0f;
  if (j.kind == 0) {
    side_stream<true>(col, j.ld, q, j.R, j.rows, ring, lane, acc, m);
    store_partial(j.P + q * j.cols + v * 8, acc);
  } else if (j.kind == 1) {
    side_stream<false>(col, j.ld, q, j.R, j.rows, ring, lane, acc, m);
    m = max(m & 0xFFFFu, m >> 16);
    if (m != 0u) atomicMax(j.amax, m);
  } else {
    const int64_t E = j.E;
    if (q >= j.cstart[E]) return;  // beyond the plan's slices
    const int64_t target = j.cstart[E + 1];
    int64_t a = 0, z = E - 1;       // expert: last e with cstart[e] <= q
    while (a < z) {
      const int64_t mid = (a + z + 1) >> 1;
      if (j.cstart[mid] <= q) a = mid; else z = mid - 1;
    }
    int64_t r_lo = j.off[a], r_hi = j.off[a + 1];
    r_lo = r_lo < 0 ? 0 : (r_lo > j.rows ? j.rows : r_lo);
    r_hi = r_hi < r_lo ? r_lo : (r_hi > j.rows ? j.rows : r_hi);
    const int64_t rb = r_lo + (q - j.cstart[a]) * target;
    const int64_t re = (rb + target < r_hi) ? rb + target : r_hi;
    const int64_t v0 = (v / 256) * 256;
    const int64_t VLc = (V - v0) < 256 ? (V - v0) : 256;
    const int64_t RL = j.block / VLc;
    for (int64_t rl = 0; rl < RL; ++rl) {
      float part[8];
#pragma unroll
      for (int c = 0; c < 8; ++c) part[c] = 0.0f;
      side_stream<true>(col, j.ld, rb + rl, RL, re, ring, lane, part, m);
#pragma unroll
      for (int c = 0; c < 8; ++c) acc[c] = rl == 0 ? part[c] : acc[c] + part[c];
    }
    store_partial(j.P + q * j.cols + v * 8, acc);
  }
}

// The side warp of CTA `cta` of `ctas`: lane l takes tasks cta*32 + l,
// cta*32 + l + 32*ctas, ... of the jobs' concatenated ranges (adjacent lanes
// take adjacent column vectors of one row lane: coalesced loads).
__device__ __forceinline__ void run_side_work(const SideWork& w, SideRing& ring, int lane,
                                              int64_t cta, int64_t ctas) {
  int jb = 0;
  int64_t base = 0;  // tasks of the jobs before jb
  for (int64_t k = cta * 32 + lane; k < w.tasks; k += ctas * 32) {
    while (jb < w.n && k - base >= w.job[jb].t1 - w.job[jb].t0) {
      base += w.job[jb].t1 - w.job[jb].t0;
      ++jb;
    }
    if (jb >= w.n) break;
    const SideJob& j = w.job[jb];
    side_task(j, j.t0 + (k - base), ring, lane);
  }
}

}  // namespace nvfp4
