// scale_sweep.cu -- windowed E4M3 block-scale sweep, quantize and pack.
//
// H-Scale summary, sec. 3 "Group-wise scale selection" and "Efficient scale
// search": every 16-wide group picks, among E4M3 codes neighbouring the
// max-abs base code (default nine smaller and six larger steps, clipped at the
// ends of the code range), the scale minimising the h-weighted reconstruction
// error; sec. B "HScaleGroupQuantize": the group is then quantized once with
// the winner and returned in native NVFP4.  ScaleSweep summary, sec. 2-3: the
// base is the FP8-rounded maximum magnitude; windows [-3,+7] (MSE) and [-8,+7]
// (WMSE).
//
// Work layout: one thread owns one group at a time (16 weights and 16 h_j in
// registers).  Lanes: GL column-group lanes x R row lanes; lane (r, gl) takes
// column groups gl, gl+GL, ... (h loaded once per column group) and rows
// r, r+R, ...  Adjacent threads own adjacent groups of one row, so a warp's
// group loads and 8-byte code stores are contiguous.  The next group's 32
// bytes are copied into shared memory with cp.async while the current one is
// being scored (two buffers per thread), which hides the load latency without
// spending registers.
//
// Where a row's column groups fill whole warps (G a multiple of 32), rows are
// handed out at run time instead: the warps of one 32-group column strip take
// chunks of two rows from that strip's counter as they finish, so that warps
// the schedulers favour do more rows and every warp of the grid ends at about
// the same time (with a fixed share per thread, the favoured warps finish
// early and leave their SMs short of warps; the run-time hand-out is 6-8%
// faster).  The counters live in a small pool of slots in device memory
// that launches take in turn (row_counters.cuh); a launch's stream waits for
// the slot's previous launch, the launch's last CTA zeroes the slot, and a
// launch being captured into a graph keeps the fixed stride.
//
// Each group is decided in three stages (fast FP32 pass over all candidates,
// exact FP64 re-scoring of near-ties, exact-decision pack); they live in
// sweep_core.cuh, shared with the online activation quantizer.

#include <algorithm>
#include <type_traits>

#include "checks.cuh"
#include "nvfp4_kernels.cuh"
#include "row_counters.cuh"
#include "side_reduce.cuh"
#include "sweep_core.cuh"

namespace nvfp4 {
// The sweep of one matrix by one thread lane: `tid` in [0, R*GL) is the
// thread's position in the lane grid that covers this matrix.  kFull: the
// candidates are all 126 positive codes in ascending order (lo, hi unused;
// the reported offset is code - base code).
template <bool kWeighted, bool kFull = false, int kMaxK = 16, int kK = 0>
__device__ __forceinline__ void sweep_matrix(SweepSmem<kMaxK>& sm, const uint16_t* __restrict__ W,
                                             int64_t out, int64_t G, int64_t ldw,
                                             const float* __restrict__ h,
                                             const float* __restrict__ Sp, int lo, int hi,
                                             uint8_t* __restrict__ codes,
                                             uint8_t* __restrict__ scales,
                                             int8_t* __restrict__ offs, int64_t GL, int64_t R,
                                             int64_t tid) {
  auto& wbuf = sm.wbuf;
  if (tid >= R * GL) return;
  const int64_t r0 = tid / GL;
  const int64_t gl = tid - r0 * GL;
  const int K = kFull ? kFullK : hi - lo + 1;
  const int lane = threadIdx.x;
  const ScaleConsts sc = scale_consts(*Sp);
  const int64_t half_in = G * 8;

  const int64_t wbytes = extent_bytes(out, G * 16, ldw, 2);
  auto issue = [&](int64_t gg, int64_t rr, int b) {
    const uint16_t* src = W + rr * ldw + gg * 16;
    cp_async16(&wbuf[b][0][lane], checked(reinterpret_cast<const uint4*>(src), W, wbytes, kSiteSweepW));
    cp_async16(&wbuf[b][1][lane],
               checked(reinterpret_cast<const uint4*>(src + 8), W, wbytes, kSiteSweepW));
  };
  int buf = 0;
  if (gl < G && r0 < out) issue(gl, r0, 0);
  cp_async_commit();

  for (int64_t g = gl; g < G; g += GL) {
    f32x2_t h2[8];
    float hs = 1.0f, hsum = 16.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i) h2[i] = f2_pack(1.0f, 1.0f);
    if constexpr (kWeighted) group_weights(h, g, h2, hs, hsum, G);

    for (int64_t r = r0; r < out; r += R) {
      const unsigned amask = __activemask();
      // keep the next group's bytes in flight while this one is scored
      {
        int64_t ng = g, nr = r + R;
        if (nr >= out) { ng = g + GL; nr = r0; }
        if (ng < G) issue(ng, nr, buf ^ 1);
        cp_async_commit();
        cp_async_wait<1>();
      }
      const int cur = buf;
      buf ^= 1;
      sweep_group<kWeighted, kFull, kMaxK, kK>(
          sm, amask, cur, h2, hs, hsum, h, g, sc, lo, K, [&](uint2 c, uint8_t s, int8_t o) {
            const int64_t gi = r * G + g;
            *checked(reinterpret_cast<uint2*>(codes + r * half_in + g * 8), codes, out * half_in,
                     kSiteSweepCodes) = c;
            *checked(scales + gi, scales, out * G, kSiteSweepScales) = s;
            if (offs) *checked(offs + gi, offs, out * G, kSiteSweepOffs) = o;
          }, G);
    }
  }
  cp_async_wait<0>();
}

// ------------------------------------------------- run-time row hand-out

constexpr int kRowChunk = 2;  // rows per hand-out

// The sweep of one matrix with rows handed out at run time.  G % 32 == 0 and
// every lane of the grid's R * G covers one column group of every row chunk
// it takes: chunk r0 first (rows 2 r0, 2 r0 + 1), then chunks R + t for the
// t its strip's counter returns, until they pass the last row.  `slot` is a
// leased counter slot (row_counters.cuh), zero at launch: counter s serves
// strip s.
template <bool kWeighted, int kK>
__device__ __forceinline__ void sweep_rows_dynamic(SweepSmem<16>& sm, const uint16_t* __restrict__ W,
                                                   int64_t out, int64_t G, int64_t ldw,
                                                   const float* __restrict__ h,
                                                   const float* __restrict__ Sp, int lo, int hi,
                                                   uint8_t* __restrict__ codes,
                                                   uint8_t* __restrict__ scales,
                                                   int8_t* __restrict__ offs, int64_t R,
                                                   unsigned int* __restrict__ slot, int64_t tid) {
  auto& wbuf = sm.wbuf;
  const int64_t r0 = tid / G;
  const int64_t g = tid - r0 * G;
  const int K = hi - lo + 1;
  const int lane = threadIdx.x;
  const ScaleConsts sc = scale_consts(*Sp);
  const int64_t half_in = G * 8;
  const int64_t wbytes = extent_bytes(out, G * 16, ldw, 2);
  auto issue = [&](int64_t rr, int b) {
    const uint16_t* src = W + rr * ldw + g * 16;
    cp_async16(&wbuf[b][0][lane], checked(reinterpret_cast<const uint4*>(src), W, wbytes, kSiteSweepW));
    cp_async16(&wbuf[b][1][lane],
               checked(reinterpret_cast<const uint4*>(src + 8), W, wbytes, kSiteSweepW));
  };
  f32x2_t h2[8];
  float hs = 1.0f, hsum = 16.0f;
#pragma unroll
  for (int i = 0; i < 8; ++i) h2[i] = f2_pack(1.0f, 1.0f);
  if constexpr (kWeighted) group_weights(h, g, h2, hs, hsum, G);
  // rows fit in 32 bits here (out <= 2^23), which keeps the loop's state small
  int r = static_cast<int>(r0) * kRowChunk;
  int end = r + kRowChunk;
  const int rows = static_cast<int>(out), Ri = static_cast<int>(R);
  int buf = 0;
  if (r < rows) issue(r, 0);
  cp_async_commit();
  while (r < rows) {
    int nr = r + 1;
    if (nr >= end) {  // warp-uniform: every lane has the same rows
      unsigned int t = 0;
      if ((lane & 31) == 0) t = atomicAdd(slot + (g >> 5), 1u);
      t = __shfl_sync(0xFFFFFFFFu, t, 0);
      nr = (Ri + static_cast<int>(t)) * kRowChunk;
      end = nr + kRowChunk;
    }
    if (nr < rows) issue(nr, buf ^ 1);
    cp_async_commit();
    cp_async_wait<1>();
    const int cur = buf;
    buf ^= 1;
    sweep_group<kWeighted, false, 16, kK>(
        sm, 0xFFFFFFFFu, cur, h2, hs, hsum, h, g, sc, lo, K, [&](uint2 cw, uint8_t sb, int8_t o) {
          const int64_t gi = static_cast<int64_t>(r) * G + g;
          *checked(reinterpret_cast<uint2*>(codes + static_cast<int64_t>(r) * half_in + g * 8),
                   codes, out * half_in, kSiteSweepCodes) = cw;
          *checked(scales + gi, scales, out * G, kSiteSweepScales) = sb;
          if (offs) *checked(offs + gi, offs, out * G, kSiteSweepOffs) = o;
        }, G);
    r = nr;
  }
  cp_async_wait<0>();
}

// Plain MSE over 11 candidates needs the fewest registers; bounded for 7
// CTAs per SM it runs about 3% faster, while the other forms lose to spills.
template <bool kWeighted, int kK>
__global__ void __launch_bounds__(kCta, (!kWeighted && kK == 11) ? 7 : 5)
scale_sweep_kernel(const uint16_t* __restrict__ W, int64_t out, int64_t G, int64_t ldw,
                   const float* __restrict__ h, const float* __restrict__ Sp, int lo, int hi,
                   uint8_t* __restrict__ codes, uint8_t* __restrict__ scales,
                   int8_t* __restrict__ offs, int64_t GL, int64_t R) {
  __shared__ SweepSmem<16> sm;
  fill_candidate_table(sm.tab);
  __syncthreads();
  const int64_t tid = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  sweep_matrix<kWeighted, false, 16, kK>(sm, W, out, G, ldw, h, Sp, lo, hi, codes, scales, offs, GL,
                                         R, tid);
}

// The same with rows handed out at run time (G % 32 == 0); same resources as
// scale_sweep_kernel, so the same number of CTAs fit on an SM.  The last CTA
// to finish zeroes the slot's counters for its next lease.
template <bool kWeighted, int kK>
__global__ void __launch_bounds__(kCta, (!kWeighted && kK == 11) ? 7 : 5)
scale_sweep_rows_kernel(const uint16_t* __restrict__ W, int64_t out, int64_t G, int64_t ldw,
                        const float* __restrict__ h, const float* __restrict__ Sp, int lo, int hi,
                        uint8_t* __restrict__ codes, uint8_t* __restrict__ scales,
                        int8_t* __restrict__ offs, int64_t R, unsigned int* slot) {
  __shared__ SweepSmem<16> sm;
  fill_candidate_table(sm.tab);
  __syncthreads();
  const int64_t tid = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (tid < R * G)
    sweep_rows_dynamic<kWeighted, kK>(sm, W, out, G, ldw, h, Sp, lo, hi, codes, scales, offs, R,
                                      slot, tid);
  finish_slot(slot, static_cast<int>(G >> 5));
}

// The run-time-row sweep with a fifth warp per CTA streaming side reductions
// (side_reduce.cuh).  Four CTAs of 160 threads fit an SM at 96 registers;
// the sweep's four warps per CTA work exactly as in scale_sweep_rows_kernel.
template <bool kWeighted, int kK>
__global__ void __launch_bounds__(kCta + 32, 4)
scale_sweep_side_kernel(const uint16_t* __restrict__ W, int64_t out, int64_t G, int64_t ldw,
                        const float* __restrict__ h, const float* __restrict__ Sp, int lo, int hi,
                        uint8_t* __restrict__ codes, uint8_t* __restrict__ scales,
                        int8_t* __restrict__ offs, int64_t R, unsigned int* slot,
                        const __grid_constant__ SideWork side) {
  __shared__ SweepSmem<16> sm;
  __shared__ SideRing ring;
  fill_candidate_table(sm.tab);
  __syncthreads();
  if (threadIdx.x < kCta) {
    const int64_t tid = static_cast<int64_t>(blockIdx.x) * kCta + threadIdx.x;
    if (tid < R * G)
      sweep_rows_dynamic<kWeighted, kK>(sm, W, out, G, ldw, h, Sp, lo, hi, codes, scales, offs, R,
                                        slot, tid);
  } else {
    run_side_work(side, ring, static_cast<int>(threadIdx.x - kCta), blockIdx.x, gridDim.x);
  }
  finish_slot(slot, static_cast<int>(G >> 5));
}

// Full sweep: every positive E4M3 code is a candidate.  The 126-entry loss
// column needs dynamic shared memory (about 76 KB per CTA).
template <bool kWeighted>
__global__ void __launch_bounds__(kCta, 2)
scale_sweep_full_kernel(const uint16_t* __restrict__ W, int64_t out, int64_t G, int64_t ldw,
                        const float* __restrict__ h, const float* __restrict__ Sp,
                        uint8_t* __restrict__ codes, uint8_t* __restrict__ scales,
                        int8_t* __restrict__ offs, int64_t GL, int64_t R) {
  extern __shared__ __align__(16) unsigned char dsmem[];
  auto& sm = *reinterpret_cast<SweepSmem<kFullK>*>(dsmem);
  fill_candidate_table(sm.tab);
  __syncthreads();
  const int64_t tid = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  sweep_matrix<kWeighted, true, kFullK>(sm, W, out, G, ldw, h, Sp, 0, 0, codes, scales, offs, GL,
                                        R, tid);
}

cudaError_t launch_scale_sweep_full(const uint16_t* W, int64_t out, int64_t in, int64_t ldw,
                                    const float* h, const float* S, uint8_t* codes,
                                    uint8_t* scales, int8_t* offs, int num_sms,
                                    cudaStream_t stream) {
  if (out == 0 || in == 0) return cudaSuccess;
  const size_t smem = sizeof(SweepSmem<kFullK>);
  const void* fn = h ? reinterpret_cast<const void*>(&scale_sweep_full_kernel<true>)
                     : reinterpret_cast<const void*>(&scale_sweep_full_kernel<false>);
  cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  int per_sm = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fn, kCta, smem);
  if (e != cudaSuccess) return e;
  if (per_sm < 1) per_sm = 1;
  const LanePlan p = sweep_plan_threads(out, in, static_cast<int64_t>(num_sms) * per_sm * kCta);
  const unsigned blocks = static_cast<unsigned>((p.threads + kCta - 1) / kCta);
  const int64_t G = in / 16;
  if (h)
    scale_sweep_full_kernel<true><<<blocks, kCta, smem, stream>>>(W, out, G, ldw, h, S, codes,
                                                                  scales, offs, p.VL, p.R);
  else
    scale_sweep_full_kernel<false><<<blocks, kCta, smem, stream>>>(W, out, G, ldw, h, S, codes,
                                                                   scales, offs, p.VL, p.R);
  return cudaGetLastError();
}

// Batched sweep: CTA b belongs to the matrix whose [cta_begin, next cta_begin)
// range holds b (binary search); within it, lanes follow that matrix's plan.
template <bool kWeighted, int kK>
__global__ void __launch_bounds__(kCta, 5)
scale_sweep_batched_kernel(const SweepDesc* __restrict__ d, int64_t n, int lo, int hi) {
  __shared__ SweepSmem<16> sm;
  fill_candidate_table(sm.tab);
  __syncthreads();
  int64_t a = 0, z = n - 1;  // last descriptor with cta_begin <= blockIdx.x
  while (a < z) {
    const int64_t mid = (a + z + 1) >> 1;
    if (d[mid].cta_begin <= static_cast<int64_t>(blockIdx.x)) a = mid; else z = mid - 1;
  }
  const SweepDesc m = d[a];
  const int64_t tid = (static_cast<int64_t>(blockIdx.x) - m.cta_begin) * kCta + threadIdx.x;
  sweep_matrix<kWeighted, false, 16, kK>(sm, m.W, m.out, m.G, m.ldw, m.h, m.S, lo, hi, m.codes,
                                         m.scales, m.offs, m.GL, m.R, tid);
}

// The batched sweep with a fifth warp per CTA streaming side reductions
// (side_reduce.cuh): four CTAs of 160 threads per SM; the side tasks are
// dealt to all CTAs of the launch, which the hardware runs in waves.
template <bool kWeighted, int kK>
__global__ void __launch_bounds__(kCta + 32, 4)
scale_sweep_batched_side_kernel(const SweepDesc* __restrict__ d, int64_t n, int lo, int hi,
                                const __grid_constant__ SideWork side) {
  __shared__ SweepSmem<16> sm;
  __shared__ SideRing ring;
  fill_candidate_table(sm.tab);
  __syncthreads();
  if (threadIdx.x < kCta) {
    int64_t a = 0, z = n - 1;  // last descriptor with cta_begin <= blockIdx.x
    while (a < z) {
      const int64_t mid = (a + z + 1) >> 1;
      if (d[mid].cta_begin <= static_cast<int64_t>(blockIdx.x)) a = mid; else z = mid - 1;
    }
    const SweepDesc m = d[a];
    const int64_t tid = (static_cast<int64_t>(blockIdx.x) - m.cta_begin) * kCta + threadIdx.x;
    sweep_matrix<kWeighted, false, 16, kK>(sm, m.W, m.out, m.G, m.ldw, m.h, m.S, lo, hi, m.codes,
                                           m.scales, m.offs, m.GL, m.R, tid);
  } else {
    run_side_work(side, ring, static_cast<int>(threadIdx.x - kCta), blockIdx.x, gridDim.x);
  }
}

cudaError_t launch_scale_sweep_batched_side(const SweepDesc* d_dev, int64_t n, int64_t total_ctas,
                                            bool weighted, int lo, int hi, const SideWork& side,
                                            cudaStream_t stream) {
  if (n == 0 || total_ctas == 0) return cudaSuccess;
  const unsigned blocks = static_cast<unsigned>(total_ctas);
  const int K = hi - lo + 1;
  if (weighted) {
    if (K == 16)
      scale_sweep_batched_side_kernel<true, 16><<<blocks, kCta + 32, 0, stream>>>(d_dev, n, lo, hi, side);
    else
      scale_sweep_batched_side_kernel<true, 0><<<blocks, kCta + 32, 0, stream>>>(d_dev, n, lo, hi, side);
  } else {
    if (K == 16)
      scale_sweep_batched_side_kernel<false, 16><<<blocks, kCta + 32, 0, stream>>>(d_dev, n, lo, hi, side);
    else
      scale_sweep_batched_side_kernel<false, 0><<<blocks, kCta + 32, 0, stream>>>(d_dev, n, lo, hi, side);
  }
  return cudaGetLastError();
}

int sweep_resident_ctas(bool weighted) {
  static const int ctas[2] = {
      resident_ctas(reinterpret_cast<const void*>(&scale_sweep_kernel<false, 0>), kCta),
      resident_ctas(reinterpret_cast<const void*>(&scale_sweep_kernel<true, 0>), kCta)};
  return ctas[weighted];
}

// Resident CTAs of the instantiation launch_scale_sweep uses for a window of
// K candidates (the compile-time 16- and 11-candidate forms can need fewer
// registers than the general one, and then more CTAs fit).
int sweep_resident_ctas(bool weighted, int K) {
  static const int ctas[2][3] = {
      {resident_ctas(reinterpret_cast<const void*>(&scale_sweep_kernel<false, 0>), kCta),
       resident_ctas(reinterpret_cast<const void*>(&scale_sweep_kernel<false, 16>), kCta),
       resident_ctas(reinterpret_cast<const void*>(&scale_sweep_kernel<false, 11>), kCta)},
      {resident_ctas(reinterpret_cast<const void*>(&scale_sweep_kernel<true, 0>), kCta),
       resident_ctas(reinterpret_cast<const void*>(&scale_sweep_kernel<true, 16>), kCta),
       resident_ctas(reinterpret_cast<const void*>(&scale_sweep_kernel<true, 11>), kCta)}};
  return ctas[weighted][K == 16 ? 1 : (K == 11 ? 2 : 0)];
}

cudaError_t launch_scale_sweep_batched(const SweepDesc* d_dev, int64_t n, int64_t total_ctas,
                                       bool weighted, int lo, int hi, cudaStream_t stream) {
  if (n == 0 || total_ctas == 0) return cudaSuccess;
  const unsigned blocks = static_cast<unsigned>(total_ctas);
  const int K = hi - lo + 1;
  if (weighted) {
    if (K == 16) scale_sweep_batched_kernel<true, 16><<<blocks, kCta, 0, stream>>>(d_dev, n, lo, hi);
    else scale_sweep_batched_kernel<true, 0><<<blocks, kCta, 0, stream>>>(d_dev, n, lo, hi);
  } else {
    if (K == 16) scale_sweep_batched_kernel<false, 16><<<blocks, kCta, 0, stream>>>(d_dev, n, lo, hi);
    else scale_sweep_batched_kernel<false, 0><<<blocks, kCta, 0, stream>>>(d_dev, n, lo, hi);
  }
  return cudaGetLastError();
}

LanePlan sweep_plan(int64_t out, int64_t in, int num_sms, bool weighted, int K) {
  return sweep_plan_threads(out, in,
                            static_cast<int64_t>(num_sms) * sweep_resident_ctas(weighted, K) * kCta);
}

LanePlan sweep_plan_threads(int64_t out, int64_t in, int64_t nt) {
  LanePlan p;
  p.V = in / 16;  // column groups per row
  p.VL = p.V < nt ? (p.V > 0 ? p.V : 1) : nt;
  int64_t R = nt / p.VL;
  if (R > out) R = out;
  if (R < 1) R = 1;
  p.R = R;
  p.threads = p.R * p.VL;
  return p;
}

bool sweep_can_carry(int64_t out, int64_t in, int num_sms) {
  const int64_t G = in / 16;
  if (G == 0 || G % 32 != 0 || G / 32 > kSlotCounters || out > (int64_t{1} << 23)) return false;
  const int64_t nt = static_cast<int64_t>(num_sms) * 4 * kCta;
  return G <= nt && out >= 4 * (nt / G);
}

cudaError_t launch_scale_sweep_side(const uint16_t* W, int64_t out, int64_t in, int64_t ldw,
                                    const float* h, const float* S, int lo, int hi,
                                    uint8_t* codes, uint8_t* scales, int8_t* offs,
                                    const SideWork& side, int num_sms, bool* carried,
                                    cudaStream_t stream) {
  *carried = false;
  if (!sweep_can_carry(out, in, num_sms)) return cudaSuccess;
  CounterLease lease(stream, true);
  unsigned int* slot = lease.slot();
  if (slot == nullptr) return cudaSuccess;
  const int64_t G = in / 16;
  const int64_t R = std::min<int64_t>(static_cast<int64_t>(num_sms) * 4 * kCta / G,
                                      (out + kRowChunk - 1) / kRowChunk);
  const unsigned blocks = static_cast<unsigned>((R * G + kCta - 1) / kCta);
  const int K = hi - lo + 1;
  auto launch = [&](auto weighted, auto kk) {
    scale_sweep_side_kernel<decltype(weighted)::value, decltype(kk)::value>
        <<<blocks, kCta + 32, 0, stream>>>(W, out, G, ldw, h, S, lo, hi, codes, scales, offs, R,
                                           slot, side);
  };
  using T16 = std::integral_constant<int, 16>;
  using T11 = std::integral_constant<int, 11>;
  using T0 = std::integral_constant<int, 0>;
  if (h) {
    if (K == 16) launch(std::true_type{}, T16{});
    else if (K == 11) launch(std::true_type{}, T11{});
    else launch(std::true_type{}, T0{});
  } else {
    if (K == 16) launch(std::false_type{}, T16{});
    else if (K == 11) launch(std::false_type{}, T11{});
    else launch(std::false_type{}, T0{});
  }
  const cudaError_t e = lease.commit(cudaGetLastError());
  *carried = e == cudaSuccess;
  return e;
}

cudaError_t launch_scale_sweep(const uint16_t* W, int64_t out, int64_t in, int64_t ldw,
                               const float* h, const float* S, int lo, int hi, uint8_t* codes,
                               uint8_t* scales, int8_t* offs, const LanePlan& p,
                               cudaStream_t stream) {
  if (out == 0) return cudaSuccess;
  const int64_t G = in / 16;
  // the two window sizes the pages use get a compile-time candidate count
  const int K = hi - lo + 1;
  // run-time row hand-out where whole warps fit a row's groups and every row
  // lane would otherwise take at least four rows
  const bool handout = G % 32 == 0 && p.VL == G && G / 32 <= kSlotCounters &&
                       out <= (int64_t{1} << 23) && out >= 4 * p.R;
  CounterLease lease(stream, handout);
  unsigned int* slot = lease.slot();
  const int64_t Rd = std::min<int64_t>(p.R, (out + kRowChunk - 1) / kRowChunk);
  auto launch = [&](auto weighted, auto kk) {
    constexpr bool kW = decltype(weighted)::value;
    constexpr int kKK = decltype(kk)::value;
    if (slot != nullptr) {
      const unsigned blocks = static_cast<unsigned>((Rd * G + kCta - 1) / kCta);
      scale_sweep_rows_kernel<kW, kKK><<<blocks, kCta, 0, stream>>>(
          W, out, G, ldw, h, S, lo, hi, codes, scales, offs, Rd, slot);
    } else {
      const unsigned blocks = static_cast<unsigned>((p.threads + kCta - 1) / kCta);
      scale_sweep_kernel<kW, kKK><<<blocks, kCta, 0, stream>>>(W, out, G, ldw, h, S, lo, hi, codes,
                                                             scales, offs, p.VL, p.R);
    }
  };
  using T16 = std::integral_constant<int, 16>;
  using T11 = std::integral_constant<int, 11>;
  using T0 = std::integral_constant<int, 0>;
  if (h) {
    if (K == 16) launch(std::true_type{}, T16{});
    else if (K == 11) launch(std::true_type{}, T11{});
    else launch(std::true_type{}, T0{});
  } else {
    if (K == 16) launch(std::false_type{}, T16{});
    else if (K == 11) launch(std::false_type{}, T11{});
    else launch(std::false_type{}, T0{});
  }
  return lease.commit(cudaGetLastError());
}

}  // namespace nvfp4
