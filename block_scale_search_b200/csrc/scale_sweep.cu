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
// Each group is decided in three stages:
//  1. Fast pass, FP32, all K candidates (the loop that bounds the kernel):
//       y_j = |w_j| / S            (|w_j| * p * (1/(S p)), p = 2^k for denormal S)
//       x_j = y_j * (1/v_c)        candidate-scaled weight      [FMUL2]
//       q_j = E2M1_RNE_sat(x_j)    hardware cvt to e2m1x2 and back to f16x2
//       e_j = y_j - q_j v_c        mixed f16 x f16 + f32 FMA (exact product)
//       L_c = sum_j h'_j e_j^2     [FMUL2, FFMA2]; h' = h * 2^k, max h' in [.5,1)
//     Losses go to a per-thread shared-memory column; the running minimum and
//     second minimum stay in registers.
//  2. Near-tie guard: per candidate, |L_fast - L_definition| is at most about
//     2^-21.4 sqrt(A L) (rounding of y; Cauchy-Schwarz with A = sum h' y^2)
//     + 2^-20.4 L (products and sums) + 2^-17.2 L (an E2M1 decision taken on
//     an FP32 quotient within 2^-22 of the exact one can pick the other side
//     of a midpoint; that element's term then grows by at most 2^-19 x/step
//     <= 3.5 * 2^-19 of itself).  Candidates whose fast loss lies within
//     2^-19 sqrt(A L) + 2^-15 L of the minimum -- about twice the two-sided
//     bound -- are re-scored exactly as the definition does: exact-real
//     E2M1 decisions, d = |w| - q v S in FP64 (exact), L = sum h d^2 in FP64
//     in element order -- and the strict "<" in offset order picks among them.
//     Exact ties (octave pairs that reconstruct every element alike, symmetric
//     errors) and near-ties therefore resolve to the lowest offset exactly as
//     the definition does.  This stage runs for well under 1% of groups.
//  3. Pack with exact decisions: the FP32 quotient is bracketed by
//     (1 -+ 2^-20); where the bracket straddles an E2M1 midpoint m, the sign of
//     fma(m v, S, -|w|) (one rounding of the exact m v S - |w|) decides, zero
//     being a tie to the even code.
#include "nvfp4_kernels.cuh"

namespace nvfp4 {

// Per-code table in shared memory, indexed by code + 16 so that b + k for
// k in [-16, 15] needs no clamping (entries beyond the ends repeat codes 1/126).
struct CandEntry {
  float iv;       // 1 / v, correctly rounded
  float iv2;      // the same again, so {iv, iv} loads as one f32x2 operand
  uint32_t nvh;   // -v as f16 bits (exact: E4M3 values are f16 values)
  float v;        // E4M3 value of the (clamped) code
};
constexpr int kTabOffset = 16;
constexpr int kTabSize = 160;
constexpr int kCta = 128;

// -------------------------------------------------------------- cp.async

__device__ __forceinline__ void cp_async16(void* smem, const void* gmem) {
  const uint32_t s = static_cast<uint32_t>(__cvta_generic_to_shared(smem));
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(s), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ float sqrt_approx(float x) {
  float r;
  asm("sqrt.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
  return r;
}

// ----------------------------------------------------- exact E2M1 decisions

// Exact E2M1 index of |w| / (v S) for two elements, given their FP32 quotients
// xl (computed with 1/v lowered by 2^-20) -- the exact quotient lies in
// (xl, xl (1 + 2^-19)).  Where both ends round alike that is the answer;
// otherwise the bracket straddles one midpoint m and the sign of
// fma(m v, S, -|w|), the correctly rounded m v S - |w|, decides (zero: a tie,
// to the even code).  Returns the two 3-bit indices in bits 0..2 and 4..6.
__device__ __forceinline__ uint32_t exact_e2m1_pair(float xl0, float xl1, float a0, float a1,
                                                    float v, float S) {
  uint32_t nlo = e2m1x2_rne(xl0, xl1) & 0x77u;
  const uint32_t nhi = e2m1x2_rne(xl0 * (1.0f + 0x1p-19f), xl1 * (1.0f + 0x1p-19f)) & 0x77u;
  if (nlo != nhi) {
#pragma unroll
    for (int t = 0; t < 2; ++t) {
      const uint32_t kl = (nlo >> (4 * t)) & 7u, kh = (nhi >> (4 * t)) & 7u;
      if (kl != kh) {
        const float m = 0.5f * (e2m1_nibble_value(kl) + e2m1_nibble_value(kh));  // exact
        const float rr = fmaf(m * v, S, -(t ? a1 : a0));
        const uint32_t k = (rr < 0.0f) ? kh : (rr > 0.0f ? kl : ((kl & 1u) ? kh : kl));
        nlo = (nlo & ~(7u << (4 * t))) | (k << (4 * t));
      }
    }
  }
  return nlo;
}

// y = |w| / S as the fast pass computes it (the same operations, so the same
// bits, wherever it is recomputed).
__device__ __forceinline__ f32x2_t scaled_pair(uint32_t w, float p, float inv_sp, bool tiny_s) {
  f32x2_t a2 = f2_pack(fabsf(bf16_lo(w)), fabsf(bf16_hi(w)));
  if (tiny_s) a2 = f2_mul(a2, f2_pack(p, p));
  return f2_mul(a2, f2_pack(inv_sp, inv_sp));
}

// Group weights h' = h * hs, hs the power of two that puts max h' in [0.5, 1)
// (exact; the argmin is invariant and neither overflow nor underflow can
// distort the sums).
__device__ __forceinline__ float weight_scale(float hmax) {
  const uint32_t ex = __float_as_uint(hmax) & 0x7F800000u;
  float hs = 1.0f;
  if (hmax > 0.0f && ex != 0x7F800000u) {
    if (ex == 0u) hs = 0x1p100f;                       // denormal maximum
    else if (ex >= (250u << 23)) hs = 0x1p-124f;       // near FLT_MAX
    else hs = __uint_as_float(0x7E800000u - ex);       // 2^(126 - E)
  }
  return hs;
}

// -------------------------------------------------------- stage 1 (fast)

// Fast FP32 loss of one candidate: E2M1 round of y/v by the hardware
// conversion, decode, exact-product error, weighted square, two accumulators.
template <bool kWeighted>
__device__ __forceinline__ float fast_candidate_loss(const f32x2_t (&y2)[8], const f32x2_t (&h2)[8],
                                                     const CandEntry& t) {
  const f32x2_t iv2 = *reinterpret_cast<const f32x2_t*>(&t.iv);  // {iv, iv}
  const uint16_t nv = static_cast<uint16_t>(t.nvh);
  f32x2_t acc0, acc1;
#pragma unroll
  for (int pj = 0; pj < 8; ++pj) {
    float x0, x1, y0, y1;
    f2_unpack(f2_mul(y2[pj], iv2), x0, x1);
    f2_unpack(y2[pj], y0, y1);
    const uint32_t qh = e2m1x2_round_f16x2(x0, x1);
    const float e0 = fma_f16_f32(static_cast<uint16_t>(qh & 0xFFFFu), nv, y0);
    const float e1 = fma_f16_f32(static_cast<uint16_t>(qh >> 16), nv, y1);
    const f32x2_t e2 = f2_pack(e0, e1);
    // plain MSE (h == 1) needs no weighting multiply
    const f32x2_t he2 = kWeighted ? f2_mul(h2[pj], e2) : e2;
    if (pj == 0) acc0 = f2_mul(he2, e2);
    else if (pj == 1) acc1 = f2_mul(he2, e2);
    else if (pj & 1) acc1 = f2_fma(he2, e2, acc1);
    else acc0 = f2_fma(he2, e2, acc0);
  }
  float a0, a1;
  f2_unpack(f2_add(acc0, acc1), a0, a1);
  return a0 + a1;
}

// ------------------------------------------------------- stage 2 (exact)

// Exact E2M1 index of one element (see exact_e2m1_pair).
__device__ __forceinline__ uint32_t exact_e2m1_one(float xl, float a, float v, float S) {
  const uint32_t kl = e2m1x2_rne(xl, 0.0f) & 7u;
  const uint32_t kh = e2m1x2_rne(xl * (1.0f + 0x1p-19f), 0.0f) & 7u;
  if (kl == kh) return kl;
  const float m = 0.5f * (e2m1_nibble_value(kl) + e2m1_nibble_value(kh));  // exact
  const float rr = fmaf(m * v, S, -a);
  return (rr < 0.0f) ? kh : (rr > 0.0f ? kl : ((kl & 1u) ? kh : kl));
}

// ------------------------------------------------------------------ kernel

// Shared memory of one sweep CTA; kMaxK candidates per group at most (16 for
// windows, 126 for the full sweep over every positive E4M3 code).
template <int kMaxK>
struct SweepSmem {
  CandEntry tab[kTabSize];
  float Lsm[kMaxK][kCta];     // per-thread column of fast losses
  uint4 wbuf[2][2][kCta];     // staged groups: [buffer][half][thread]
  double tsm[kCta / 32][16];  // per-warp exchange of exact loss terms
};
constexpr int kFullK = 126;

__device__ __forceinline__ void fill_candidate_table(CandEntry* tab) {
  for (int i = threadIdx.x; i < kTabSize; i += blockDim.x) {
    const int c = clamp_code(i - kTabOffset);
    const float v = e4m3_value(c);
    const float iv = __frcp_rn(v);
    const uint32_t nvh = __half_as_ushort(__float2half_rn(-v));
    tab[i] = CandEntry{iv, iv, nvh | (nvh << 16), v};
  }
}

// The sweep of one matrix by one thread lane: `tid` in [0, R*GL) is the
// thread's position in the lane grid that covers this matrix.  kFull: the
// candidates are all 126 positive codes in ascending order (lo, hi unused;
// the reported offset is code - base code).
template <bool kWeighted, bool kFull = false, int kMaxK = 16>
__device__ __forceinline__ void sweep_matrix(SweepSmem<kMaxK>& sm, const uint16_t* __restrict__ W,
                                             int64_t out, int64_t G, int64_t ldw,
                                             const float* __restrict__ h,
                                             const float* __restrict__ Sp, int lo, int hi,
                                             uint8_t* __restrict__ codes,
                                             uint8_t* __restrict__ scales,
                                             int8_t* __restrict__ offs, int64_t GL, int64_t R,
                                             int64_t tid) {
  const CandEntry* tab = sm.tab;
  auto& Lsm = sm.Lsm;
  auto& wbuf = sm.wbuf;
  auto& tsm = sm.tsm;
  if (tid >= R * GL) return;
  const int64_t r0 = tid / GL;
  const int64_t gl = tid - r0 * GL;
  const int K = kFull ? kFullK : hi - lo + 1;
  const int lane = threadIdx.x;

  const float S = *Sp;
  const bool tiny_s = S < 0x1p-100f;         // keep 1/(S p) finite for denormal S
  const float p = tiny_s ? 0x1p100f : 1.0f;
  const float inv_sp = __frcp_rn(S * p);
  // the base-code bracket needs 1/S normal; outside that range the IEEE
  // divisions decide every group
  const bool exact_base = tiny_s || !(S < 0x1p100f);
  const float inv_s6 = __frcp_rn(S) * (1.0f / 6.0f);
  const int64_t half_in = G * 8;

  auto issue = [&](int64_t gg, int64_t rr, int b) {
    const uint16_t* src = W + rr * ldw + gg * 16;
    cp_async16(&wbuf[b][0][lane], src);
    cp_async16(&wbuf[b][1][lane], src + 8);
  };
  int buf = 0;
  if (gl < G && r0 < out) issue(gl, r0, 0);
  cp_async_commit();

  for (int64_t g = gl; g < G; g += GL) {
    f32x2_t h2[8];
    float hs = 1.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i) h2[i] = f2_pack(1.0f, 1.0f);
    if constexpr (kWeighted) {
      const float4* hp = reinterpret_cast<const float4*>(h + g * 16);
      float4 hv[4];
      float hmax = 0.0f;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        hv[i] = hp[i];
        hmax = fmaxf(fmaxf(fmaxf(hmax, hv[i].x), fmaxf(hv[i].y, hv[i].z)), hv[i].w);
      }
      hs = weight_scale(hmax);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        h2[2 * i] = f2_pack(hv[i].x * hs, hv[i].y * hs);
        h2[2 * i + 1] = f2_pack(hv[i].z * hs, hv[i].w * hs);
      }
    }

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
      const uint4 wa = wbuf[cur][0][lane], wb = wbuf[cur][1][lane];
      const uint32_t wr[8] = {wa.x, wa.y, wa.z, wa.w, wb.x, wb.y, wb.z, wb.w};

      // group absmax on the sign-cleared bit patterns
      uint32_t mb = 0;
#pragma unroll
      for (int i = 0; i < 8; ++i) mb = __vmaxu2(mb, wr[i] & 0x7FFF7FFFu);
      mb = max(mb & 0xFFFFu, mb >> 16);
      const bool nonzero = mb != 0u;   // all-zero group: scale 0, codes 0

      f32x2_t y2[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) y2[i] = scaled_pair(wr[i], p, inv_sp, tiny_s);
      int b = 1, bi = 0;
      float T = 0.0f;
      bool flagged = false;
      if (nonzero) {
        f32x2_t A2 = f2_pack(0.0f, 0.0f);  // sum h' y^2, for the error bound of stage 2
#pragma unroll
        for (int i = 0; i < 8; ++i) A2 = f2_fma(kWeighted ? f2_mul(h2[i], y2[i]) : y2[i], y2[i], A2);
        float A0, A1;
        f2_unpack(A2, A0, A1);
        const float A = A0 + A1;

        // base code: E4M3_RNE_sat(fl32(fl32(a / 6) / S)), clamped to [1, 126].
        // An FP32 approximation within 2^-21 decides unless an E4M3 rounding
        // boundary lies within 2^-20 of it; then the two IEEE divisions do.
        const float a = __uint_as_float(mb << 16);
        const float ua = a * inv_s6;
        const int blo = e4m3_code_rne_sat(ua * (1.0f - 0x1p-20f));
        const int bhi = e4m3_code_rne_sat(ua * (1.0f + 0x1p-20f));
        b = (blo == bhi && !exact_base) ? blo : e4m3_code_rne_sat(__fdiv_rn(__fdiv_rn(a, 6.0f), S));
        b = clamp_code(b);
        const CandEntry* ce = kFull ? tab + (1 + kTabOffset) : tab + (b + lo + kTabOffset);

        // ---- stage 1: fast FP32 losses of all candidates
        float best = __uint_as_float(0x7F800000u), second = best;
        for (int i = 0; i < K; ++i) {
          const float Li = fast_candidate_loss<kWeighted>(y2, h2, ce[i]);
          Lsm[i][lane] = Li;
          if (Li < best) { second = best; best = Li; bi = i; }
          else if (Li < second) { second = Li; }
        }

        // ---- stage 2 guard.  L is flagged when L - best <= c1 sqrt(A L) + c2 L;
        // as the right side grows more slowly than L, that is L <= T with
        // sqrt(T) the positive root of (1 - c2) s^2 - c1 sqrt(A) s - best = 0
        // (T rounded up with margin for the approximate square roots).  Some
        // other candidate is flagged iff the second-smallest loss is.
        constexpr float c1 = 0x1p-19f, c2 = 0x1p-15f;
        constexpr float k2 = 1.0f / (2.0f * (1.0f - c2));
        const float ca = c1 * sqrt_approx(A);
        const float sr = (ca + sqrt_approx(fmaf(ca, ca, 4.0f * (1.0f - c2) * best))) * k2;
        T = sr * sr * (1.0f + 0x1p-16f);
        flagged = second <= T;
      }

      // ---- stage 2, rare: the warp resolves its flagged groups together.  For
      // each flagged group, the active lanes share its 16 elements, each
      // computing the definition's term h (|w| - q v S)^2 in FP64 with an exact
      // E2M1 decision; the terms are summed in element order, and the first
      // strict minimum in offset order among the flagged candidates wins.
      __syncwarp(amask);
      unsigned fl = __ballot_sync(amask, flagged);
      if (fl) {
        const int lid = lane & 31;
        const int rank = __popc(amask & ((1u << lid) - 1u));
        const int nact = __popc(amask);
        double* tw = &tsm[lane >> 5][0];
        while (fl) {
          const int f = __ffs(fl) - 1;
          fl &= fl - 1u;
          const int tx = (lane & ~31) + f;
          const int b_f = __shfl_sync(amask, b, f);
          const float T_f = __shfl_sync(amask, T, f);
          const int64_t g_f = __shfl_sync(amask, static_cast<long long>(g), f);
          const int cur_f = __shfl_sync(amask, cur, f);
          const float hs_f = __shfl_sync(amask, hs, f);
          const CandEntry* ce_f = kFull ? tab + (1 + kTabOffset) : tab + (b_f + lo + kTabOffset);
          const uint32_t* wf = reinterpret_cast<const uint32_t*>(&wbuf[cur_f][0][0]);
          double bestd = __longlong_as_double(0x7FF0000000000000ll);
          int bid = 0;
          for (int i = 0; i < K; ++i) {
            if (Lsm[i][tx] > T_f) continue;  // same for every lane
            const CandEntry t = ce_f[i];
            const float ivl = t.iv * (1.0f - 0x1p-20f);
            const double vS = __dmul_rn(static_cast<double>(t.v), static_cast<double>(S));
            for (int j = rank; j < 16; j += nact) {
              // element j of group f: bf16 word (j >> 1) of its two staged halves
              const uint32_t word = wf[((j >> 3) * kCta + tx) * 4 + ((j >> 1) & 3)];
              const float aj = fabsf((j & 1) ? bf16_hi(word) : bf16_lo(word));
              const float yj = (tiny_s ? aj * p : aj) * inv_sp;
              const float hj = kWeighted ? h[g_f * 16 + j] * hs_f : 1.0f;
              const uint32_t k = exact_e2m1_one(yj * ivl, aj, t.v, S);
              const double q = static_cast<double>(e2m1_nibble_value(k));
              const double d = fma(-q, vS, static_cast<double>(aj));  // exact
              tw[j] = __dmul_rn(static_cast<double>(hj), __dmul_rn(d, d));
            }
            __syncwarp(amask);
            double Ld = 0.0;
#pragma unroll
            for (int j = 0; j < 16; ++j) Ld = __dadd_rn(Ld, tw[j]);
            __syncwarp(amask);
            if (Ld < bestd) { bestd = Ld; bid = i; }
          }
          if (lid == f) bi = bid;
        }
      }

      const int64_t gi = r * G + g;
      uint8_t* cdst = codes + r * half_in + g * 8;
      if (!nonzero) {
        *reinterpret_cast<uint2*>(cdst) = make_uint2(0u, 0u);
        scales[gi] = 0;
        if (offs) offs[gi] = 0;
        continue;
      }
      const int wcode = kFull ? 1 + bi : clamp_code(b + lo + bi);
      const CandEntry win = tab[wcode + kTabOffset];

      // ---- stage 3: quantize once with the winner, exact decisions, pack
      const f32x2_t ivlo = f2_pack(win.iv * (1.0f - 0x1p-20f), win.iv * (1.0f - 0x1p-20f));
      uint32_t packed[2] = {0u, 0u};
#pragma unroll
      for (int pj = 0; pj < 8; ++pj) {
        float xl0, xl1;
        f2_unpack(f2_mul(y2[pj], ivlo), xl0, xl1);
        const uint32_t nib = exact_e2m1_pair(xl0, xl1, fabsf(bf16_lo(wr[pj])),
                                             fabsf(bf16_hi(wr[pj])), win.v, S);
        // signs: bf16 bit 15 (low element) and bit 31 (high element); +0 for zero
        const uint32_t sgn = ((wr[pj] >> 15) & 1u) << 3 | ((wr[pj] >> 31) & 1u) << 7;
        const uint32_t nz = ((nib & 7u) ? 0x8u : 0u) | ((nib & 0x70u) ? 0x80u : 0u);
        packed[pj >> 2] |= (nib | (sgn & nz)) << (8 * (pj & 3));
      }
      *reinterpret_cast<uint2*>(cdst) = make_uint2(packed[0], packed[1]);
      scales[gi] = static_cast<uint8_t>(wcode);
      // ascending offsets + strict "<": lo + bi is the lowest offset reaching it
      if (offs) offs[gi] = static_cast<int8_t>(kFull ? wcode - b : lo + bi);
    }
  }
  cp_async_wait<0>();
}

template <bool kWeighted>
__global__ void __launch_bounds__(kCta, 5)
scale_sweep_kernel(const uint16_t* __restrict__ W, int64_t out, int64_t G, int64_t ldw,
                   const float* __restrict__ h, const float* __restrict__ Sp, int lo, int hi,
                   uint8_t* __restrict__ codes, uint8_t* __restrict__ scales,
                   int8_t* __restrict__ offs, int64_t GL, int64_t R) {
  __shared__ SweepSmem<16> sm;
  fill_candidate_table(sm.tab);
  __syncthreads();
  const int64_t tid = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  sweep_matrix<kWeighted>(sm, W, out, G, ldw, h, Sp, lo, hi, codes, scales, offs, GL, R, tid);
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
template <bool kWeighted>
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
  sweep_matrix<kWeighted>(sm, m.W, m.out, m.G, m.ldw, m.h, m.S, lo, hi, m.codes, m.scales,
                          m.offs, m.GL, m.R, tid);
}

int sweep_resident_ctas(bool weighted) {
  static const int ctas[2] = {
      resident_ctas(reinterpret_cast<const void*>(&scale_sweep_kernel<false>), kCta),
      resident_ctas(reinterpret_cast<const void*>(&scale_sweep_kernel<true>), kCta)};
  return ctas[weighted];
}

cudaError_t launch_scale_sweep_batched(const SweepDesc* d_dev, int64_t n, int64_t total_ctas,
                                       bool weighted, int lo, int hi, cudaStream_t stream) {
  if (n == 0 || total_ctas == 0) return cudaSuccess;
  if (weighted)
    scale_sweep_batched_kernel<true><<<static_cast<unsigned>(total_ctas), kCta, 0, stream>>>(
        d_dev, n, lo, hi);
  else
    scale_sweep_batched_kernel<false><<<static_cast<unsigned>(total_ctas), kCta, 0, stream>>>(
        d_dev, n, lo, hi);
  return cudaGetLastError();
}

LanePlan sweep_plan(int64_t out, int64_t in, int num_sms, bool weighted) {
  return sweep_plan_threads(out, in, static_cast<int64_t>(num_sms) * sweep_resident_ctas(weighted) * kCta);
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

cudaError_t launch_scale_sweep(const uint16_t* W, int64_t out, int64_t in, int64_t ldw,
                               const float* h, const float* S, int lo, int hi, uint8_t* codes,
                               uint8_t* scales, int8_t* offs, const LanePlan& p,
                               cudaStream_t stream) {
  if (out == 0) return cudaSuccess;
  const unsigned blocks = static_cast<unsigned>((p.threads + kCta - 1) / kCta);
  const int64_t G = in / 16;
  if (h)
    scale_sweep_kernel<true><<<blocks, kCta, 0, stream>>>(W, out, G, ldw, h, S, lo, hi, codes,
                                                          scales, offs, p.VL, p.R);
  else
    scale_sweep_kernel<false><<<blocks, kCta, 0, stream>>>(W, out, G, ldw, h, S, lo, hi, codes,
                                                           scales, offs, p.VL, p.R);
  return cudaGetLastError();
}

}  // namespace nvfp4
