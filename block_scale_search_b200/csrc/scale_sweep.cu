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
// 32-byte group loads and 8-byte code stores are contiguous.
//
// Each group is decided in three stages:
//  1. Fast pass, FP32, all K candidates (the loop that bounds the kernel):
//       y_j = |w_j| / S            (|w_j| * p * (1/(S p)), p = 2^k for denormal S)
//       x_j = y_j * (1/v_c)        candidate-scaled weight      [FMUL2]
//       q_j = E2M1_RNE_sat(x_j)    hardware cvt to e2m1x2 and back to f16x2
//       e_j = y_j - q_j v_c        mixed f16 x f16 + f32 FMA (exact product)
//       L_c = sum_j h'_j e_j^2     [FMUL2, FFMA2]; h' = h * 2^k, max h' in [.5,1)
//     All K losses stay in registers (K <= 16).
//  2. Near-tie guard: the fast pass's error against the exact definition is
//     bounded per candidate by 2^-19 sqrt(A L) + 2^-20 L (A = sum h' y^2; the
//     terms come from the rounding of y, of each product and sum, and from
//     E2M1 decisions taken on an FP32 quotient within 2^-21.7 of the exact
//     one).  Candidates whose loss lies within four times that bound of the
//     minimum are re-scored exactly as the definition does -- exact-real
//     E2M1 decisions, d = |w| - q v S in FP64 (exact), L = sum h d^2 in FP64
//     in element order -- and the strict "<" in offset order picks among them.
//     Exact ties (octave pairs that reconstruct every element alike, symmetric
//     errors) and near-ties therefore resolve to the lowest offset exactly as
//     the definition does.  This stage runs for a small fraction of groups.
//  3. Pack with exact decisions: the FP32 quotient is bracketed by
//     (1 -+ 2^-20); where the bracket straddles an E2M1 midpoint m, the sign of
//     fma(m v, S, -|w|) (one rounding of the exact m v S - |w|) decides, zero
//     being a tie to the even code.
#include "nvfp4_kernels.cuh"

namespace nvfp4 {

// Per-code table in shared memory, indexed by code + 16 so that b + k for
// k in [-16, 15] needs no clamping (entries beyond the ends repeat codes 1/126).
struct CandEntry {
  float v;        // E4M3 value of the (clamped) code
  float iv;       // 1 / v, correctly rounded
  uint32_t nvh;   // -v as f16 bits (exact: E4M3 values are f16 values)
  uint32_t code;  // the clamped code
};
constexpr int kTabOffset = 16;
constexpr int kTabSize = 160;

__device__ __forceinline__ double exact_group_loss(const uint32_t (&wr)[8], const f32x2_t (&h2)[8],
                                                   bool weighted, float S, float v) {
  // The definition, in the definition's order: exact E2M1 decision by
  // comparison with the midpoints (each m * v * S exact in double), exact
  // error, squared, weighted, summed in element order -- no contraction.
  const double vS = __dmul_rn(static_cast<double>(v), static_cast<double>(S));
  const double mid[7] = {0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0};
  const double grid[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};
  double L = 0.0;
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    const uint32_t word = wr[j >> 1];
    const double a = fabs(static_cast<double>((j & 1) ? bf16_hi(word) : bf16_lo(word)));
    int k = 0;
    if (vS > 0.0) {
      for (int i = 0; i < 7; ++i) {
        const double t = __dmul_rn(mid[i], vS);
        if (a > t) {
          k = i + 1;
        } else {
          if (a == t) k = (i & 1) ? i + 1 : i;
          break;
        }
      }
    }
    const double d = __dsub_rn(a, __dmul_rn(grid[k], vS));
    float h0, h1;
    f2_unpack(h2[j >> 1], h0, h1);
    const double hj = weighted ? static_cast<double>((j & 1) ? h1 : h0) : 1.0;
    L = __dadd_rn(L, __dmul_rn(hj, __dmul_rn(d, d)));
  }
  return L;
}

template <bool kWeighted, bool kV8>
__global__ void __launch_bounds__(128)
scale_sweep_kernel(const uint16_t* __restrict__ W, int64_t out, int64_t G, int64_t ldw,
                   const float* __restrict__ h, const float* __restrict__ Sp, int lo, int hi,
                   uint8_t* __restrict__ codes, uint8_t* __restrict__ scales,
                   int8_t* __restrict__ offs, int64_t GL, int64_t R) {
  __shared__ CandEntry tab[kTabSize];
  for (int i = threadIdx.x; i < kTabSize; i += blockDim.x) {
    const int c = clamp_code(i - kTabOffset);
    const float v = e4m3_value(c);
    const uint32_t nvh = __half_as_ushort(__float2half_rn(-v));
    tab[i] = CandEntry{v, __frcp_rn(v), nvh | (nvh << 16), static_cast<uint32_t>(c)};
  }
  __syncthreads();

  const int64_t tid = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (tid >= R * GL) return;
  const int64_t r0 = tid / GL;
  const int64_t gl = tid - r0 * GL;
  const int K = hi - lo + 1;

  const float S = *Sp;
  const bool tiny_s = S < 0x1p-100f;         // keep 1/(S p) finite for denormal S
  const float p = tiny_s ? 0x1p100f : 1.0f;
  const float inv_sp = __frcp_rn(S * p);
  const int64_t half_in = G * 8;

  for (int64_t g = gl; g < G; g += GL) {
    f32x2_t h2[8];
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
      // exact power-of-two normalisation to max h' in [0.5, 1): the argmin is
      // invariant, and neither overflow nor underflow can distort the sums
      const uint32_t ex = __float_as_uint(hmax) & 0x7F800000u;
      float hs = 1.0f;
      if (hmax > 0.0f && ex != 0x7F800000u) {
        if (ex == 0u) hs = 0x1p100f;                       // denormal maximum
        else if (ex >= (250u << 23)) hs = 0x1p-124f;       // near FLT_MAX
        else hs = __uint_as_float(0x7E800000u - ex);       // 2^(126 - E)
      }
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        h2[2 * i] = f2_pack(hv[i].x * hs, hv[i].y * hs);
        h2[2 * i + 1] = f2_pack(hv[i].z * hs, hv[i].w * hs);
      }
    }

    for (int64_t r = r0; r < out; r += R) {
      const uint16_t* src = W + r * ldw + g * 16;
      uint32_t wr[8];
      if constexpr (kV8) {
        ld_stream_v8(src, wr);
      } else {
        const uint4 a = ld_stream_v4(src), b = ld_stream_v4(src + 8);
        wr[0] = a.x; wr[1] = a.y; wr[2] = a.z; wr[3] = a.w;
        wr[4] = b.x; wr[5] = b.y; wr[6] = b.z; wr[7] = b.w;
      }
      // group absmax on the sign-cleared bit patterns
      uint32_t mb = 0;
#pragma unroll
      for (int i = 0; i < 8; ++i) mb = __vmaxu2(mb, wr[i] & 0x7FFF7FFFu);
      mb = max(mb & 0xFFFFu, mb >> 16);
      const int64_t gi = r * G + g;
      uint8_t* cdst = codes + r * half_in + g * 8;
      if (mb == 0u) {  // all-zero group: scale 0, codes 0
        *reinterpret_cast<uint2*>(cdst) = make_uint2(0u, 0u);
        scales[gi] = 0;
        if (offs) offs[gi] = 0;
        continue;
      }
      f32x2_t y2[8];
      const f32x2_t is2 = f2_pack(inv_sp, inv_sp);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        f32x2_t a2 = f2_pack(fabsf(bf16_lo(wr[i])), fabsf(bf16_hi(wr[i])));
        if (tiny_s) a2 = f2_mul(a2, f2_pack(p, p));
        y2[i] = f2_mul(a2, is2);
      }
      f32x2_t A2 = f2_pack(0.0f, 0.0f);  // sum h' y^2, for the error bound of stage 2
#pragma unroll
      for (int i = 0; i < 8; ++i) A2 = f2_fma(f2_mul(h2[i], y2[i]), y2[i], A2);
      float A0, A1;
      f2_unpack(A2, A0, A1);
      const float A = A0 + A1;

      // base code: E4M3_RNE_sat(fl32(fl32(a / 6) / S)), clamped to [1, 126]
      const float a = __uint_as_float(mb << 16);
      const float u = __fdiv_rn(__fdiv_rn(a, 6.0f), S);
      const int b = clamp_code(e4m3_code_rne_sat(u));
      const CandEntry* ce = tab + (b + lo + kTabOffset);

      // ---- stage 1: fast FP32 losses of all candidates
      float L[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        L[i] = __uint_as_float(0x7F800000u);
        if (i < K) {
          const CandEntry t = ce[i];
          const f32x2_t iv2 = f2_pack(t.iv, t.iv);
          const uint16_t nv = static_cast<uint16_t>(t.nvh);
          f32x2_t acc = f2_pack(0.0f, 0.0f);
#pragma unroll
          for (int pj = 0; pj < 8; ++pj) {
            float x0, x1, y0, y1;
            f2_unpack(f2_mul(y2[pj], iv2), x0, x1);
            f2_unpack(y2[pj], y0, y1);
            const uint32_t qh = e2m1x2_round_f16x2(x0, x1);
            const float e0 = fma_f16_f32(static_cast<uint16_t>(qh & 0xFFFFu), nv, y0);
            const float e1 = fma_f16_f32(static_cast<uint16_t>(qh >> 16), nv, y1);
            const f32x2_t e2 = f2_pack(e0, e1);
            acc = f2_fma(f2_mul(h2[pj], e2), e2, acc);
          }
          float a0, a1;
          f2_unpack(acc, a0, a1);
          L[i] = a0 + a1;
        }
      }
      int bi = 0;
      float best = L[0];
#pragma unroll
      for (int i = 1; i < 16; ++i)
        if (L[i] < best) { best = L[i]; bi = i; }

      // ---- stage 2: near-tie guard and exact re-scoring
      const uint32_t bcode = ce[bi].code;
      uint32_t tied = 0;
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        if (i < K && i != bi && ce[i].code != bcode) {
          const float bound = 0x1p-15f * sqrtf(A * L[i]) + 0x1p-16f * L[i];
          if (L[i] <= best + bound) tied |= 1u << i;
        }
      }
      if (tied) {
        tied |= 1u << bi;
        double bestd = __longlong_as_double(0x7FF0000000000000ll);
        int bid = bi;
        for (int i = 0; i < K; ++i) {
          if (!((tied >> i) & 1u)) continue;
          const double Ld = exact_group_loss(wr, h2, kWeighted, S, ce[i].v);
          if (Ld < bestd) { bestd = Ld; bid = i; }
        }
        bi = bid;
      }
      const CandEntry win = ce[bi];

      // ---- stage 3: quantize once with the winner, exact decisions, pack
      const float vb = win.v;
      const f32x2_t ivlo = f2_pack(win.iv * (1.0f - 0x1p-20f), win.iv * (1.0f - 0x1p-20f));
      uint32_t packed[2] = {0u, 0u};
#pragma unroll
      for (int pj = 0; pj < 8; ++pj) {
        float xl0, xl1;
        f2_unpack(f2_mul(y2[pj], ivlo), xl0, xl1);
        const float xh0 = xl0 * (1.0f + 0x1p-19f), xh1 = xl1 * (1.0f + 0x1p-19f);
        uint32_t nlo = e2m1x2_rne(xl0, xl1);
        const uint32_t nhi = e2m1x2_rne(xh0, xh1);
        if (nlo != nhi) {  // rare: a quotient within 2^-20 of a midpoint
#pragma unroll
          for (int t = 0; t < 2; ++t) {
            const uint32_t kl = (nlo >> (4 * t)) & 7u, kh = (nhi >> (4 * t)) & 7u;
            if (kl != kh) {
              const float ql = e2m1_nibble_value(kl), qh = e2m1_nibble_value(kh);
              const float m = 0.5f * (ql + qh);                    // exact midpoint
              const uint32_t word = wr[pj];
              const float aj = fabsf(t ? bf16_hi(word) : bf16_lo(word));
              const float rr = fmaf(m * vb, S, -aj);               // sign(m v S - |w|)
              const uint32_t k = (rr < 0.0f) ? kh : (rr > 0.0f ? kl : ((kl & 1u) ? kh : kl));
              nlo = (nlo & ~(7u << (4 * t))) | (k << (4 * t));
            }
          }
        }
        // signs: bf16 bit 15 (low element) and bit 31 (high element)
        const uint32_t sgn = ((wr[pj] >> 15) & 1u) << 3 | ((wr[pj] >> 31) & 1u) << 7;
        const uint32_t nz = ((nlo & 7u) ? 0x8u : 0u) | ((nlo & 0x70u) ? 0x80u : 0u);
        packed[pj >> 2] |= ((nlo & 0x77u) | (sgn & nz)) << (8 * (pj & 3));
      }
      *reinterpret_cast<uint2*>(cdst) = make_uint2(packed[0], packed[1]);
      scales[gi] = static_cast<uint8_t>(win.code);
      // ascending offsets + strict "<": lo + bi is the lowest offset reaching it
      if (offs) offs[gi] = static_cast<int8_t>(lo + bi);
    }
  }
}

LanePlan sweep_plan(int64_t out, int64_t in, int num_sms, bool weighted, bool v8) {
  static const int ctas[2][2] = {
      {resident_ctas(reinterpret_cast<const void*>(&scale_sweep_kernel<false, false>), 128),
       resident_ctas(reinterpret_cast<const void*>(&scale_sweep_kernel<false, true>), 128)},
      {resident_ctas(reinterpret_cast<const void*>(&scale_sweep_kernel<true, false>), 128),
       resident_ctas(reinterpret_cast<const void*>(&scale_sweep_kernel<true, true>), 128)}};
  LanePlan p;
  p.V = in / 16;  // column groups per row
  const int64_t nt = static_cast<int64_t>(num_sms) * ctas[weighted][v8] * 128;
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
                               uint8_t* scales, int8_t* offs, bool v8, const LanePlan& p,
                               cudaStream_t stream) {
  if (out == 0) return cudaSuccess;
  const unsigned blocks = static_cast<unsigned>((p.threads + 127) / 128);
  const int64_t G = in / 16;
#define NVFP4_SWEEP_LAUNCH(WT, V8)                                                          \
  scale_sweep_kernel<WT, V8><<<blocks, 128, 0, stream>>>(W, out, G, ldw, h, S, lo, hi,     \
                                                         codes, scales, offs, p.VL, p.R)
  if (h) {
    if (v8) NVFP4_SWEEP_LAUNCH(true, true); else NVFP4_SWEEP_LAUNCH(true, false);
  } else {
    if (v8) NVFP4_SWEEP_LAUNCH(false, true); else NVFP4_SWEEP_LAUNCH(false, false);
  }
#undef NVFP4_SWEEP_LAUNCH
  return cudaGetLastError();
}

}  // namespace nvfp4
