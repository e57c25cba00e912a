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
// One thread owns one group at a time: its 16 weights and 16 h_j live in
// registers, each candidate is evaluated in FP32 and the running argmin is kept
// with a strict "<" in ascending offset order (ties to the lowest offset).
// Lanes: GL column-group lanes x R row lanes; lane (r, gl) handles column
// groups gl, gl+GL, ... (h loaded once per column group) and rows r, r+R, ...
// Adjacent threads own adjacent groups of one row, so the 32-byte group loads
// and 8-byte code stores of a warp are contiguous.
//
// Numerics (all decisions match the exact definition up to FP32 rounding of
// the scaled weight; see the header):
//   y_j = |w_j| / S            (computed as |w_j| * p * (1/(S*p)), p = 2^k
//                              keeps 1/(S p) finite for denormal S)
//   x_j = y_j * (1/v_c)         the weight in units of the candidate scale
//   q_j = E2M1_RNE_sat(x_j)     exact IEEE rounding of x_j
//   e_j = y_j - q_j * v_c       exact (FFMA); identical reconstructions at two
//                              candidates give bit-identical errors, so exact
//                              ties stay ties and go to the lowest offset
//   L_c = sum_j h'_j e_j^2      h' = h * 2^-k (exact), max h' in [0.5, 1)
#include "nvfp4_kernels.cuh"

namespace nvfp4 {

template <bool kWeighted, bool kV8>
__global__ void __launch_bounds__(128)
scale_sweep_kernel(const uint16_t* __restrict__ W, int64_t out, int64_t G, int64_t ldw,
                   const float* __restrict__ h, const float* __restrict__ Sp, int lo, int hi,
                   uint8_t* __restrict__ codes, uint8_t* __restrict__ scales,
                   int8_t* __restrict__ offs, int64_t GL, int64_t R) {
  const int64_t tid = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (tid >= R * GL) return;
  const int64_t r0 = tid / GL;
  const int64_t gl = tid - r0 * GL;

  const float S = *Sp;
  // Power-of-two pre-scale so that 1/(S*p) is finite and normal.
  const float p = (S < 0x1p-100f) ? 0x1p100f : 1.0f;
  const float inv_sp = __frcp_rn(S * p);
  const int64_t half_in = G * 8;

  for (int64_t g = gl; g < G; g += GL) {
    float hw[16];
    if constexpr (kWeighted) {
      const float4* hp = reinterpret_cast<const float4*>(h + g * 16);
      float hmax = 0.0f;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float4 t = hp[i];
        hw[4 * i + 0] = t.x; hw[4 * i + 1] = t.y; hw[4 * i + 2] = t.z; hw[4 * i + 3] = t.w;
      }
#pragma unroll
      for (int j = 0; j < 16; ++j) hmax = fmaxf(hmax, hw[j]);
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
      for (int j = 0; j < 16; ++j) hw[j] *= hs;
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
      if (mb == 0u) {  // all-zero group: scale 0, codes 0
        *reinterpret_cast<uint2*>(codes + r * half_in + g * 8) = make_uint2(0u, 0u);
        scales[gi] = 0;
        if (offs) offs[gi] = 0;
        continue;
      }
      float y[16];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        y[2 * i] = (fabsf(bf16_lo(wr[i])) * p) * inv_sp;
        y[2 * i + 1] = (fabsf(bf16_hi(wr[i])) * p) * inv_sp;
      }
      // base code: E4M3_RNE_sat(fl32(fl32(a / 6) / S)), clamped to [1, 126]
      const float a = __uint_as_float(mb << 16);
      const float u = __fdiv_rn(__fdiv_rn(a, 6.0f), S);
      const int b = clamp_code(e4m3_code_rne_sat(u));

      float best = __uint_as_float(0x7F800000u);
      int bc = b, bk = lo;
      for (int k = lo; k <= hi; ++k) {
        const int c = clamp_code(b + k);
        const float v = e4m3_value(c);
        const float iv = __frcp_rn(v);
        float acc = 0.0f;
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const float q = e2m1_round(y[j] * iv);
          const float e = fmaf(-q, v, y[j]);
          if constexpr (kWeighted) acc = fmaf(hw[j] * e, e, acc);
          else acc = fmaf(e, e, acc);
        }
        if (acc < best) { best = acc; bc = c; bk = k; }
      }
      // quantize once with the winner and pack (element 2i -> low nibble)
      const float iv = __frcp_rn(e4m3_value(bc));
      uint32_t packed[2] = {0u, 0u};
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float x0 = copysignf(y[2 * i] * iv, bf16_lo(wr[i]));
        const float x1 = copysignf(y[2 * i + 1] * iv, bf16_hi(wr[i]));
        packed[i >> 2] |= e2m1x2_rne(x0, x1) << (8 * (i & 3));
      }
#pragma unroll
      for (int i = 0; i < 2; ++i) {  // a zero magnitude is stored as +0
        const uint32_t w = packed[i];
        const uint32_t nz = (w | (w >> 1) | (w >> 2)) & 0x11111111u;
        packed[i] = w & (0x77777777u | (nz << 3));
      }
      *reinterpret_cast<uint2*>(codes + r * half_in + g * 8) = make_uint2(packed[0], packed[1]);
      scales[gi] = static_cast<uint8_t>(bc);
      // ascending offsets + strict "<": bk is the lowest offset reaching bc
      if (offs) offs[gi] = static_cast<int8_t>(bk);
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
