// dequantize.cu -- NVFP4 decode: W[r, j] = sign * fl32(g[k] * v(scale)) * S.
//
// H-Scale summary, sec. 3 "NVFP4 quantization": the effective group scale is
// the product of the FP32 global scale and the E4M3 local scale.  g * v is
// exact in FP32 (at most 6 significant bits), so the one rounding is the final
// multiply by S.  One thread per group: 9 bytes in, 64 bytes out.
#include "checks.cuh"
#include "nvfp4_kernels.cuh"

namespace nvfp4 {

__global__ void __launch_bounds__(256)
dequantize_kernel(const uint8_t* __restrict__ codes, const uint8_t* __restrict__ scales,
                  const float* __restrict__ Sp, int64_t ngroups, float* __restrict__ out) {
  const float S = *Sp;
  for (int64_t gi = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; gi < ngroups;
       gi += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const uint2 c = *checked(reinterpret_cast<const uint2*>(codes + gi * 8), codes, ngroups * 8,
                             kSiteDequantIn);
    const int sc = *checked(scales + gi, scales, ngroups, kSiteDequantIn);
    const float v = (sc == 0 || sc > 126) ? (sc == 0 ? 0.0f : __uint_as_float(0x7FC00000u))
                                          : e4m3_value(sc);
    const uint32_t w[2] = {c.x, c.y};
    float r[16];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const uint32_t byte = (w[i >> 2] >> (8 * (i & 3))) & 0xFFu;
      const uint32_t hh = e2m1x2_to_f16x2(byte);
      const float g0 = __half2float(__ushort_as_half(static_cast<unsigned short>(hh & 0xFFFFu)));
      const float g1 = __half2float(__ushort_as_half(static_cast<unsigned short>(hh >> 16)));
      r[2 * i] = (g0 * v) * S;
      r[2 * i + 1] = (g1 * v) * S;
    }
    float4* o = reinterpret_cast<float4*>(out + gi * 16);
#pragma unroll
    for (int i = 0; i < 4; ++i)
      *checked(o + i, out, ngroups * 64, kSiteDequantOut) =
          make_float4(r[4 * i], r[4 * i + 1], r[4 * i + 2], r[4 * i + 3]);
  }
}

cudaError_t launch_dequantize(const uint8_t* codes, const uint8_t* scales, const float* S,
                              int64_t out, int64_t in, float* W_out, int num_sms,
                              cudaStream_t stream) {
  const int64_t ngroups = out * (in / 16);
  if (ngroups == 0) return cudaSuccess;
  int64_t blocks = (ngroups + 255) / 256;
  const int64_t cap = static_cast<int64_t>(num_sms) * 8;
  if (blocks > cap) blocks = cap;
  dequantize_kernel<<<static_cast<unsigned>(blocks), 256, 0, stream>>>(codes, scales, S, ngroups,
                                                                       W_out);
  return cudaGetLastError();
}

}  // namespace nvfp4
