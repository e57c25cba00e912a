// nvfp4_device.cuh -- device-side number-format helpers for the sm_100a
// kernels (E4M3 scale codes, E2M1 values, bf16 unpacking, streaming loads).
//
// NVFP4 (H-Scale summary, sec. 3 "NVFP4 quantization"): 16 E2M1 values share
// one E4M3 scale; a tensor-wide FP32 scale multiplies both.  E4M3 has 126
// positive finite codes 0x01..0x7E whose bit-pattern order is value order
// (ScaleSweep summary, sec. 2), so "offset k" means "k codes away".
#pragma once

#include <cstdint>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

namespace nvfp4 {

// ---------------------------------------------------------------- E4M3 codes

// Value of positive E4M3 code c (1..126) as an exact float.  Normal codes
// (c >= 8) have exponent field c>>3 and mantissa c&7, i.e. float bits
// (c << 20) + (120 << 23); subnormal codes are c * 2^-9.
__device__ __forceinline__ float e4m3_value(int c) {
  float normal = __uint_as_float((static_cast<uint32_t>(c) << 20) + 0x3C000000u);
  float sub = static_cast<float>(c) * 0x1p-9f;
  return c >= 8 ? normal : sub;
}

// Round a non-negative float to the nearest E4M3 code (ties to even code),
// saturating to 0x7E; the hardware conversion implements exactly this.
__device__ __forceinline__ int e4m3_code_rne_sat(float f) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(0.0f), "f"(f));
  return r & 0xFF;  // second source lands in the low byte
}

__device__ __forceinline__ int clamp_code(int c) { return min(max(c, 1), 126); }

// --------------------------------------------------------------- E2M1 values

// Two floats -> two E2M1 nibbles, round-to-nearest-even, saturating at 6.
// `lo` lands in bits 0..3, `hi` in bits 4..7.
__device__ __forceinline__ uint32_t e2m1x2_rne(float lo, float hi) {
  uint32_t r;
  asm("{ .reg .b8 t; cvt.rn.satfinite.e2m1x2.f32 t, %1, %2; cvt.u32.u8 %0, t; }"
      : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// Two E2M1 nibbles (bits 0..3, 4..7) -> f16x2 (low half = bits 0..3).
__device__ __forceinline__ uint32_t e2m1x2_to_f16x2(uint32_t byte) {
  uint32_t r;
  asm("{ .reg .b8 t; cvt.u8.u32 t, %1; cvt.rn.f16x2.e2m1x2 %0, t; }" : "=r"(r) : "r"(byte));
  return r;
}

// Round x >= 0 to the E2M1 grid {0,.5,1,1.5,2,3,4,6} with ties to the even
// code and saturation at 6, using only the FP pipes: on [2^e, 2^(e+1)) the grid
// step is 2^(e-1) (e >= 0) and 0.5 below 1, so adding and subtracting
// M = 2^(max(e,0)+22) rounds to that step with IEEE ties-to-even, and even
// multiples of the step are exactly the even codes.
__device__ __forceinline__ float e2m1_round(float x) {
  float m = fmaxf(__uint_as_float(__float_as_uint(x) & 0x7F800000u), 1.0f);
  float t = fmaf(m, 0x1p22f, x);
  float q = fmaf(m, -0x1p22f, t);
  return fminf(q, 6.0f);
}

// Decode an E2M1 nibble pair with the sign dropped (bits 0..2 and 4..6 used).
__device__ __forceinline__ float e2m1_nibble_value(uint32_t nib) {
  const uint32_t hh = e2m1x2_to_f16x2(nib & 7u);
  return __half2float(__ushort_as_half(static_cast<unsigned short>(hh & 0xFFFFu)));
}

// ------------------------------------------------------------ packed FP32x2
// sm_100 executes these as one instruction for two lanes of FP32 work.
typedef unsigned long long f32x2_t;
__device__ __forceinline__ f32x2_t f2_pack(float lo, float hi) {
  f32x2_t r;
  asm("mov.b64 %0, {%1,%2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void f2_unpack(f32x2_t v, float& lo, float& hi) {
  asm("mov.b64 {%0,%1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ f32x2_t f2_fma(f32x2_t a, f32x2_t b, f32x2_t c) {
  f32x2_t r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
  return r;
}
__device__ __forceinline__ f32x2_t f2_add(f32x2_t a, f32x2_t b) {
  f32x2_t r;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ f32x2_t f2_mul(f32x2_t a, f32x2_t b) {
  f32x2_t r;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}

// Round two non-negative floats to E2M1 (RNE, saturating) and decode them
// back to an f16x2 of grid values: low half <- lo, high half <- hi.
__device__ __forceinline__ uint32_t e2m1x2_round_f16x2(float lo, float hi) {
  uint32_t r;
  asm("{ .reg .b8 t; cvt.rn.satfinite.e2m1x2.f32 t, %1, %2; cvt.rn.f16x2.e2m1x2 %0, t; }"
      : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// e = c - q * v with q, v half-precision (exact product) and one rounding.
__device__ __forceinline__ float fma_f16_f32(uint16_t q, uint16_t nv, float c) {
  float r;
  asm("fma.rn.f32.f16 %0, %1, %2, %3;" : "=f"(r) : "h"(q), "h"(nv), "f"(c));
  return r;
}

// -------------------------------------------------------------------- bf16

__device__ __forceinline__ float bf16_lo(uint32_t u) { return __uint_as_float(u << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t u) { return __uint_as_float(u & 0xFFFF0000u); }

// ------------------------------------------------------------------ loads

__device__ __forceinline__ uint4 ld_stream_v4(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "l"(p));
  return r;
}

// 32 bytes in one instruction (sm_100 256-bit load); p must be 32-byte aligned.
__device__ __forceinline__ void ld_stream_v8(const void* p, uint32_t (&r)[8]) {
  asm volatile("ld.global.nc.L1::no_allocate.v8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]),
                 "=r"(r[6]), "=r"(r[7])
               : "l"(p));
}

}  // namespace nvfp4
