// checks.cuh -- bounds checks of the checked build (-DNVFP4HS_CHECKS).
//
// In the checked build every global-memory access of the per-step kernels
// (diagonal Hessian, global scale, sweep, dequantize) goes through checked():
// an address outside the buffer's extent -- the extent the kernel's own size
// arguments imply -- is counted, the first one is kept (site and byte
// offset), and the access is redirected to a small dummy buffer instead, so
// the kernel goes on without touching memory it does not own and without a
// fault.  nvfp4_debug_checks() reads (and can clear) the record.  In the
// normal build checked() returns its pointer unchanged and nothing is kept.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

namespace nvfp4 {

// Where a failed check happened (the top 16 bits of the first record).
enum CheckSite : int {
  kSiteDiagX = 1, kSiteDiagPartial, kSiteDiagH,
  kSiteAbsmaxW, kSiteAbsmaxPartial,
  kSiteSweepW, kSiteSweepH, kSiteSweepCodes, kSiteSweepScales, kSiteSweepOffs,
  kSiteDequantIn, kSiteDequantOut,
};

struct CheckState {
  unsigned long long first;  // (site << 48) | byte offset of the first failure (+1), 0: none
  unsigned int count;        // failed checks
  unsigned int pad;
};

// Sums and clears the records of every translation unit built with checks
// (nvfp4hs_capi.cu keeps the list); false in the normal build.
bool checks_compiled();
cudaError_t collect_checks(CheckState* out, bool reset);
int register_check_reader(cudaError_t (*reader)(CheckState*, bool));

#ifdef NVFP4HS_CHECKS
namespace {
__device__ CheckState g_check_state;
__device__ __align__(64) unsigned char g_check_dummy[64];

cudaError_t read_checks_here(CheckState* out, bool reset) {
  CheckState s{};
  cudaError_t e = cudaMemcpyFromSymbol(&s, g_check_state, sizeof(s));
  if (e != cudaSuccess) return e;
  out->count += s.count;
  if (out->first == 0) out->first = s.first;
  if (reset) {
    const CheckState z{};
    e = cudaMemcpyToSymbol(g_check_state, &z, sizeof(z));
  }
  return e;
}
const int g_check_reader_registered = register_check_reader(&read_checks_here);
}  // namespace

template <typename T>
__device__ __forceinline__ T* checked(T* p, const void* base, int64_t bytes, int site) {
  const int64_t off = reinterpret_cast<const char*>(p) - reinterpret_cast<const char*>(base);
  if (off >= 0 && off + static_cast<int64_t>(sizeof(T)) <= bytes) return p;
  atomicAdd(&g_check_state.count, 1u);
  atomicCAS(&g_check_state.first, 0ull,
            (static_cast<unsigned long long>(site) << 48) |
                (static_cast<unsigned long long>(off + 1) & 0xFFFFFFFFFFFFull));
  return reinterpret_cast<T*>(g_check_dummy);
}
#else
template <typename T>
__device__ __forceinline__ T* checked(T* p, const void*, int64_t, int) {
  return p;
}
#endif

// Extent in bytes of a row-major [rows, cols] matrix of `elem`-byte elements
// with leading dimension ld (0 for an empty one).
__host__ __device__ __forceinline__ int64_t extent_bytes(int64_t rows, int64_t cols, int64_t ld,
                                                         int64_t elem) {
  return rows > 0 && cols > 0 ? ((rows - 1) * ld + cols) * elem : 0;
}

}  // namespace nvfp4
