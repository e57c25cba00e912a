// global_scale_noalloc.cu -- the global-scale step for callers that cannot
// allocate device memory.
//
// Some callers cannot call cudaMalloc: plugin or custom-op hooks that are
// handed tensors but no allocator, processes working under a hard device-memory
// cap or inside a memory pool planned in advance, where an extra allocation can
// fail or fragment the pool.  nvfp4_global_scale needs a small scratch buffer
// (one partial maximum per CTA of the first kernel); this entry point takes it
// from a fixed array compiled into the library instead.  The array is
// kNoAllocScratchBytes (64 KiB), held on every GPU that loads the library until
// the process exits; a problem whose partials would not fit is rejected.
//
// The array's name in host code is only a host-side stand-in, so its device
// address comes from cudaGetSymbolAddress, with the caller's device current.
// The lookup is repeated on every call (it is a cheap host call): a cached
// address would belong to the context it was taken in and would go stale after
// cudaDeviceReset or under another context on the same device.  The first call
// on a device also makes the runtime load this library's device code there, so
// it should come before any stream capture.  All calls share the one array:
// calls whose work overlaps on the GPU (different streams, no ordering) race on
// it.  Nothing in it has to start at zero -- every launch writes each slot that
// it later reads -- so nothing is cleared.
#include "nvfp4hs.h"

#include <cmath>

#include "nvfp4_kernels.cuh"
#include "nvtx_range.cuh"

namespace {

constexpr size_t kNoAllocScratchBytes = 64 * 1024;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

// Device address of the scratch array in the current context; nullptr with
// *err set on failure (the runtime's last-error state is then cleared, so a
// later call does not see this one's error).
void* scratch_on_current_device(cudaError_t* err) {
  void* p = nullptr;
  *err = cudaGetSymbolAddress(&p, g_noalloc_scratch);
  if (*err != cudaSuccess) {
    cudaGetLastError();
    return nullptr;
  }
  return p;
}

// SM count of the current device; 0 with *err set on failure.
int current_sms(cudaError_t* err) {
  int dev = 0, n = 0;
  *err = cudaGetDevice(&dev);
  if (*err == cudaSuccess) *err = cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  if (*err != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  return n;
}

bool is_aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

}  // namespace

extern "C" int nvfp4_global_scale_noalloc(const void* W, int64_t out, int64_t in, int64_t ldw,
                                          float q_max, float* S, float* amax, int* status,
                                          void* stream) {
  NVFP4_RANGE("nvfp4_global_scale_noalloc");
  // the same argument checks as nvfp4_global_scale, before any CUDA call
  if (out < 0 || in < 0) return NVFP4_ERR_INVALID_ARG;
  if (W == nullptr && out > 0 && in > 0) return NVFP4_ERR_INVALID_ARG;
  if (in % 8 != 0 || ldw < in || out > (int64_t{1} << 40) || in > (int64_t{1} << 40) ||
      ldw > (int64_t{1} << 40))
    return NVFP4_ERR_SHAPE;
  if (!is_aligned(W, 16) || ldw % 8 != 0) return NVFP4_ERR_ALIGN;
  if (S == nullptr || !std::isfinite(q_max) || !(q_max > 0.0f)) return NVFP4_ERR_INVALID_ARG;
  if (!is_aligned(S, 4) || !is_aligned(amax, 4) || !is_aligned(status, 4)) return NVFP4_ERR_ALIGN;

  cudaError_t err = cudaSuccess;
  const int sms = current_sms(&err);
  if (sms <= 0) return nvfp4::record_cuda_status(err == cudaSuccess ? cudaErrorNoDevice : err);
  const nvfp4::LanePlan p = nvfp4::global_scale_plan(out, in, sms);
  if (nvfp4::global_scale_workspace_bytes(p) > kNoAllocScratchBytes) return NVFP4_ERR_WORKSPACE;
  void* scratch = scratch_on_current_device(&err);
  if (scratch == nullptr) return nvfp4::record_cuda_status(err);
  return nvfp4::record_cuda_status(nvfp4::launch_global_scale(
      static_cast<const uint16_t*>(W), out, ldw, q_max, S, amax, status,
      static_cast<uint32_t*>(scratch), p, static_cast<cudaStream_t>(stream)));
}
