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
// address is looked up with cudaGetSymbolAddress, once per device, on the
// first call made while that device is current.  All calls share the one
// array: calls whose work overlaps on the GPU (different streams, no ordering)
// race on it.  Nothing in it has to start at zero -- every launch writes each
// slot that it later reads -- so nothing is cleared.
#include "nvfp4hs.h"

#include <cmath>
#include <mutex>

#include "nvfp4_kernels.cuh"

namespace {

constexpr size_t kNoAllocScratchBytes = 64 * 1024;
constexpr int kMaxDevices = 128;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_setup_mutex;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of the scratch array on the current device (set up once per
// device); nullptr with *err set if the lookup fails.
void* scratch_on_current_device(cudaError_t* err) {
  int dev = 0;
  *err = cudaGetDevice(&dev);
  if (*err != cudaSuccess) return nullptr;
  if (dev < 0 || dev >= kMaxDevices) {
    *err = cudaErrorInvalidDevice;
    return nullptr;
  }
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  if (g_scratch_addr[dev] == nullptr) {
    void* p = nullptr;
    *err = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (*err != cudaSuccess) return nullptr;
    g_scratch_addr[dev] = p;
  }
  *err = cudaSuccess;
  return g_scratch_addr[dev];
}

int current_sms() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  return n;
}

bool is_aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

}  // namespace

extern "C" int nvfp4_global_scale_noalloc(const void* W, int64_t out, int64_t in, int64_t ldw,
                                          float q_max, float* S, float* amax, int* status,
                                          void* stream) {
  // the same argument checks as nvfp4_global_scale, before any CUDA call
  if (out < 0 || in < 0) return NVFP4_ERR_INVALID_ARG;
  if (W == nullptr && out > 0 && in > 0) return NVFP4_ERR_INVALID_ARG;
  if (in % 8 != 0 || ldw < in || out > (int64_t{1} << 40) || in > (int64_t{1} << 40) ||
      ldw > (int64_t{1} << 40))
    return NVFP4_ERR_SHAPE;
  if (!is_aligned(W, 16) || ldw % 8 != 0) return NVFP4_ERR_ALIGN;
  if (S == nullptr || !std::isfinite(q_max) || !(q_max > 0.0f)) return NVFP4_ERR_INVALID_ARG;
  if (!is_aligned(S, 4) || !is_aligned(amax, 4) || !is_aligned(status, 4)) return NVFP4_ERR_ALIGN;

  const int sms = current_sms();
  if (sms <= 0) {
    cudaGetLastError();
    return NVFP4_ERR_CUDA;
  }
  const nvfp4::LanePlan p = nvfp4::global_scale_plan(out, in, sms);
  if (nvfp4::global_scale_workspace_bytes(p) > kNoAllocScratchBytes) return NVFP4_ERR_WORKSPACE;
  cudaError_t err = cudaSuccess;
  void* scratch = scratch_on_current_device(&err);
  if (scratch == nullptr) return NVFP4_ERR_CUDA;
  const cudaError_t e = nvfp4::launch_global_scale(
      static_cast<const uint16_t*>(W), out, ldw, q_max, S, amax, status,
      static_cast<uint32_t*>(scratch), p, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? NVFP4_OK : NVFP4_ERR_CUDA;
}
