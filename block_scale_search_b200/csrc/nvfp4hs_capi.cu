// nvfp4hs_capi.cu -- the extern "C" entry points declared in include/nvfp4hs.h.
//
// Every entry point validates its arguments on the host, before any CUDA call,
// and returns a negative nvfp4_status on failure with nothing enqueued.  Only
// then does it look up the current device's SM count (cached) to size the grid
// and launch.  No C++ exception crosses this boundary.
#include "nvfp4hs.h"

#include <atomic>
#include <cmath>
#include <cstdint>

#include "nvfp4_kernels.cuh"

namespace {

constexpr int64_t kMaxDim = int64_t{1} << 40;  // guards index arithmetic
thread_local int g_last_cuda_error = 0;

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

int cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return NVFP4_OK;
  g_last_cuda_error = static_cast<int>(e);
  return NVFP4_ERR_CUDA;
}

// SM count of the current device, cached per device ordinal (0 on failure).
int current_sm_count() {
  static std::atomic<int> cache[128];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) {
    cudaGetLastError();
    return 0;
  }
  if (dev < 128) {
    const int c = cache[dev].load(std::memory_order_relaxed);
    if (c > 0) return c;
  }
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  if (dev < 128) cache[dev].store(n, std::memory_order_relaxed);
  return n;
}

int check_diag_hessian(const void* X, int64_t tokens, int64_t in, int64_t ldx, const float* h,
                       int accumulate) {
  if (h == nullptr || (X == nullptr && tokens > 0)) return NVFP4_ERR_INVALID_ARG;
  if (tokens < 0 || in <= 0 || (accumulate != 0 && accumulate != 1)) return NVFP4_ERR_INVALID_ARG;
  if (in % 8 != 0 || ldx < in || in > kMaxDim || tokens > kMaxDim || ldx > kMaxDim)
    return NVFP4_ERR_SHAPE;
  if (!aligned(X, 16) || ldx % 8 != 0 || !aligned(h, 4)) return NVFP4_ERR_ALIGN;
  return NVFP4_OK;
}

int check_matrix(const void* W, int64_t out, int64_t in, int64_t ldw, int64_t in_multiple) {
  if (out < 0 || in < 0) return NVFP4_ERR_INVALID_ARG;
  if (W == nullptr && out > 0 && in > 0) return NVFP4_ERR_INVALID_ARG;
  if (in % in_multiple != 0 || ldw < in || out > kMaxDim || in > kMaxDim || ldw > kMaxDim)
    return NVFP4_ERR_SHAPE;
  if (!aligned(W, 16) || ldw % 8 != 0) return NVFP4_ERR_ALIGN;
  return NVFP4_OK;
}

}  // namespace

namespace nvfp4 {
int resident_ctas(const void* kernel, int threads_per_cta) {
  int n = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kernel, threads_per_cta, 0) != cudaSuccess) {
    cudaGetLastError();
    n = 0;
  }
  return n > 0 ? n : 1;
}
}  // namespace nvfp4

extern "C" {

int nvfp4_version(void) { return 100; }  // 0.1.0

int nvfp4_last_cuda_error(void) { return g_last_cuda_error; }

size_t nvfp4_diag_hessian_workspace_size(int64_t tokens, int64_t in) {
  if (tokens < 0 || in <= 0 || in % 8 != 0 || in > kMaxDim) return 0;
  const int sms = current_sm_count();
  if (sms <= 0) return 0;
  const nvfp4::LanePlan p = nvfp4::diag_hessian_plan(tokens, in, sms);
  return nvfp4::diag_hessian_workspace_bytes(p, in);
}

int nvfp4_diag_hessian(const void* X, int64_t tokens, int64_t in, int64_t ldx, float* h,
                       int accumulate, void* workspace, size_t workspace_bytes, void* stream) {
  int st = check_diag_hessian(X, tokens, in, ldx, h, accumulate);
  if (st != NVFP4_OK) return st;
  if (workspace == nullptr) return NVFP4_ERR_WORKSPACE;
  if (!aligned(workspace, 16)) return NVFP4_ERR_ALIGN;
  const int sms = current_sm_count();
  if (sms <= 0) return cuda_status(cudaErrorNoDevice);
  const nvfp4::LanePlan p = nvfp4::diag_hessian_plan(tokens, in, sms);
  if (workspace_bytes < nvfp4::diag_hessian_workspace_bytes(p, in)) return NVFP4_ERR_WORKSPACE;
  return cuda_status(nvfp4::launch_diag_hessian(static_cast<const uint16_t*>(X), tokens, in, ldx,
                                                h, accumulate, static_cast<float*>(workspace), p,
                                                static_cast<cudaStream_t>(stream)));
}

size_t nvfp4_global_scale_workspace_size(int64_t out, int64_t in) {
  if (out < 0 || in < 0 || in % 8 != 0 || in > kMaxDim || out > kMaxDim) return 0;
  const int sms = current_sm_count();
  if (sms <= 0) return 0;
  return nvfp4::global_scale_workspace_bytes(nvfp4::global_scale_plan(out, in, sms));
}

int nvfp4_global_scale(const void* W, int64_t out, int64_t in, int64_t ldw, float q_max,
                       float* S, float* amax, int* status, void* workspace,
                       size_t workspace_bytes, void* stream) {
  int st = check_matrix(W, out, in, ldw, 8);
  if (st != NVFP4_OK) return st;
  if (S == nullptr || !std::isfinite(q_max) || !(q_max > 0.0f)) return NVFP4_ERR_INVALID_ARG;
  if (!aligned(S, 4) || !aligned(amax, 4) || !aligned(status, 4)) return NVFP4_ERR_ALIGN;
  if (workspace == nullptr) return NVFP4_ERR_WORKSPACE;
  if (!aligned(workspace, 16)) return NVFP4_ERR_ALIGN;
  const int sms = current_sm_count();
  if (sms <= 0) return cuda_status(cudaErrorNoDevice);
  const nvfp4::LanePlan p = nvfp4::global_scale_plan(out, in, sms);
  if (workspace_bytes < nvfp4::global_scale_workspace_bytes(p)) return NVFP4_ERR_WORKSPACE;
  return cuda_status(nvfp4::launch_global_scale(static_cast<const uint16_t*>(W), out, ldw, q_max,
                                                S, amax, status,
                                                static_cast<uint32_t*>(workspace), p,
                                                static_cast<cudaStream_t>(stream)));
}

int nvfp4_scale_sweep_quantize(const void* W, int64_t out, int64_t in, int64_t ldw,
                               const float* h, const float* S, int lo, int hi,
                               uint8_t* codes, uint8_t* scales, int8_t* chosen_offset,
                               void* stream) {
  int st = check_matrix(W, out, in, ldw, 16);
  if (st != NVFP4_OK) return st;
  const bool empty = out == 0 || in == 0;
  if (!empty && (S == nullptr || codes == nullptr || scales == nullptr))
    return NVFP4_ERR_INVALID_ARG;
  if (lo < -16 || lo > 0 || hi < 0 || hi > 15 || hi - lo > 15) return NVFP4_ERR_WINDOW;
  if (!aligned(h, 16) || !aligned(S, 4) || !aligned(codes, 8)) return NVFP4_ERR_ALIGN;
  if (empty) return NVFP4_OK;
  const int sms = current_sm_count();
  if (sms <= 0) return cuda_status(cudaErrorNoDevice);
  const nvfp4::LanePlan p = nvfp4::sweep_plan(out, in, sms, h != nullptr);
  return cuda_status(nvfp4::launch_scale_sweep(static_cast<const uint16_t*>(W), out, in, ldw, h,
                                               S, lo, hi, codes, scales, chosen_offset, p,
                                               static_cast<cudaStream_t>(stream)));
}

int nvfp4_dequantize(const uint8_t* codes, const uint8_t* scales, const float* S, int64_t out,
                     int64_t in, float* W_out, void* stream) {
  if (out < 0 || in < 0) return NVFP4_ERR_INVALID_ARG;
  if (in % 16 != 0 || out > kMaxDim || in > kMaxDim) return NVFP4_ERR_SHAPE;
  if (out == 0 || in == 0) return NVFP4_OK;
  if (codes == nullptr || scales == nullptr || S == nullptr || W_out == nullptr)
    return NVFP4_ERR_INVALID_ARG;
  if (!aligned(codes, 8) || !aligned(S, 4) || !aligned(W_out, 16)) return NVFP4_ERR_ALIGN;
  const int sms = current_sm_count();
  if (sms <= 0) return cuda_status(cudaErrorNoDevice);
  return cuda_status(nvfp4::launch_dequantize(codes, scales, S, out, in, W_out, sms,
                                              static_cast<cudaStream_t>(stream)));
}

}  // extern "C"
