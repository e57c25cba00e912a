// nvfp4_kernels.cuh -- internal launch interface between the C ABI
// (nvfp4hs_capi.cu) and the kernels.  Not part of the public API.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

#include "nvfp4_device.cuh"

namespace nvfp4 {

// Grids are sized to exactly one wave: SMs x resident CTAs per SM (from the
// occupancy calculator for the compiled kernel) x CTA size.  Resident-CTA
// counts are properties of the binary, so plans (and workspace sizes) are
// deterministic for a given device.
int resident_ctas(const void* kernel, int threads_per_cta);

// A lane grid: R row-lanes x VL column-lanes over V column units per row.
struct LanePlan {
  int64_t V = 0, VL = 1, R = 1, threads = 1;
};

LanePlan diag_hessian_plan(int64_t tokens, int64_t in, int num_sms);
size_t diag_hessian_workspace_bytes(const LanePlan& p, int64_t in);
cudaError_t launch_diag_hessian(const uint16_t* X, int64_t T, int64_t in, int64_t ldx, float* h,
                                int accumulate, float* partials, const LanePlan& p,
                                cudaStream_t stream);

LanePlan global_scale_plan(int64_t out, int64_t in, int num_sms);
size_t global_scale_workspace_bytes(const LanePlan& p);
cudaError_t launch_global_scale(const uint16_t* W, int64_t out, int64_t ldw, float q_max,
                                float* S, float* amax, int* status, uint32_t* partial,
                                const LanePlan& p, cudaStream_t stream);

LanePlan sweep_plan(int64_t out, int64_t in, int num_sms, bool weighted);
cudaError_t launch_scale_sweep(const uint16_t* W, int64_t out, int64_t in, int64_t ldw,
                               const float* h, const float* S, int lo, int hi, uint8_t* codes,
                               uint8_t* scales, int8_t* offs, const LanePlan& p,
                               cudaStream_t stream);

cudaError_t launch_dequantize(const uint8_t* codes, const uint8_t* scales, const float* S,
                              int64_t out, int64_t in, float* W_out, int num_sms,
                              cudaStream_t stream);

}  // namespace nvfp4
