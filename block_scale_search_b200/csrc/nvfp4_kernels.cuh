// nvfp4_kernels.cuh -- internal launch interface between the C ABI
// (nvfp4hs_capi.cu) and the kernels.  Not part of the public API.
#pragma once

#include <cstddef>
#include <cstdint>
#include <vector>
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
size_t diag_hessian_grouped_workspace_bytes(int64_t total, int64_t experts, int64_t in,
                                            int num_sms);
cudaError_t launch_diag_hessian_grouped(const uint16_t* X, const int64_t* row_offsets, int64_t E,
                                        int64_t total, int64_t in, int64_t ldx, float* h,
                                        int accumulate, void* workspace, int num_sms,
                                        cudaStream_t stream);
// The grouped kernel's plan (slices of expert-contiguous rows, planned on
// the device) and partials in its workspace, for streaming its partial pass
// from another launch (side_reduce.cuh, kind 2).
struct GroupedSide {
  int64_t* cstart;  // [E + 2]: first slice of each expert, slices, rows per slice
  float* P;         // [cap, in] partials
  int64_t cap, nt;  // slices at most; the plan's target slice count
  int block;        // the partial kernel's CTA size (row lanes x vectors)
};
GroupedSide grouped_diag_side(int64_t E, int64_t in, void* workspace, int num_sms);
cudaError_t launch_grouped_diag_plan(const int64_t* off, int64_t E, int64_t total,
                                     const GroupedSide& g, cudaStream_t stream);
cudaError_t launch_grouped_diag_finalize(int64_t E, int64_t in, float* h, int accumulate,
                                         const GroupedSide& g, cudaStream_t stream);
size_t diag_hessian_workspace_bytes(const LanePlan& p, int64_t in);
cudaError_t launch_diag_hessian(const uint16_t* X, int64_t T, int64_t in, int64_t ldx, float* h,
                                int accumulate, float* partials, const LanePlan& p,
                                cudaStream_t stream);
// The second pass alone: h[j] (+)= sum over the `rows` partial rows, in order.
cudaError_t launch_diag_hessian_finalize(const float* partials, int64_t rows, int64_t in, float* h,
                                         int accumulate, cudaStream_t stream);

LanePlan global_scale_plan(int64_t out, int64_t in, int num_sms);
int absmax_resident_ctas();

// One matrix of a batched global scale, as the kernel reads it.
struct MatDesc {
  const uint16_t* W;
  int64_t out, ldw;
  int64_t V, VL, R;   // lane plan over 8-element vectors
  int64_t cta_begin;  // first CTA of this matrix
};
cudaError_t launch_global_scale_batched(const MatDesc* d_dev, int64_t n, int64_t total_ctas,
                                        float q_max, float* S, float* amax, int* status,
                                        uint32_t* partial, cudaStream_t stream);
size_t global_scale_workspace_bytes(const LanePlan& p);
cudaError_t launch_global_scale(const uint16_t* W, int64_t out, int64_t ldw, float q_max,
                                float* S, float* amax, int* status, uint32_t* partial,
                                const LanePlan& p, cudaStream_t stream);
// S (and amax, status) from n partial maxima of sign-cleared bf16 patterns.
cudaError_t launch_global_scale_finalize(const uint32_t* partial, int n, float q_max, float* S,
                                         float* amax, int* status, cudaStream_t stream);

LanePlan sweep_plan(int64_t out, int64_t in, int num_sms, bool weighted, int K);
LanePlan sweep_plan_threads(int64_t out, int64_t in, int64_t threads);
int sweep_resident_ctas(bool weighted);
int sweep_resident_ctas(bool weighted, int K);
constexpr int kSweepCta = 128;

// One matrix of a batched sweep, as the kernel reads it from device memory.
struct SweepDesc {
  const uint16_t* W;
  const float* h;
  const float* S;
  uint8_t* codes;
  uint8_t* scales;
  int8_t* offs;
  int64_t out, G, ldw, GL, R;
  int64_t cta_begin;  // first CTA of this matrix; CTAs up to the next matrix's
};
cudaError_t launch_scale_sweep_full(const uint16_t* W, int64_t out, int64_t in, int64_t ldw,
                                    const float* h, const float* S, uint8_t* codes,
                                    uint8_t* scales, int8_t* offs, int num_sms,
                                    cudaStream_t stream);
cudaError_t launch_scale_sweep_batched(const SweepDesc* d_dev, int64_t n, int64_t total_ctas,
                                       bool weighted, int lo, int hi, cudaStream_t stream);
// A sweep that streams side reductions (side_reduce.cuh) with a fifth warp
// per CTA.  Only shapes that hand rows out at run time qualify
// (sweep_can_carry); *carried says whether it was launched that way -- if
// not, nothing was launched and the caller sweeps and reduces by itself.
struct SideWork;
bool sweep_can_carry(int64_t out, int64_t in, int num_sms);
cudaError_t launch_scale_sweep_side(const uint16_t* W, int64_t out, int64_t in, int64_t ldw,
                                    const float* h, const float* S, int lo, int hi,
                                    uint8_t* codes, uint8_t* scales, int8_t* offs,
                                    const SideWork& side, int num_sms, bool* carried,
                                    cudaStream_t stream);
// The batched sweep with a streaming fifth warp per CTA (4 CTAs per SM).
cudaError_t launch_scale_sweep_batched_side(const SweepDesc* d_dev, int64_t n, int64_t total_ctas,
                                            bool weighted, int lo, int hi, const SideWork& side,
                                            cudaStream_t stream);
cudaError_t launch_scale_sweep(const uint16_t* W, int64_t out, int64_t in, int64_t ldw,
                               const float* h, const float* S, int lo, int hi, uint8_t* codes,
                               uint8_t* scales, int8_t* offs, const LanePlan& p,
                               cudaStream_t stream);

// A layer's projections in one call (layer.cu).  input: index of the
// calibration input whose h weights the matrix, -1 for plain MSE.
struct LayerWeight {
  const uint16_t* W;
  int64_t out, in, ldw;
  int input;
  float* S;
  float* amax;
  int* status;
  uint8_t* codes;
  uint8_t* scales;
  int8_t* offs;
};
struct LayerInput {
  const uint16_t* X;
  int64_t tokens, in, ldx;
  float* h;
};
size_t layer_workspace_bytes(const LayerWeight* w, int nw, const LayerInput* x, int nx, int sms);
// The order quantize_layer sweeps the weights in (indices into w): the
// permutation with the lowest estimated time for up to kMaxOrderedWeights
// weights; for more, the best choice of the first weight with the others in
// the caller's order.  Ties keep the caller's order.
constexpr int kMaxOrderedWeights = 4;
std::vector<int> layer_sweep_order(const LayerWeight* w, int nw, const LayerInput* x, int nx,
                                   int sms, int lo, int hi);
cudaError_t quantize_layer(const LayerWeight* w, int nw, const LayerInput* x, int nx, float q_max,
                           int lo, int hi, void* workspace, int sms, const cudaEvent_t* events,
                           cudaStream_t stream);

// Online activation quantization: per-token S and the MSE sweep in one launch.
// A team of 1, 2 or 4 warps owns a row at a time (chosen from the shape).
int act_quant_team_warps(int64_t tokens, int64_t in, int num_sms, bool k11);
cudaError_t launch_quantize_activations(const uint16_t* A, int64_t tokens, int64_t in,
                                        int64_t lda, float q_max, int lo, int hi, float* S,
                                        uint8_t* codes, uint8_t* scales, int8_t* offs,
                                        int* status, int num_sms, cudaStream_t stream);

// Row-major scale bytes -> the tensor-core MMA's tiled 128 x 4 scale layout.
size_t blocked_scales_bytes(int64_t rows, int64_t cols);
cudaError_t launch_scales_to_blocked(const uint8_t* sf, int64_t rows, int64_t cols, int64_t ld,
                                     uint8_t* out, int num_sms, cudaStream_t stream);

cudaError_t launch_dequantize(const uint8_t* codes, const uint8_t* scales, const float* S,
                              int64_t out, int64_t in, float* W_out, int num_sms,
                              cudaStream_t stream);

// H-Scale as GPTQ's local quantizer (gptq.cu).
// Opt-in phase timing of launch_gptq (see nvfp4_gptq_set_timing).
void gptq_set_timing(bool on);
cudaError_t gptq_phase_times(float* ms, int n, bool* overflow);
size_t gptq_workspace_bytes(int64_t out, int64_t in, int64_t tokens, int sms);
cudaError_t launch_gptq(const uint16_t* W, int64_t out, int64_t in, int64_t ldw, const uint16_t* X,
                        int64_t tokens, int64_t ldx, float q_max, int lo, int hi, float damp,
                        bool weighted, uint8_t* codes, uint8_t* scales, float* S, float* h,
                        int* status, void* workspace, size_t workspace_bytes, int sms,
                        cudaStream_t stream);
// The windowed sweep of an FP32 matrix (GPTQ's local call on its own).
cudaError_t launch_sweep_f32(const float* W, int64_t out, int64_t in, int64_t ldw, const float* h,
                             const float* S, int lo, int hi, uint8_t* codes, uint8_t* scales,
                             int num_sms, cudaStream_t stream);

// Maps a CUDA error to the entry points' status: NVFP4_OK for cudaSuccess,
// otherwise NVFP4_ERR_CUDA, with the code kept for nvfp4_last_cuda_error()
// (per host thread).  Defined with the entry points in nvfp4hs_capi.cu.
int record_cuda_status(cudaError_t e);

}  // namespace nvfp4
