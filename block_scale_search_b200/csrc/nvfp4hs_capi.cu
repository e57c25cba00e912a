// nvfp4hs_capi.cu -- the extern "C" entry points declared in include/nvfp4hs.h.
//
// Every entry point validates its arguments on the host, before any CUDA call,
// and returns a negative nvfp4_status on failure with nothing enqueued.  Only
// then does it look up the current device's SM count (cached) to size the grid
// and launch.  No C++ exception crosses this boundary.
#include "nvfp4hs.h"

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdint>
#include <functional>
#include <vector>

#include "checks.cuh"
#include "nvfp4_kernels.cuh"
#include "nvtx_range.cuh"
#include "row_counters.cuh"
#include "side_reduce.cuh"

namespace {

constexpr int64_t kMaxDim = int64_t{1} << 40;  // guards index arithmetic
thread_local int g_last_cuda_error = 0;

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

int cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return NVFP4_OK;
  g_last_cuda_error = static_cast<int>(e);
  return NVFP4_ERR_CUDA;
}

// NVFP4_ERR_CAPTURE when `s` is being captured into a CUDA graph, else
// NVFP4_OK.  The batched and grouped calls stage their descriptor tables
// from host memory that is gone once they return; a graph replay would read
// it later, so those calls refuse a capturing stream instead.
int refuse_capture(cudaStream_t s) {
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(s, &cs) != cudaSuccess) {
    cudaGetLastError();
    return NVFP4_OK;  // let the call's own CUDA calls report the stream's state
  }
  return cs == cudaStreamCaptureStatusNone ? NVFP4_OK : NVFP4_ERR_CAPTURE;
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

// Arguments of nvfp4_quantize_layer, converted for the planner; NVFP4_OK or
// the first failing status.
int check_layer(const nvfp4_layer_weight* w, int nw, const nvfp4_layer_input* x, int nx,
                std::vector<nvfp4::LayerWeight>* wv, std::vector<nvfp4::LayerInput>* xv) {
  if (nw < 0 || nx < 0 || (nw > 0 && w == nullptr) || (nx > 0 && x == nullptr))
    return NVFP4_ERR_INVALID_ARG;
  for (int k = 0; k < nx; ++k) {
    const nvfp4_layer_input& in = x[k];
    int st = check_diag_hessian(in.X, in.tokens, in.in, in.ldx, in.h, 0);
    if (st != NVFP4_OK) return st;
    if (!aligned(in.h, 16)) return NVFP4_ERR_ALIGN;  // the sweep reads h in 16-byte vectors
    if (xv) xv->push_back(nvfp4::LayerInput{static_cast<const uint16_t*>(in.X), in.tokens, in.in,
                                            in.ldx, in.h});
  }
  for (int j = 0; j < nw; ++j) {
    const nvfp4_layer_weight& m = w[j];
    int st = check_matrix(m.W, m.out, m.in, m.ldw, 16);
    if (st != NVFP4_OK) return st;
    if (m.out == 0 || m.in == 0) return NVFP4_ERR_SHAPE;
    if (m.S == nullptr || m.codes == nullptr || m.scales == nullptr) return NVFP4_ERR_INVALID_ARG;
    if (m.input < -1 || m.input >= nx) return NVFP4_ERR_INVALID_ARG;
    if (m.input >= 0 && x[m.input].in != m.in) return NVFP4_ERR_SHAPE;
    if (!aligned(m.S, 4) || !aligned(m.amax, 4) || !aligned(m.status, 4) || !aligned(m.codes, 8))
      return NVFP4_ERR_ALIGN;
    if (wv) wv->push_back(nvfp4::LayerWeight{static_cast<const uint16_t*>(m.W), m.out, m.in, m.ldw,
                                             m.input, m.S, m.amax, m.status, m.codes, m.scales,
                                             m.chosen_offset});
  }
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

namespace nvfp4 {
int record_cuda_status(cudaError_t e) { return cuda_status(e); }

// The checked build's per-translation-unit records (checks.cuh).
namespace {
std::vector<cudaError_t (*)(CheckState*, bool)>& check_readers() {
  static std::vector<cudaError_t (*)(CheckState*, bool)> v;
  return v;
}
}  // namespace

int register_check_reader(cudaError_t (*reader)(CheckState*, bool)) {
  check_readers().push_back(reader);
  return static_cast<int>(check_readers().size());
}

bool checks_compiled() {
#ifdef NVFP4HS_CHECKS
  return true;
#else
  return false;
#endif
}

cudaError_t collect_checks(CheckState* out, bool reset) {
  *out = CheckState{};
  for (auto* reader : check_readers()) {
    const cudaError_t e = reader(out, reset);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}
}  // namespace nvfp4

extern "C" {

int nvfp4_version(void) { return 100; }  // 0.1.0

int nvfp4_last_cuda_error(void) { return g_last_cuda_error; }

int nvfp4_debug_checks_compiled(void) { return nvfp4::checks_compiled() ? 1 : 0; }

int nvfp4_debug_checks(unsigned long long* first, unsigned int* count, int reset) {
  if (first == nullptr || count == nullptr || (reset != 0 && reset != 1))
    return NVFP4_ERR_INVALID_ARG;
  nvfp4::CheckState st{};
  const cudaError_t e = nvfp4::collect_checks(&st, reset != 0);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return cuda_status(e);
  }
  *first = st.first;
  *count = st.count;
  return NVFP4_OK;
}

size_t nvfp4_diag_hessian_workspace_size(int64_t tokens, int64_t in) {
  if (tokens < 0 || in <= 0 || in % 8 != 0 || in > kMaxDim) return 0;
  const int sms = current_sm_count();
  if (sms <= 0) return 0;
  const nvfp4::LanePlan p = nvfp4::diag_hessian_plan(tokens, in, sms);
  return nvfp4::diag_hessian_workspace_bytes(p, in);
}

int nvfp4_diag_hessian(const void* X, int64_t tokens, int64_t in, int64_t ldx, float* h,
                       int accumulate, void* workspace, size_t workspace_bytes, void* stream) {
  NVFP4_RANGE("nvfp4_diag_hessian");
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
  NVFP4_RANGE("nvfp4_global_scale");
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
  NVFP4_RANGE("nvfp4_scale_sweep_quantize");
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
  const nvfp4::LanePlan p = nvfp4::sweep_plan(out, in, sms, h != nullptr, hi - lo + 1);
  return cuda_status(nvfp4::launch_scale_sweep(static_cast<const uint16_t*>(W), out, in, ldw, h,
                                               S, lo, hi, codes, scales, chosen_offset, p,
                                               static_cast<cudaStream_t>(stream)));
}

}  // extern "C"

namespace {

// Several layers' descriptors as one: inputs appended layer by layer, each
// weight's input index moved by its layer's first input.
int flatten_layers(const nvfp4_layer* layers, int n_layers, std::vector<nvfp4_layer_weight>* w,
                   std::vector<nvfp4_layer_input>* x) {
  if (n_layers < 0 || (n_layers > 0 && layers == nullptr)) return NVFP4_ERR_INVALID_ARG;
  int64_t nw = 0, nx = 0;
  for (int l = 0; l < n_layers; ++l) {
    const nvfp4_layer& L = layers[l];
    if (L.n_weights < 0 || L.n_inputs < 0 || (L.n_weights > 0 && L.weights == nullptr) ||
        (L.n_inputs > 0 && L.inputs == nullptr))
      return NVFP4_ERR_INVALID_ARG;
    nw += L.n_weights;
    nx += L.n_inputs;
  }
  if (nw > (1 << 20) || nx > (1 << 20)) return NVFP4_ERR_INVALID_ARG;
  w->clear();
  x->clear();
  for (int l = 0; l < n_layers; ++l) {
    const nvfp4_layer& L = layers[l];
    const int base = static_cast<int>(x->size());
    for (int k = 0; k < L.n_inputs; ++k) x->push_back(L.inputs[k]);
    for (int j = 0; j < L.n_weights; ++j) {
      nvfp4_layer_weight d = L.weights[j];
      if (d.input < -1 || d.input >= L.n_inputs) return NVFP4_ERR_INVALID_ARG;
      if (d.input >= 0) d.input += base;
      w->push_back(d);
    }
  }
  return NVFP4_OK;
}

}  // namespace

extern "C" {

size_t nvfp4_gptq_workspace_size(int64_t out, int64_t in, int64_t tokens) {
  constexpr int64_t kIntMax = (int64_t{1} << 31) - 1;
  if (out <= 0 || in <= 0 || tokens < 0 || in % 16 != 0 || in > 16 * 65535 || out > kIntMax ||
      tokens > kIntMax)
    return 0;
  const int sms = current_sm_count();
  if (sms <= 0) return 0;
  return nvfp4::gptq_workspace_bytes(out, in, tokens, sms);
}

int nvfp4_gptq_quantize(const void* W, int64_t out, int64_t in, int64_t ldw, const void* X,
                        int64_t tokens, int64_t ldx, float q_max, int lo, int hi, float damp,
                        int weighted, uint8_t* codes, uint8_t* scales, float* S, float* h,
                        int* status, void* workspace, size_t workspace_bytes, void* stream) {
  NVFP4_RANGE("nvfp4_gptq_quantize");
  if (W == nullptr || codes == nullptr || scales == nullptr || S == nullptr || h == nullptr ||
      (X == nullptr && tokens > 0))
    return NVFP4_ERR_INVALID_ARG;
  if (out <= 0 || in <= 0 || tokens < 0 || (weighted != 0 && weighted != 1))
    return NVFP4_ERR_INVALID_ARG;
  // cuBLAS and cuSOLVER take int sizes and leading dimensions
  constexpr int64_t kIntMax = (int64_t{1} << 31) - 1;
  // in / 16 is also a grid dimension of the factor's reflection
  if (in % 16 != 0 || ldw < in || ldx < in || in > 16 * 65535 || out > kIntMax ||
      tokens > kIntMax || ldw > kMaxDim || ldx > kIntMax)
    return NVFP4_ERR_SHAPE;
  if (!std::isfinite(q_max) || !(q_max > 0.0f) || !std::isfinite(damp) || damp < 0.0f)
    return NVFP4_ERR_INVALID_ARG;
  if (lo < -16 || lo > 0 || hi < 0 || hi > 15 || hi - lo > 15) return NVFP4_ERR_WINDOW;
  // W's rows are read in 16-byte vectors (its global scale, the batch kernel)
  if (!aligned(W, 16) || ldw % 8 != 0 || !aligned(X, 16) || ldx % 8 != 0 || !aligned(codes, 8) ||
      !aligned(S, 4) || !aligned(h, 16) || !aligned(status, 4))
    return NVFP4_ERR_ALIGN;
  if (workspace == nullptr) return NVFP4_ERR_WORKSPACE;
  if (!aligned(workspace, 256)) return NVFP4_ERR_ALIGN;
  const int sms = current_sm_count();
  if (sms <= 0) return cuda_status(cudaErrorNoDevice);
  const size_t need = nvfp4::gptq_workspace_bytes(out, in, tokens, sms);
  if (need == 0) return cuda_status(cudaErrorUnknown);
  if (workspace_bytes < need) return NVFP4_ERR_WORKSPACE;
  return cuda_status(nvfp4::launch_gptq(
      static_cast<const uint16_t*>(W), out, in, ldw, static_cast<const uint16_t*>(X), tokens, ldx,
      q_max, lo, hi, damp, weighted != 0, codes, scales, S, h, status, workspace, workspace_bytes,
      sms, static_cast<cudaStream_t>(stream)));
}

int nvfp4_gptq_set_timing(int on) {
  if (on != 0 && on != 1) return NVFP4_ERR_INVALID_ARG;
  nvfp4::gptq_set_timing(on != 0);
  return NVFP4_OK;
}

int nvfp4_gptq_phase_times(float* ms, int n) {
  if (ms == nullptr || n < 0 || n > NVFP4_GPTQ_PHASES) return NVFP4_ERR_INVALID_ARG;
  bool overflow = false;
  const cudaError_t e = nvfp4::gptq_phase_times(ms, n, &overflow);
  if (e != cudaSuccess) return cuda_status(e);
  return overflow ? NVFP4_ERR_WORKSPACE : NVFP4_OK;
}

int nvfp4_scale_sweep_quantize_f32(const float* W, int64_t out, int64_t in, int64_t ldw,
                                   const float* h, const float* S, int lo, int hi,
                                   uint8_t* codes, uint8_t* scales, void* stream) {
  NVFP4_RANGE("nvfp4_scale_sweep_quantize_f32");
  if (out < 0 || in < 0) return NVFP4_ERR_INVALID_ARG;
  const bool empty = out == 0 || in == 0;
  if (!empty && (W == nullptr || S == nullptr || codes == nullptr || scales == nullptr))
    return NVFP4_ERR_INVALID_ARG;
  if (in % 16 != 0 || ldw < in || out > kMaxDim || in > kMaxDim || ldw > kMaxDim)
    return NVFP4_ERR_SHAPE;
  if (lo < -16 || lo > 0 || hi < 0 || hi > 15 || hi - lo > 15) return NVFP4_ERR_WINDOW;
  if (!aligned(W, 4) || !aligned(h, 16) || !aligned(S, 4) || !aligned(codes, 8))
    return NVFP4_ERR_ALIGN;
  if (empty) return NVFP4_OK;
  const int sms = current_sm_count();
  if (sms <= 0) return cuda_status(cudaErrorNoDevice);
  return cuda_status(nvfp4::launch_sweep_f32(W, out, in, ldw, h, S, lo, hi, codes, scales, sms,
                                             static_cast<cudaStream_t>(stream)));
}

size_t nvfp4_quantize_layers_workspace_size(const nvfp4_layer* layers, int n_layers) {
  std::vector<nvfp4_layer_weight> w;
  std::vector<nvfp4_layer_input> x;
  if (flatten_layers(layers, n_layers, &w, &x) != NVFP4_OK) return 0;
  return nvfp4_quantize_layer_workspace_size(w.data(), static_cast<int>(w.size()), x.data(),
                                             static_cast<int>(x.size()));
}

int nvfp4_quantize_layers(const nvfp4_layer* layers, int n_layers, float q_max, int lo, int hi,
                          void* workspace, size_t workspace_bytes, void* const* sweep_events,
                          void* stream) {
  NVFP4_RANGE("nvfp4_quantize_layers");
  std::vector<nvfp4_layer_weight> w;
  std::vector<nvfp4_layer_input> x;
  const int st = flatten_layers(layers, n_layers, &w, &x);
  if (st != NVFP4_OK) return st;
  return nvfp4_quantize_layer(w.data(), static_cast<int>(w.size()), x.data(),
                              static_cast<int>(x.size()), q_max, lo, hi, workspace,
                              workspace_bytes, sweep_events, stream);
}

size_t nvfp4_quantize_layer_workspace_size(const nvfp4_layer_weight* weights, int n_weights,
                                           const nvfp4_layer_input* inputs, int n_inputs) {
  std::vector<nvfp4::LayerWeight> wv;
  std::vector<nvfp4::LayerInput> xv;
  if (check_layer(weights, n_weights, inputs, n_inputs, &wv, &xv) != NVFP4_OK) return 0;
  const int sms = current_sm_count();
  if (sms <= 0) return 0;
  return nvfp4::layer_workspace_bytes(wv.data(), n_weights, xv.data(), n_inputs, sms);
}

int nvfp4_quantize_layer_order(const nvfp4_layer_weight* weights, int n_weights,
                               const nvfp4_layer_input* inputs, int n_inputs, int lo, int hi,
                               int* order) {
  std::vector<nvfp4::LayerWeight> wv;
  std::vector<nvfp4::LayerInput> xv;
  const int st = check_layer(weights, n_weights, inputs, n_inputs, &wv, &xv);
  if (st != NVFP4_OK) return st;
  if (lo < -16 || lo > 0 || hi < 0 || hi > 15 || hi - lo > 15) return NVFP4_ERR_WINDOW;
  if (order == nullptr && n_weights > 0) return NVFP4_ERR_INVALID_ARG;
  const int sms = current_sm_count();
  if (sms <= 0) return cuda_status(cudaErrorNoDevice);
  const std::vector<int> perm =
      nvfp4::layer_sweep_order(wv.data(), n_weights, xv.data(), n_inputs, sms, lo, hi);
  for (int j = 0; j < n_weights; ++j) order[j] = perm[j];
  return NVFP4_OK;
}

int nvfp4_quantize_layer(const nvfp4_layer_weight* weights, int n_weights,
                         const nvfp4_layer_input* inputs, int n_inputs, float q_max, int lo,
                         int hi, void* workspace, size_t workspace_bytes,
                         void* const* sweep_events, void* stream) {
  NVFP4_RANGE("nvfp4_quantize_layer");
  std::vector<nvfp4::LayerWeight> wv;
  std::vector<nvfp4::LayerInput> xv;
  int st = check_layer(weights, n_weights, inputs, n_inputs, &wv, &xv);
  if (st != NVFP4_OK) return st;
  if (!std::isfinite(q_max) || !(q_max > 0.0f)) return NVFP4_ERR_INVALID_ARG;
  if (lo < -16 || lo > 0 || hi < 0 || hi > 15 || hi - lo > 15) return NVFP4_ERR_WINDOW;
  if (n_weights == 0 && n_inputs == 0) return NVFP4_OK;
  if (workspace == nullptr) return NVFP4_ERR_WORKSPACE;
  if (!aligned(workspace, 256)) return NVFP4_ERR_ALIGN;
  const int sms = current_sm_count();
  if (sms <= 0) return cuda_status(cudaErrorNoDevice);
  if (workspace_bytes < nvfp4::layer_workspace_bytes(wv.data(), n_weights, xv.data(), n_inputs, sms))
    return NVFP4_ERR_WORKSPACE;
  if (sweep_events != nullptr)
    for (int j = 0; j < 2 * n_weights; ++j)
      if (sweep_events[j] == nullptr) return NVFP4_ERR_INVALID_ARG;
  return cuda_status(nvfp4::quantize_layer(
      wv.data(), n_weights, xv.data(), n_inputs, q_max, lo, hi, workspace, sms,
      reinterpret_cast<cudaEvent_t const*>(sweep_events), static_cast<cudaStream_t>(stream)));
}

int nvfp4_debug_row_counters(void** ptr, size_t* bytes) {
  if (ptr == nullptr || bytes == nullptr) return NVFP4_ERR_INVALID_ARG;
  return cuda_status(nvfp4::row_counters_symbol(ptr, bytes));
}

int nvfp4_scale_sweep_quantize_full(const void* W, int64_t out, int64_t in, int64_t ldw,
                                    const float* h, const float* S, uint8_t* codes,
                                    uint8_t* scales, int8_t* chosen_offset, void* stream) {
  NVFP4_RANGE("nvfp4_scale_sweep_quantize_full");
  int st = check_matrix(W, out, in, ldw, 16);
  if (st != NVFP4_OK) return st;
  const bool empty = out == 0 || in == 0;
  if (!empty && (S == nullptr || codes == nullptr || scales == nullptr))
    return NVFP4_ERR_INVALID_ARG;
  if (!aligned(h, 16) || !aligned(S, 4) || !aligned(codes, 8)) return NVFP4_ERR_ALIGN;
  if (empty) return NVFP4_OK;
  const int sms = current_sm_count();
  if (sms <= 0) return cuda_status(cudaErrorNoDevice);
  return cuda_status(nvfp4::launch_scale_sweep_full(static_cast<const uint16_t*>(W), out, in, ldw,
                                                    h, S, codes, scales, chosen_offset, sms,
                                                    static_cast<cudaStream_t>(stream)));
}

int nvfp4_quantize_activations(const void* A, int64_t tokens, int64_t in, int64_t lda,
                               float q_max, int lo, int hi, float* S, uint8_t* codes,
                               uint8_t* scales, int8_t* chosen_offset, int* status,
                               void* stream) {
  NVFP4_RANGE("nvfp4_quantize_activations");
  int st = check_matrix(A, tokens, in, lda, 16);
  if (st != NVFP4_OK) return st;
  if (!std::isfinite(q_max) || !(q_max > 0.0f)) return NVFP4_ERR_INVALID_ARG;
  if (tokens > 0 && S == nullptr) return NVFP4_ERR_INVALID_ARG;
  if (tokens > 0 && in > 0 && (codes == nullptr || scales == nullptr))
    return NVFP4_ERR_INVALID_ARG;
  if (lo < -16 || lo > 0 || hi < 0 || hi > 15 || hi - lo > 15) return NVFP4_ERR_WINDOW;
  if (!aligned(S, 4) || !aligned(codes, 8) || !aligned(status, 4)) return NVFP4_ERR_ALIGN;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (status != nullptr) {
    const cudaError_t e = cudaMemsetAsync(status, 0, sizeof(int), s);
    if (e != cudaSuccess) return cuda_status(e);
  }
  if (tokens == 0) return NVFP4_OK;
  const int sms = current_sm_count();
  if (sms <= 0) return cuda_status(cudaErrorNoDevice);
  return cuda_status(nvfp4::launch_quantize_activations(static_cast<const uint16_t*>(A), tokens,
                                                        in, lda, q_max, lo, hi, S, codes, scales,
                                                        chosen_offset, status, sms, s));
}

size_t nvfp4_blocked_scales_size(int64_t rows, int64_t cols) {
  if (rows < 0 || cols < 0 || rows > kMaxDim || cols > kMaxDim) return 0;
  return nvfp4::blocked_scales_bytes(rows, cols);
}

int nvfp4_scales_to_blocked(const uint8_t* scales, int64_t rows, int64_t cols, int64_t ld,
                            uint8_t* out, void* stream) {
  NVFP4_RANGE("nvfp4_scales_to_blocked");
  if (rows < 0 || cols < 0) return NVFP4_ERR_INVALID_ARG;
  if (ld < cols || rows > kMaxDim || cols > kMaxDim || ld > kMaxDim) return NVFP4_ERR_SHAPE;
  if (rows == 0 || cols == 0) return NVFP4_OK;
  if (scales == nullptr || out == nullptr) return NVFP4_ERR_INVALID_ARG;
  if (!aligned(out, 16)) return NVFP4_ERR_ALIGN;
  const int sms = current_sm_count();
  if (sms <= 0) return cuda_status(cudaErrorNoDevice);
  return cuda_status(nvfp4::launch_scales_to_blocked(scales, rows, cols, ld, out, sms,
                                                     static_cast<cudaStream_t>(stream)));
}

int nvfp4_dequantize(const uint8_t* codes, const uint8_t* scales, const float* S, int64_t out,
                     int64_t in, float* W_out, void* stream) {
  NVFP4_RANGE("nvfp4_dequantize");
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


// ------------------------------------------------------------- grouped / batched

size_t nvfp4_diag_hessian_grouped_workspace_size(int64_t total_tokens, int64_t experts, int64_t in) {
  if (total_tokens < 0 || experts <= 0 || experts > 65535 || in <= 0 || in % 8 != 0 ||
      in > kMaxDim || total_tokens > kMaxDim)
    return 0;
  const int sms = current_sm_count();
  if (sms <= 0) return 0;
  return nvfp4::diag_hessian_grouped_workspace_bytes(total_tokens, experts, in, sms);
}

int nvfp4_diag_hessian_grouped(const void* X, const int64_t* row_offsets, int64_t experts,
                               int64_t total_tokens, int64_t in, int64_t ldx, float* h,
                               int accumulate, void* workspace, size_t workspace_bytes,
                               void* stream) {
  NVFP4_RANGE("nvfp4_diag_hessian_grouped");
  int st = check_diag_hessian(X, total_tokens, in, ldx, h, accumulate);
  if (st != NVFP4_OK) return st;
  if (row_offsets == nullptr || experts <= 0) return NVFP4_ERR_INVALID_ARG;
  if (experts > 65535) return NVFP4_ERR_SHAPE;
  if (!aligned(row_offsets, 8)) return NVFP4_ERR_ALIGN;
  if (workspace == nullptr) return NVFP4_ERR_WORKSPACE;
  if (!aligned(workspace, 256)) return NVFP4_ERR_ALIGN;
  // at least one partial row per expert plus one, whatever the device
  if (workspace_bytes < static_cast<size_t>(experts + 1) * static_cast<size_t>(in) * sizeof(float))
    return NVFP4_ERR_WORKSPACE;
  const int sms = current_sm_count();
  if (sms <= 0) return cuda_status(cudaErrorNoDevice);
  if (workspace_bytes < nvfp4::diag_hessian_grouped_workspace_bytes(total_tokens, experts, in, sms))
    return NVFP4_ERR_WORKSPACE;
  return cuda_status(nvfp4::launch_diag_hessian_grouped(
      static_cast<const uint16_t*>(X), row_offsets, experts, total_tokens, in, ldx, h, accumulate,
      workspace, sms, static_cast<cudaStream_t>(stream)));
}

namespace {

int check_batch(const nvfp4_matrix_desc* descs, int64_t n, int64_t in_multiple) {
  if (n < 0 || (n > 0 && descs == nullptr)) return NVFP4_ERR_INVALID_ARG;
  for (int64_t i = 0; i < n; ++i) {
    const int st = check_matrix(descs[i].W, descs[i].out, descs[i].in, descs[i].ldw, in_multiple);
    if (st != NVFP4_OK) return st;
  }
  return NVFP4_OK;
}

// CTAs per matrix: a one-wave budget shared in proportion to elements, >= 1 each.
std::vector<int64_t> share_ctas(const std::vector<int64_t>& elems, int64_t budget) {
  int64_t total = 0;
  for (int64_t e : elems) total += e;
  std::vector<int64_t> c(elems.size(), 1);
  if (total > 0)
    for (size_t i = 0; i < elems.size(); ++i) {
      const double share = static_cast<double>(budget) * static_cast<double>(elems[i]) /
                           static_cast<double>(total);
      c[i] = share < 1.0 ? 1 : static_cast<int64_t>(share + 0.5);
    }
  return c;
}

size_t round256(size_t x) { return (x + 255) & ~size_t{255}; }

// The batched sweep's device descriptors: `budget` CTAs shared by the
// matrices' group counts (eight waves' worth for the plain batched sweep:
// with many small matrices a one-wave share rounds to whole CTAs and can
// spill a few into a mostly empty second wave, and every CTA ends with its
// slowest warp; the more, shorter CTAs the hardware deals out as others
// finish, the smaller both tails -- measured on the 128-expert layer: 2, 4,
// 8, 16 waves take 2.33, 2.12, 2.07, 2.08 ms).  Returns the CTAs in all.
int64_t plan_sweep_batch(const nvfp4_sweep_desc* descs, int64_t n,
                         const std::vector<int64_t>& groups, int64_t budget,
                         std::vector<nvfp4::SweepDesc>* dv) {
  const std::vector<int64_t> ctas = share_ctas(groups, budget);
  dv->assign(n, nvfp4::SweepDesc{});
  int64_t total_ctas = 0;
  for (int64_t i = 0; i < n; ++i) {
    const nvfp4_sweep_desc& d = descs[i];
    nvfp4::SweepDesc& m = (*dv)[i];
    const int64_t c = groups[i] == 0 ? 1 : ctas[i];
    const nvfp4::LanePlan p = nvfp4::sweep_plan_threads(d.out, d.in, c * nvfp4::kSweepCta);
    m.W = static_cast<const uint16_t*>(d.W);
    m.h = d.h;
    m.S = d.S;
    m.codes = d.codes;
    m.scales = d.scales;
    m.offs = d.chosen_offset;
    m.out = groups[i] == 0 ? 0 : d.out;  // an empty matrix does no work
    m.G = d.in / 16;
    m.ldw = d.ldw;
    m.GL = p.VL;
    m.R = p.R;
    m.cta_begin = total_ctas;
    total_ctas += c;
  }
  return total_ctas;
}

struct GsBatchPlan {
  std::vector<nvfp4::MatDesc> d;
  int64_t total_ctas = 0;
};

GsBatchPlan plan_global_scale_batch(const nvfp4_matrix_desc* descs, int64_t n, int sms) {
  GsBatchPlan p;
  std::vector<int64_t> elems(n);
  for (int64_t i = 0; i < n; ++i) elems[i] = descs[i].out * descs[i].in;
  // two waves' worth of CTAs: with one, the many small matrices' rounded
  // shares leave the wave's end ragged (128 experts x 3 matrices: 5.64 TB/s
  // with one wave, 6.41 with two, 6.29 with four)
  const std::vector<int64_t> ctas =
      share_ctas(elems, 2 * static_cast<int64_t>(sms) * nvfp4::absmax_resident_ctas());
  p.d.resize(n);
  for (int64_t i = 0; i < n; ++i) {
    nvfp4::MatDesc& m = p.d[i];
    m.W = static_cast<const uint16_t*>(descs[i].W);
    m.out = descs[i].out;
    m.ldw = descs[i].ldw;
    m.V = descs[i].in / 8;
    const int64_t nt = ctas[i] * 256;
    m.VL = m.V < nt ? (m.V > 0 ? m.V : 1) : nt;
    int64_t R = nt / m.VL;
    if (R > m.out) R = m.out;
    if (R < 1) R = 1;
    m.R = R;
    m.cta_begin = p.total_ctas;
    p.total_ctas += ctas[i];
  }
  return p;
}

}  // namespace

size_t nvfp4_global_scale_batched_workspace_size(const nvfp4_matrix_desc* descs, int64_t n) {
  if (check_batch(descs, n, 8) != NVFP4_OK) return 0;
  const int sms = current_sm_count();
  if (sms <= 0) return 0;
  const GsBatchPlan p = plan_global_scale_batch(descs, n, sms);
  return round256(static_cast<size_t>(n) * sizeof(nvfp4::MatDesc)) +
         static_cast<size_t>(p.total_ctas) * sizeof(uint32_t) + 256;
}

int nvfp4_global_scale_batched(const nvfp4_matrix_desc* descs, int64_t n, float q_max, float* S,
                               float* amax, int* status, void* workspace, size_t workspace_bytes,
                               void* stream) {
  NVFP4_RANGE("nvfp4_global_scale_batched");
  int st = check_batch(descs, n, 8);
  if (st != NVFP4_OK) return st;
  if (n == 0) return NVFP4_OK;
  if (S == nullptr || !std::isfinite(q_max) || !(q_max > 0.0f)) return NVFP4_ERR_INVALID_ARG;
  if (!aligned(S, 4) || !aligned(amax, 4) || !aligned(status, 4)) return NVFP4_ERR_ALIGN;
  if (workspace == nullptr) return NVFP4_ERR_WORKSPACE;
  if (!aligned(workspace, 256)) return NVFP4_ERR_ALIGN;
  if ((st = refuse_capture(static_cast<cudaStream_t>(stream))) != NVFP4_OK) return st;
  const int sms = current_sm_count();
  if (sms <= 0) return cuda_status(cudaErrorNoDevice);
  const GsBatchPlan p = plan_global_scale_batch(descs, n, sms);
  const size_t head = round256(static_cast<size_t>(n) * sizeof(nvfp4::MatDesc));
  if (workspace_bytes < head + static_cast<size_t>(p.total_ctas) * sizeof(uint32_t))
    return NVFP4_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  nvfp4::MatDesc* d_dev = static_cast<nvfp4::MatDesc*>(workspace);
  // the table is staged from host memory before this call returns
  cudaError_t e = cudaMemcpyAsync(d_dev, p.d.data(), static_cast<size_t>(n) * sizeof(nvfp4::MatDesc),
                                  cudaMemcpyHostToDevice, s);
  if (e != cudaSuccess) return cuda_status(e);
  uint32_t* partial = reinterpret_cast<uint32_t*>(static_cast<char*>(workspace) + head);
  return cuda_status(nvfp4::launch_global_scale_batched(d_dev, n, p.total_ctas, q_max, S, amax,
                                                        status, partial, s));
}

}  // extern "C"

namespace {

// Validation of nvfp4_quantize_grouped_layer's arguments (NVFP4_OK or the
// first failing status); the matrices' descriptors for the batched S.
int check_grouped_layer(const nvfp4_sweep_desc* first, int64_t nf, const nvfp4_sweep_desc* second,
                        int64_t ns, const nvfp4_grouped_input* x1, const nvfp4_grouped_input* x2,
                        int64_t experts, float* S, std::vector<nvfp4_matrix_desc>* md,
                        bool* weighted1, bool* weighted2) {
  if (nf < 0 || ns < 0 || (nf > 0 && first == nullptr) || (ns > 0 && second == nullptr))
    return NVFP4_ERR_INVALID_ARG;
  if (x1 == nullptr || x2 == nullptr || S == nullptr || experts <= 0) return NVFP4_ERR_INVALID_ARG;
  if (experts > 65535) return NVFP4_ERR_SHAPE;
  for (const nvfp4_grouped_input* x : {x1, x2}) {
    int st = check_diag_hessian(x->X, x->total_tokens, x->in, x->ldx, x->h, 0);
    if (st != NVFP4_OK) return st;
    if (x->row_offsets == nullptr) return NVFP4_ERR_INVALID_ARG;
    if (!aligned(x->row_offsets, 8) || !aligned(x->h, 16)) return NVFP4_ERR_ALIGN;
  }
  if (!aligned(S, 4)) return NVFP4_ERR_ALIGN;
  md->clear();
  for (int b = 0; b < 2; ++b) {
    const nvfp4_sweep_desc* d = b == 0 ? first : second;
    const int64_t n = b == 0 ? nf : ns;
    bool any_h = false, all_h = true;
    for (int64_t i = 0; i < n; ++i) {
      const nvfp4_sweep_desc& m = d[i];
      int st = check_matrix(m.W, m.out, m.in, m.ldw, 16);
      if (st != NVFP4_OK) return st;
      if (m.out == 0 || m.in == 0) return NVFP4_ERR_SHAPE;
      if (m.codes == nullptr || m.scales == nullptr) return NVFP4_ERR_INVALID_ARG;
      // each matrix's S is its place in the one S array the call writes
      if (m.S != S + (b == 0 ? i : nf + i)) return NVFP4_ERR_INVALID_ARG;
      if (!aligned(m.h, 16) || !aligned(m.codes, 8)) return NVFP4_ERR_ALIGN;
      any_h = any_h || m.h != nullptr;
      all_h = all_h && m.h != nullptr;
      md->push_back(nvfp4_matrix_desc{m.W, m.out, m.in, m.ldw});
    }
    if (any_h && !all_h) return NVFP4_ERR_INVALID_ARG;  // one objective per batch
    *(b == 0 ? weighted1 : weighted2) = any_h;
  }
  return NVFP4_OK;
}

struct GroupedLayerLayout {
  size_t gd1 = 0, gd2 = 0, gs = 0, sw1 = 0, sw2 = 0, bytes = 0;
  GsBatchPlan gsp;
};

GroupedLayerLayout grouped_layer_layout(int64_t nf, int64_t ns, const nvfp4_grouped_input* x1,
                                        const nvfp4_grouped_input* x2, int64_t experts,
                                        const std::vector<nvfp4_matrix_desc>& md, int sms) {
  GroupedLayerLayout L;
  size_t off = 0;
  L.gd1 = off;
  off = round256(off + nvfp4::diag_hessian_grouped_workspace_bytes(x1->total_tokens, experts,
                                                                   x1->in, sms));
  L.gd2 = off;
  off = round256(off + nvfp4::diag_hessian_grouped_workspace_bytes(x2->total_tokens, experts,
                                                                   x2->in, sms));
  L.gsp = plan_global_scale_batch(md.data(), static_cast<int64_t>(md.size()), sms);
  L.gs = off;
  off = round256(off + round256(md.size() * sizeof(nvfp4::MatDesc)) +
                 static_cast<size_t>(L.gsp.total_ctas) * sizeof(uint32_t));
  L.sw1 = off;
  off = round256(off + static_cast<size_t>(nf) * sizeof(nvfp4::SweepDesc));
  L.sw2 = off;
  off = round256(off + static_cast<size_t>(ns) * sizeof(nvfp4::SweepDesc));
  L.bytes = off;
  return L;
}

// Which batch a grouped layer call sweeps first.  The input of the batch swept
// first has its h computed on its own beforehand; the other input's h is
// streamed beside that sweep.  Costs are estimated in HBM-byte equivalents:
//   R(x)   = the bytes of input x (its reduction is bound by HBM);
//   Sw(b)  = weight elements x candidates x 1.3 (a sweep, bound by FP32
//            arithmetic, takes about 2.1e-13 s per element and candidate on
//            B200, as long as 1.3 bytes take at the copy bandwidth);
//   carrying R(x) beside Sw(b) takes max(Sw(b) + 0.38 R(x), R(x)) (a carrying
//   sweep slows by about 38% of the streamed reduction's time on its own).
// The call with a first is R(x_a) + carry(a, x_b) + Sw(b); the batch whose order
// costs less goes first (a tie keeps the caller's order).  The second batch
// may go first only if none of its h point into the first input's h, which
// would not be ready yet.
bool grouped_layer_second_first(const nvfp4_sweep_desc* first, int64_t nf,
                                const nvfp4_sweep_desc* second, int64_t ns,
                                const nvfp4_grouped_input& x1, const nvfp4_grouped_input& x2,
                                int64_t experts, int lo, int hi) {
  const float* h1_lo = x1.h;
  const float* h1_hi = x1.h + experts * x1.in;
  for (int64_t i = 0; i < ns; ++i) {
    const float* h = second[i].h;
    if (h != nullptr && std::less_equal<const float*>()(h1_lo, h) && std::less<const float*>()(h, h1_hi))
      return false;
  }
  constexpr double kSweepBytes = 1.3, kCarry = 0.38;
  const double K = static_cast<double>(hi - lo + 1);
  auto sweep = [&](const nvfp4_sweep_desc* d, int64_t n) {
    double e = 0.0;
    for (int64_t i = 0; i < n; ++i) e += static_cast<double>(d[i].out) * static_cast<double>(d[i].in);
    return e * K * kSweepBytes;
  };
  auto bytes = [](const nvfp4_grouped_input& x) {
    return 2.0 * static_cast<double>(x.total_tokens) * static_cast<double>(x.in);
  };
  auto cost = [&](double ra, double swa, int64_t na, double rb, double swb) {
    const double carry = na > 0 ? std::max(swa + kCarry * rb, rb) : rb;
    return ra + carry + swb;
  };
  const double s1 = sweep(first, nf), s2 = sweep(second, ns);
  const double r1 = bytes(x1), r2 = bytes(x2);
  return cost(r2, s2, ns, r1, s1) < cost(r1, s1, nf, r2, s2);
}

}  // namespace

extern "C" {

size_t nvfp4_scale_sweep_quantize_batched_workspace_size(int64_t n) {
  if (n < 0) return 0;
  return round256(static_cast<size_t>(n) * sizeof(nvfp4::SweepDesc)) + 256;
}

int nvfp4_scale_sweep_quantize_batched(const nvfp4_sweep_desc* descs, int64_t n, int lo, int hi,
                                       void* workspace, size_t workspace_bytes, void* stream) {
  NVFP4_RANGE("nvfp4_scale_sweep_quantize_batched");
  if (n < 0 || (n > 0 && descs == nullptr)) return NVFP4_ERR_INVALID_ARG;
  if (lo < -16 || lo > 0 || hi < 0 || hi > 15 || hi - lo > 15) return NVFP4_ERR_WINDOW;
  bool any_h = false, all_h = true;
  std::vector<int64_t> groups(n);
  for (int64_t i = 0; i < n; ++i) {
    const nvfp4_sweep_desc& d = descs[i];
    int st = check_matrix(d.W, d.out, d.in, d.ldw, 16);
    if (st != NVFP4_OK) return st;
    const bool empty = d.out == 0 || d.in == 0;
    if (!empty && (d.S == nullptr || d.codes == nullptr || d.scales == nullptr))
      return NVFP4_ERR_INVALID_ARG;
    if (!aligned(d.h, 16) || !aligned(d.S, 4) || !aligned(d.codes, 8)) return NVFP4_ERR_ALIGN;
    any_h = any_h || d.h != nullptr;
    all_h = all_h && d.h != nullptr;
    groups[i] = empty ? 0 : d.out * (d.in / 16);
  }
  if (any_h && !all_h) return NVFP4_ERR_INVALID_ARG;  // one objective per batch
  if (n == 0) return NVFP4_OK;
  if (workspace == nullptr) return NVFP4_ERR_WORKSPACE;
  if (!aligned(workspace, 256)) return NVFP4_ERR_ALIGN;
  if (workspace_bytes < round256(static_cast<size_t>(n) * sizeof(nvfp4::SweepDesc)))
    return NVFP4_ERR_WORKSPACE;
  if (const int cst = refuse_capture(static_cast<cudaStream_t>(stream)); cst != NVFP4_OK) return cst;
  const int sms = current_sm_count();
  if (sms <= 0) return cuda_status(cudaErrorNoDevice);
  const bool weighted = any_h;
  std::vector<nvfp4::SweepDesc> dv;
  const int64_t total_ctas = plan_sweep_batch(
      descs, n, groups, 8 * static_cast<int64_t>(sms) * nvfp4::sweep_resident_ctas(weighted), &dv);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  nvfp4::SweepDesc* d_dev = static_cast<nvfp4::SweepDesc*>(workspace);
  cudaError_t e = cudaMemcpyAsync(d_dev, dv.data(), static_cast<size_t>(n) * sizeof(nvfp4::SweepDesc),
                                  cudaMemcpyHostToDevice, s);
  if (e != cudaSuccess) return cuda_status(e);
  return cuda_status(nvfp4::launch_scale_sweep_batched(d_dev, n, total_ctas, weighted, lo, hi, s));
}

size_t nvfp4_quantize_grouped_layer_workspace_size(const nvfp4_sweep_desc* first, int64_t n_first,
                                                   const nvfp4_sweep_desc* second, int64_t n_second,
                                                   const nvfp4_grouped_input* first_input,
                                                   const nvfp4_grouped_input* second_input,
                                                   int64_t experts, float* S) {
  std::vector<nvfp4_matrix_desc> md;
  bool w1 = false, w2 = false;
  if (check_grouped_layer(first, n_first, second, n_second, first_input, second_input, experts, S,
                          &md, &w1, &w2) != NVFP4_OK)
    return 0;
  const int sms = current_sm_count();
  if (sms <= 0) return 0;
  return grouped_layer_layout(n_first, n_second, first_input, second_input, experts, md, sms).bytes;
}

int nvfp4_quantize_grouped_layer_order(const nvfp4_sweep_desc* first, int64_t n_first,
                                       const nvfp4_sweep_desc* second, int64_t n_second,
                                       const nvfp4_grouped_input* first_input,
                                       const nvfp4_grouped_input* second_input, int64_t experts,
                                       float* S, int lo, int hi) {
  std::vector<nvfp4_matrix_desc> md;
  bool w1 = false, w2 = false;
  const int st = check_grouped_layer(first, n_first, second, n_second, first_input, second_input,
                                     experts, S, &md, &w1, &w2);
  if (st != NVFP4_OK) return st;
  if (lo < -16 || lo > 0 || hi < 0 || hi > 15 || hi - lo > 15) return NVFP4_ERR_WINDOW;
  return grouped_layer_second_first(first, n_first, second, n_second, *first_input, *second_input,
                                    experts, lo, hi)
             ? 1
             : 0;
}

int nvfp4_quantize_grouped_layer(const nvfp4_sweep_desc* first, int64_t n_first,
                                 const nvfp4_sweep_desc* second, int64_t n_second,
                                 const nvfp4_grouped_input* first_input,
                                 const nvfp4_grouped_input* second_input, int64_t experts,
                                 float q_max, int lo, int hi, float* S, float* amax, int* status,
                                 void* workspace, size_t workspace_bytes,
                                 void* const* sweep_events, void* stream) {
  NVFP4_RANGE("nvfp4_quantize_grouped_layer");
  std::vector<nvfp4_matrix_desc> md;
  bool w1 = false, w2 = false;
  int st = check_grouped_layer(first, n_first, second, n_second, first_input, second_input,
                               experts, S, &md, &w1, &w2);
  if (st != NVFP4_OK) return st;
  if (!std::isfinite(q_max) || !(q_max > 0.0f)) return NVFP4_ERR_INVALID_ARG;
  if (lo < -16 || lo > 0 || hi < 0 || hi > 15 || hi - lo > 15) return NVFP4_ERR_WINDOW;
  if (!aligned(amax, 4) || !aligned(status, 4)) return NVFP4_ERR_ALIGN;
  if (sweep_events != nullptr)
    for (int k = 0; k < 4; ++k)
      if (sweep_events[k] == nullptr) return NVFP4_ERR_INVALID_ARG;
  if (workspace == nullptr) return NVFP4_ERR_WORKSPACE;
  if (!aligned(workspace, 256)) return NVFP4_ERR_ALIGN;
  if ((st = refuse_capture(static_cast<cudaStream_t>(stream))) != NVFP4_OK) return st;
  const int sms = current_sm_count();
  if (sms <= 0) return cuda_status(cudaErrorNoDevice);
  const GroupedLayerLayout L =
      grouped_layer_layout(n_first, n_second, first_input, second_input, experts, md, sms);
  if (workspace_bytes < L.bytes) return NVFP4_ERR_WORKSPACE;
  char* ws = static_cast<char*>(workspace);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const nvfp4_grouped_input& x1 = *first_input;
  const nvfp4_grouped_input& x2 = *second_input;
  // a: the batch swept first, its input's h computed on its own beforehand;
  // b: the batch swept second, its input's h streamed beside a's sweep
  const bool swap = grouped_layer_second_first(first, n_first, second, n_second, x1, x2, experts,
                                               lo, hi);
  const nvfp4_sweep_desc* da = swap ? second : first;
  const nvfp4_sweep_desc* db = swap ? first : second;
  const int64_t na = swap ? n_second : n_first, nb = swap ? n_first : n_second;
  const bool wa = swap ? w2 : w1, wb = swap ? w1 : w2;
  const nvfp4_grouped_input& xa = swap ? x2 : x1;
  const nvfp4_grouped_input& xb = swap ? x1 : x2;
  char* const gda = ws + (swap ? L.gd2 : L.gd1);
  char* const gdb = ws + (swap ? L.gd1 : L.gd2);
  const size_t swa = swap ? L.sw2 : L.sw1, swb = swap ? L.sw1 : L.sw2;
  const int eva = swap ? 2 : 0, evb = swap ? 0 : 2;  // sweep_events pairs: first's, second's
  auto fail = [](cudaError_t e) { return e != cudaSuccess; };
  cudaError_t e;
  // 1. h of a's input (a's sweep needs it), b's input's slice plan, and every
  //    matrix's S
  if (fail(e = nvfp4::launch_diag_hessian_grouped(static_cast<const uint16_t*>(xa.X),
                                                  xa.row_offsets, experts, xa.total_tokens, xa.in,
                                                  xa.ldx, xa.h, 0, gda, sms, s)))
    return cuda_status(e);
  const nvfp4::GroupedSide gb = nvfp4::grouped_diag_side(experts, xb.in, gdb, sms);
  if (fail(e = nvfp4::launch_grouped_diag_plan(xb.row_offsets, experts, xb.total_tokens, gb, s)))
    return cuda_status(e);
  const int64_t nm = static_cast<int64_t>(md.size());
  if (nm > 0) {
    nvfp4::MatDesc* gd = reinterpret_cast<nvfp4::MatDesc*>(ws + L.gs);
    if (fail(e = cudaMemcpyAsync(gd, L.gsp.d.data(), static_cast<size_t>(nm) * sizeof(nvfp4::MatDesc),
                                 cudaMemcpyHostToDevice, s)))
      return cuda_status(e);
    uint32_t* partial = reinterpret_cast<uint32_t*>(
        ws + L.gs + round256(static_cast<size_t>(nm) * sizeof(nvfp4::MatDesc)));
    if (fail(e = nvfp4::launch_global_scale_batched(gd, nm, L.gsp.total_ctas, q_max, S, amax,
                                                    status, partial, s)))
      return cuda_status(e);
  }
  // 2. a's sweep, its CTAs' fifth warp streaming b's input's partials (the
  //    grouped kernel's tasks: slice x vector)
  nvfp4::SideWork side{};
  side.n = 0;
  side.tasks = 0;
  if (xb.total_tokens > 0) {
    nvfp4::SideJob& j = side.job[side.n++];
    j.A = static_cast<const uint16_t*>(xb.X);
    j.rows = xb.total_tokens;
    j.ld = xb.ldx;
    j.cols = xb.in;
    j.P = gb.P;
    j.off = xb.row_offsets;
    j.cstart = gb.cstart;
    j.E = experts;
    j.block = gb.block;
    j.kind = 2;
    j.t0 = 0;
    j.t1 = gb.cap * (xb.in / 8);
    side.tasks = j.t1;
  }
  auto record = [&](int k) -> cudaError_t {
    return sweep_events != nullptr ? cudaEventRecord(static_cast<cudaEvent_t>(sweep_events[k]), s)
                                   : cudaSuccess;
  };
  auto sweep_batch = [&](const nvfp4_sweep_desc* d, int64_t n, bool weighted, size_t off,
                         bool carry) -> cudaError_t {
    if (n == 0) return cudaSuccess;
    std::vector<int64_t> groups(n);
    for (int64_t i = 0; i < n; ++i) groups[i] = d[i].out * (d[i].in / 16);
    std::vector<nvfp4::SweepDesc> dv;
    const int64_t per_sm = carry ? 4 : nvfp4::sweep_resident_ctas(weighted);
    const int64_t total = plan_sweep_batch(d, n, groups, 8 * static_cast<int64_t>(sms) * per_sm, &dv);
    nvfp4::SweepDesc* dd = reinterpret_cast<nvfp4::SweepDesc*>(ws + off);
    cudaError_t c = cudaMemcpyAsync(dd, dv.data(), static_cast<size_t>(n) * sizeof(nvfp4::SweepDesc),
                                    cudaMemcpyHostToDevice, s);
    if (c != cudaSuccess) return c;
    return carry ? nvfp4::launch_scale_sweep_batched_side(dd, n, total, weighted, lo, hi, side, s)
                 : nvfp4::launch_scale_sweep_batched(dd, n, total, weighted, lo, hi, s);
  };
  const bool carry = na > 0 && side.tasks > 0;
  if (fail(e = record(eva)) || fail(e = sweep_batch(da, na, wa, swa, carry)) ||
      fail(e = record(eva + 1)))
    return cuda_status(e);
  if (!carry && xb.total_tokens > 0) {
    // nothing to carry it: the grouped partial pass on its own
    if (fail(e = nvfp4::launch_diag_hessian_grouped(static_cast<const uint16_t*>(xb.X),
                                                    xb.row_offsets, experts, xb.total_tokens,
                                                    xb.in, xb.ldx, xb.h, 0, gdb, sms, s)))
      return cuda_status(e);
  } else if (fail(e = nvfp4::launch_grouped_diag_finalize(experts, xb.in, xb.h, 0, gb, s))) {
    return cuda_status(e);
  }
  // 3. b's sweep
  if (fail(e = record(evb)) || fail(e = sweep_batch(db, nb, wb, swb, false)) ||
      fail(e = record(evb + 1)))
    return cuda_status(e);
  return NVFP4_OK;
}

}  // extern "C"
