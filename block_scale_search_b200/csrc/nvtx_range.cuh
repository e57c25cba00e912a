// nvtx_range.cuh -- an NVTX range around each entry point, so that a profiler
// timeline (Nsight Systems, or ncu's --nvtx filters) shows which library call
// enqueued which kernels.  NVTX3 is header-only: with no profiler attached the
// push and pop are a check of a function pointer and return at once.  Build
// with -DNVFP4HS_NO_NVTX to leave them out entirely.
#pragma once

#ifndef NVFP4HS_NO_NVTX
#include <nvtx3/nvToolsExt.h>

namespace nvfp4 {
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};
}  // namespace nvfp4
#define NVFP4_RANGE(name) ::nvfp4::NvtxRange nvfp4_nvtx_range_(name)
#else
#define NVFP4_RANGE(name) ((void)0)
#endif
