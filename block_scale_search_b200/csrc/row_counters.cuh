// row_counters.cuh -- run-time work hand-out for kernels whose warps would
// otherwise take a fixed share of rows.
//
// With a fixed share per thread, the warps a scheduler favours finish early
// and leave their SMs short of warps for the rest of the launch.  Instead,
// warps take their next rows from a counter in device memory as they finish,
// so that every warp of the grid ends at about the same time.  The counters
// form a small pool of slots that launches take in turn (CounterLease): a
// launch's stream first waits for the slot's previous launch, and the
// launch's last CTA zeroes the slot for the next (finish_slot).
#pragma once

#include <mutex>

#include <cuda_runtime.h>

namespace nvfp4 {

constexpr int kCounterSlots = 64;           // slots, taken in turn
constexpr int kSlotCounters = 256;          // counters a launch may use
constexpr int kSlotWords = kSlotCounters + 2;  // counters, CTAs done, launches served

// Called by every thread of every CTA of a launch that holds `slot`, after
// the CTA's last hand-out: the CTA that finishes last zeroes the first
// `used` counters and the done count, and counts the launch as served.
__device__ __forceinline__ void finish_slot(unsigned int* slot, int used) {
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    if (atomicAdd(slot + kSlotCounters, 1u) == gridDim.x - 1) {
      for (int i = 0; i < used; ++i) slot[i] = 0u;
      slot[kSlotCounters] = 0u;
      slot[kSlotCounters + 1] += 1u;
      __threadfence();
    }
  }
}

// One launch's lease of a counter slot on the current device.  Construct it
// right before the launch (want = false: no lease), pass slot() (null: no
// slot -- stream capture or a CUDA error; keep the fixed share) to the
// kernel, and call commit() with the launch's status right after.  The pool's
// mutex is held from construction to destruction.
class CounterLease {
 public:
  CounterLease(cudaStream_t stream, bool want);
  ~CounterLease() = default;
  CounterLease(const CounterLease&) = delete;
  CounterLease& operator=(const CounterLease&) = delete;
  unsigned int* slot() const { return slot_; }
  // Records the event that frees the slot once the launch has completed.
  cudaError_t commit(cudaError_t launch_status);

 private:
  struct Pool;
  Pool* pool_ = nullptr;
  cudaStream_t stream_ = nullptr;
  std::unique_lock<std::mutex> lock_;
  int index_ = -1;
  unsigned int* slot_ = nullptr;
};

// Address and size of the counter slots on the current device.
cudaError_t row_counters_symbol(void** ptr, size_t* bytes);

}  // namespace nvfp4
