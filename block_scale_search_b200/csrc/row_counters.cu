// row_counters.cu -- the counter slots of row_counters.cuh and their leases.
#include "row_counters.cuh"

namespace nvfp4 {

// Zero at module load; every launch that takes a slot leaves it zeroed again
// (apart from its count of launches served, kept for tests).
__device__ unsigned int g_row_counters[kCounterSlots][kSlotWords];

namespace {

// A launch recorded into a graph may be replayed any number of times, also
// concurrently, so captured launches keep the fixed share.
bool capturing(cudaStream_t s) {
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(s, &cs) != cudaSuccess) {
    cudaGetLastError();
    return true;
  }
  return cs != cudaStreamCaptureStatusNone;
}

}  // namespace

// The slots of one device, handed out in turn.  A launch that takes a slot
// first makes its stream wait for the event recorded after the slot's
// previous launch: on the same stream that costs nothing (stream order), on
// another it orders the two launches, so two launches never share a slot at
// the same time and no launch is ever refused one.
struct CounterLease::Pool {
  std::mutex mu;
  unsigned int* base = nullptr;  // device address of g_row_counters
  cudaEvent_t ev[kCounterSlots] = {};
  bool used[kCounterSlots] = {};
  bool retired[kCounterSlots] = {};
  int next = 0;

  // The next usable slot (its event created), or -1.  Called with mu held.
  int acquire() {
    if (base == nullptr) {
      void* p = nullptr;
      if (cudaGetSymbolAddress(&p, g_row_counters) != cudaSuccess) {
        cudaGetLastError();
        return -1;
      }
      base = static_cast<unsigned int*>(p);
    }
    for (int k = 0; k < kCounterSlots; ++k) {
      const int i = (next + k) % kCounterSlots;
      if (retired[i]) continue;
      if (ev[i] == nullptr &&
          cudaEventCreateWithFlags(&ev[i], cudaEventDisableTiming) != cudaSuccess) {
        cudaGetLastError();
        ev[i] = nullptr;
        return -1;
      }
      next = (i + 1) % kCounterSlots;
      return i;
    }
    return -1;
  }
};

CounterLease::CounterLease(cudaStream_t stream, bool want) : stream_(stream) {
  static Pool pools[128];
  if (!want || capturing(stream)) return;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 128) {
    cudaGetLastError();
    return;
  }
  pool_ = &pools[dev];
  lock_ = std::unique_lock<std::mutex>(pool_->mu);
  index_ = pool_->acquire();
  if (index_ < 0) return;
  if (pool_->used[index_] && cudaStreamWaitEvent(stream, pool_->ev[index_], 0) != cudaSuccess) {
    cudaGetLastError();
    index_ = -1;
    return;
  }
  slot_ = pool_->base + static_cast<size_t>(index_) * kSlotWords;
}

cudaError_t CounterLease::commit(cudaError_t launch_status) {
  if (slot_ == nullptr || launch_status != cudaSuccess) return launch_status;
  // if the event cannot be recorded, the slot's next user could not wait for
  // this launch, so the slot is retired
  if (cudaEventRecord(pool_->ev[index_], stream_) != cudaSuccess) {
    pool_->retired[index_] = true;
    return cudaGetLastError();
  }
  pool_->used[index_] = true;
  return cudaSuccess;
}

cudaError_t row_counters_symbol(void** ptr, size_t* bytes) {
  *bytes = sizeof(g_row_counters);
  return cudaGetSymbolAddress(ptr, g_row_counters);
}

}  // namespace nvfp4
