// row_counters.cu -- the counter slots of row_counters.cuh and their leases.
#include "row_counters.cuh"

namespace nvfp4 {

// Zero at module load; every launch that leases a slot leaves it zeroed again
// (apart from its count of launches served, kept for tests).
__device__ unsigned int g_row_counters[kCounterSlots][kSlotWords];

namespace {

// cuEventQuery, reached through the runtime so that the library needs no
// link to the driver library; unlike the runtime's query it leaves the
// runtime's last-error state alone while the event is pending.
using EventQueryFn = int (*)(cudaEvent_t);
EventQueryFn event_query() {
  static const EventQueryFn fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
    if (cudaGetDriverEntryPoint("cuEventQuery", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess) {
      cudaGetLastError();
      return static_cast<EventQueryFn>(nullptr);
    }
    return reinterpret_cast<EventQueryFn>(p);
  }();
  return fn;
}

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

// The slots of one device: a slot is leased to one launch at a time and is
// free again once the event recorded after that launch has completed.
struct CounterLease::Pool {
  std::mutex mu;
  unsigned int* base = nullptr;  // device address of g_row_counters
  cudaEvent_t ev[kCounterSlots] = {};
  bool leased[kCounterSlots] = {};
  bool retired[kCounterSlots] = {};
  int next = 0;

  // A free slot (its event created), or -1.  Called with mu held.
  int acquire() {
    if (base == nullptr) {
      void* p = nullptr;
      if (cudaGetSymbolAddress(&p, g_row_counters) != cudaSuccess) {
        cudaGetLastError();
        return -1;
      }
      base = static_cast<unsigned int*>(p);
    }
    const EventQueryFn query = event_query();
    if (query == nullptr) return -1;
    for (int k = 0; k < kCounterSlots; ++k) {
      const int i = (next + k) % kCounterSlots;
      if (ev[i] == nullptr) {
        if (cudaEventCreateWithFlags(&ev[i], cudaEventDisableTiming) != cudaSuccess) {
          cudaGetLastError();
          ev[i] = nullptr;
          return -1;
        }
        leased[i] = false;
      }
      if (retired[i] || (leased[i] && query(ev[i]) != 0)) continue;  // pending or failed
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
  if (index_ >= 0) slot_ = pool_->base + static_cast<size_t>(index_) * kSlotWords;
}

cudaError_t CounterLease::commit(cudaError_t launch_status) {
  if (slot_ == nullptr || launch_status != cudaSuccess) return launch_status;
  // if the event cannot be recorded nothing would tell when the slot is
  // free again, so it is retired
  if (cudaEventRecord(pool_->ev[index_], stream_) != cudaSuccess) {
    pool_->retired[index_] = true;
    return cudaGetLastError();
  }
  pool_->leased[index_] = true;
  return cudaSuccess;
}

cudaError_t row_counters_symbol(void** ptr, size_t* bytes) {
  *bytes = sizeof(g_row_counters);
  return cudaGetSymbolAddress(ptr, g_row_counters);
}

}  // namespace nvfp4
