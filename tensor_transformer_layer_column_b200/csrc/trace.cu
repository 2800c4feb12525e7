// Optional launch tracing for measurement tools (tp_trace_begin / tp_trace_end).
//
// While a trace is open, every kernel the library enqueues is bracketed by two
// caller-created CUDA events recorded on the launch stream, and its class and
// algorithmic FLOP count are written to caller arrays.  Closed, it costs one
// relaxed atomic load per launch.
#include <cuda_runtime.h>

#include <atomic>
#include <mutex>

#include "internal.h"

namespace tp {

namespace {

struct TraceState {
  std::mutex mu;
  std::atomic<bool> on{false};
  cudaEvent_t* events = nullptr;
  int* kinds = nullptr;
  double* flops = nullptr;
  int capacity = 0;
  int count = 0;      // launches seen while open (may exceed capacity)
};

TraceState& state() {
  static TraceState s;
  return s;
}

}  // namespace

TraceScope::TraceScope(cudaStream_t stream, int kind, double flops) : stream_(stream), slot_(-1) {
  TraceState& s = state();
  if (!s.on.load(std::memory_order_relaxed)) return;
  std::lock_guard<std::mutex> lk(s.mu);
  if (!s.on.load(std::memory_order_relaxed)) return;
  const int i = s.count++;
  if (i >= s.capacity) return;
  slot_ = i;
  s.kinds[i] = kind;
  if (s.flops) s.flops[i] = flops;
  cudaEventRecord(s.events[2 * i], stream_);
}

TraceScope::~TraceScope() {
  if (slot_ < 0) return;
  TraceState& s = state();
  std::lock_guard<std::mutex> lk(s.mu);
  if (s.events) cudaEventRecord(s.events[2 * slot_ + 1], stream_);
}

}  // namespace tp

extern "C" {

tp_status tp_trace_begin(void* const* events, int* kinds, double* flops, int capacity) {
  tp::TraceState& s = tp::state();
  std::lock_guard<std::mutex> lk(s.mu);
  if (capacity < 0 || (capacity > 0 && (!events || !kinds))) return TP_ERR_INVALID_ARG;
  s.events = reinterpret_cast<cudaEvent_t*>(const_cast<void**>(events));
  s.kinds = kinds;
  s.flops = flops;
  s.capacity = capacity;
  s.count = 0;
  s.on.store(capacity > 0, std::memory_order_relaxed);
  return TP_OK;
}

int tp_trace_end(void) {
  tp::TraceState& s = tp::state();
  std::lock_guard<std::mutex> lk(s.mu);
  const int n = s.count;
  s.on.store(false, std::memory_order_relaxed);
  s.events = nullptr;
  s.kinds = nullptr;
  s.flops = nullptr;
  s.capacity = 0;
  s.count = 0;
  return n;
}

}  // extern "C"
