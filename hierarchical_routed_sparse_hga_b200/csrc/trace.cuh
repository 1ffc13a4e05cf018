// Launch counting and optional per-kernel CUDA-event timing (see the
// diagnostics section of hga.h).  Host-side only.
#pragma once

#include <cuda_runtime.h>

#include <atomic>
#include <mutex>
#include <vector>

#include "hga.h"

namespace hga {

struct TimingSlot {
  cudaEvent_t begin = nullptr, end = nullptr;
  int kind = 0;
};

struct Tracer {
  std::mutex mu;
  std::atomic<uint64_t> launches{0};
  bool on = false;
  std::vector<TimingSlot> slots;
  size_t next = 0;
  double ms[HGA_K_COUNT] = {};
  uint64_t count[HGA_K_COUNT] = {};
};

inline Tracer& tracer() {
  static Tracer t;
  return t;
}

inline cudaError_t record(cudaEvent_t ev, cudaStream_t s) {
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(s, &cs) != cudaSuccess) return cudaErrorUnknown;
  if (cs == cudaStreamCaptureStatusActive)
    return cudaEventRecordWithFlags(ev, s, cudaEventRecordExternal);
  return cudaEventRecord(ev, s);
}

// Runs `launch` (a kernel launch on stream s), counting it and, when timing
// is on, bracketing it with a pair of events.  Returns the launch status.
template <typename F>
hga_status_t traced_launch(int kind, cudaStream_t s, F&& launch) {
  Tracer& t = tracer();
  t.launches.fetch_add(1, std::memory_order_relaxed);
  TimingSlot* slot = nullptr;
  if (t.on) {
    std::lock_guard<std::mutex> lock(t.mu);
    if (t.next < t.slots.size()) {
      slot = &t.slots[t.next++];
      slot->kind = kind;
    }
  }
  if (slot && record(slot->begin, s) != cudaSuccess) return HGA_ERR_CUDA;
  launch();
  if (cudaGetLastError() != cudaSuccess) return HGA_ERR_CUDA;
  if (slot && record(slot->end, s) != cudaSuccess) return HGA_ERR_CUDA;
  return HGA_OK;
}

}  // namespace hga
