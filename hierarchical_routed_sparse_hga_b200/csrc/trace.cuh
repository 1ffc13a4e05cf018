// Launch counting and optional per-kernel CUDA-event timing (see the
// diagnostics section of hga.h).  Host-side only.
#pragma once

#include <cuda_runtime.h>

#include <atomic>
#include <mutex>
#include <type_traits>
#include <utility>
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
  uint32_t kinds = ~0u;  // kinds whose launches are bracketed (bit per kind)
  std::vector<TimingSlot> slots;
  size_t next = 0;
  double ms[HGA_K_COUNT] = {};
  uint64_t count[HGA_K_COUNT] = {};
};

inline Tracer& tracer() {
  static Tracer t;
  return t;
}

// The CUDA error behind the last HGA_ERR_CUDA a launch returned (per thread).
inline cudaError_t& last_launch_error() {
  static thread_local cudaError_t e = cudaSuccess;
  return e;
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
  if (t.on && ((t.kinds >> kind) & 1u)) {
    std::lock_guard<std::mutex> lock(t.mu);
    if (t.next < t.slots.size()) {
      slot = &t.slots[t.next++];
      slot->kind = kind;
    }
  }
  if (slot && record(slot->begin, s) != cudaSuccess) return HGA_ERR_CUDA;
  if constexpr (std::is_same_v<decltype(launch()), cudaError_t>) {
    const cudaError_t e = launch();
    if (e != cudaSuccess) {
      cudaGetLastError();
      last_launch_error() = e;
      return HGA_ERR_CUDA;
    }
  } else {
    launch();
  }
  if (const cudaError_t e = cudaGetLastError(); e != cudaSuccess) {
    last_launch_error() = e;
    return HGA_ERR_CUDA;
  }
  if (slot && record(slot->end, s) != cudaSuccess) return HGA_ERR_CUDA;
  return HGA_OK;
}

// Launches `kernel` on stream s with programmatic stream serialization, so
// that it may be scheduled while the kernel before it drains (the kernel
// itself orders its reads with pdl_wait()).  Returns the launch status.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t s, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

}  // namespace hga
