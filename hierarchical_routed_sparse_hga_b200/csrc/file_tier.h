// Step a7, third tier: history K/V in files (NVMe), read back per segment.
// ("Long-Context Fine-Tuning with Limited VRAM", adnankhan.ai notes, section
// "Raw Abstract / Excerpt": older KV is detached into RAM or NVMe; the
// seventnews page, section "意义何在": NVMe-backed tiered storage is
// implemented there but not benchmarked.)
//
// Host-side code only.  A K or V file holds the whole context in the layout
// of the device buffers, [batch, n_kv_heads, ctx_cap, head_dim] elements, so
// one 8-token group is one contiguous run of 8 * head_dim elements (2 KiB for
// bf16, d = 128) at offset ((b * Hkv + h) * ctx_cap + 8 g) * row bytes.
// Reads and writes run on a pool of threads that take runs of consecutive
// groups (consecutive in the file and in the staging buffer) from a shared
// counter and issue one pread / pwrite per run, retrying short transfers.
#pragma once

#include <stdint.h>
#include <unistd.h>

#include <algorithm>
#include <atomic>
#include <cerrno>
#include <thread>
#include <vector>

namespace hga {
namespace file_tier {

struct Run {
  int64_t file_off;   // bytes
  int64_t mem_off;    // bytes
  int64_t bytes;
};

// Reads (or writes) `bytes` at `off`, retrying on EINTR and short counts.
inline bool full_pread(int fd, char* dst, int64_t bytes, int64_t off) {
  while (bytes > 0) {
    const ssize_t n = pread(fd, dst, size_t(bytes), off);
    if (n < 0 && errno == EINTR) continue;
    if (n <= 0) return false;
    dst += n;
    off += n;
    bytes -= n;
  }
  return true;
}

inline bool full_pwrite(int fd, const char* src, int64_t bytes, int64_t off) {
  while (bytes > 0) {
    const ssize_t n = pwrite(fd, src, size_t(bytes), off);
    if (n < 0 && errno == EINTR) continue;
    if (n <= 0) return false;
    src += n;
    off += n;
    bytes -= n;
  }
  return true;
}

// Runs every transfer of `runs` for both files (K and V: the same offsets in
// the two files and the two buffers) on `n_threads` threads.  Returns false
// if any transfer failed.
template <bool kWrite>
inline bool transfer(const std::vector<Run>& runs, int fd_k, int fd_v, char* mem_k, char* mem_v,
                     int n_threads) {
  std::atomic<size_t> next{0};
  std::atomic<bool> ok{true};
  auto work = [&] {
    while (ok.load(std::memory_order_relaxed)) {
      const size_t i = next.fetch_add(1, std::memory_order_relaxed);
      if (i >= 2 * runs.size()) return;
      const Run& r = runs[i >> 1];
      const bool is_v = i & 1;
      const int fd = is_v ? fd_v : fd_k;
      char* mem = (is_v ? mem_v : mem_k) + r.mem_off;
      const bool done = kWrite ? full_pwrite(fd, mem, r.bytes, r.file_off)
                               : full_pread(fd, mem, r.bytes, r.file_off);
      if (!done) ok.store(false, std::memory_order_relaxed);
    }
  };
  const int nt = std::max(1, std::min(n_threads, int(2 * runs.size())));
  std::vector<std::thread> pool;
  pool.reserve(size_t(nt > 1 ? nt - 1 : 0));
  for (int t = 1; t < nt; ++t) pool.emplace_back(work);
  work();
  for (auto& t : pool) t.join();
  return ok.load();
}

}  // namespace file_tier
}  // namespace hga
