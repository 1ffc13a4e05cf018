// Shared device helpers for libhga (element loads, block-wide scans, the
// per-device status word).  Everything here is compiled into one translation
// unit (libhga.cu), so the status word needs no relocatable device code.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "hga.h"

namespace hga {

constexpr int kBlock = HGA_BLOCK;
constexpr int kGroup = HGA_GROUP;
constexpr int kQBlock = HGA_QBLOCK;
constexpr int kGroupsPerBlock = kBlock / kGroup;

// Latched device-side status (first error wins); read by hga_get_device_status.
__device__ int g_device_status = 0;

__device__ __forceinline__ void latch_status(int code) {
  atomicCAS(&g_device_status, 0, code);
}

// Programmatic dependent launch.  The hot-path kernels are launched with
// programmatic stream serialization: pdl_launch_dependents() lets the next
// kernel on the stream be scheduled once every CTA of this grid has run it
// (so no CTA of this grid can be kept off an SM by its dependents), and
// pdl_wait() blocks until the previous kernel has completed and its writes
// are visible.  Every thread calls pdl_wait() before its first access to
// global memory that a previous kernel may write or read.  Both are no-ops
// in a launch without the attribute.
__device__ __forceinline__ void pdl_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// Per-item completion flags between the kernels of one fused call: the
// producing CTA stores the call's token with release semantics after its
// writes (every writing thread fenced first); the consuming thread waits,
// bounded, until it reads the token with acquire semantics.  On timeout it
// latches HGA_ERR_TIMEOUT, raises *abort and returns false.
__device__ __forceinline__ void flag_release(int* flag, uint32_t token) {
  asm volatile("st.release.gpu.global.b32 [%0], %1;" ::"l"(flag), "r"(token) : "memory");
}

__device__ __forceinline__ bool flag_wait(const int* flag, uint32_t token, volatile int* abort,
                                          long long limit_cycles = 2000000000LL) {
  const long long t0 = clock64();
  while (true) {
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(flag) : "memory");
    if (v == token) return true;
    if (*abort) return false;
    if (clock64() - t0 > limit_cycles) {
      latch_status(HGA_ERR_TIMEOUT);
      *abort = 1;
      return false;
    }
    __nanosleep(100);
  }
}

// ---------------------------------------------------------------------------
// element loads: 8 consecutive elements -> 8 floats (16 B for bf16, 32 B for f32)
// ---------------------------------------------------------------------------
__device__ __forceinline__ void load8(const __nv_bfloat16* p, float* f) {
  uint4 u = *reinterpret_cast<const uint4*>(p);
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
  }
}

__device__ __forceinline__ void load8(const float* p, float* f) {
  float4 a = reinterpret_cast<const float4*>(p)[0];
  float4 b = reinterpret_cast<const float4*>(p)[1];
  f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w;
  f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
}

// 8 consecutive elements as loaded (kept raw until used, so that many rows'
// loads can be in flight in few registers), and their addition to 8 float
// sums in element order
template <typename T>
struct Raw8;
template <>
struct Raw8<__nv_bfloat16> {
  uint4 u;
  __device__ __forceinline__ void load(const __nv_bfloat16* p) {
    u = *reinterpret_cast<const uint4*>(p);
  }
  __device__ __forceinline__ void add_to(float* acc) const {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      acc[2 * i] += __uint_as_float(w[i] << 16);
      acc[2 * i + 1] += __uint_as_float(w[i] & 0xffff0000u);
    }
  }
  __device__ __forceinline__ void get(float* f) const {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      f[2 * i] = __uint_as_float(w[i] << 16);
      f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
  }
};
template <>
struct Raw8<float> {
  float4 a, b;
  __device__ __forceinline__ void load(const float* p) {
    a = reinterpret_cast<const float4*>(p)[0];
    b = reinterpret_cast<const float4*>(p)[1];
  }
  __device__ __forceinline__ void add_to(float* acc) const {
    acc[0] += a.x; acc[1] += a.y; acc[2] += a.z; acc[3] += a.w;
    acc[4] += b.x; acc[5] += b.y; acc[6] += b.z; acc[7] += b.w;
  }
  __device__ __forceinline__ void get(float* f) const {
    f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w;
    f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
  }
};

__device__ __forceinline__ float to_float(__nv_bfloat16 x) { return __bfloat162float(x); }
__device__ __forceinline__ float to_float(float x) { return x; }

template <typename T> __device__ __forceinline__ T from_float(float x);
template <> __device__ __forceinline__ float from_float<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_float<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

__device__ __forceinline__ void store8(float* p, const float* f) {
  reinterpret_cast<float4*>(p)[0] = make_float4(f[0], f[1], f[2], f[3]);
  reinterpret_cast<float4*>(p)[1] = make_float4(f[4], f[5], f[6], f[7]);
}

__device__ __forceinline__ void store8(__nv_bfloat16* p, const float* f) {
  uint32_t w[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    __nv_bfloat162 h = __floats2bfloat162_rn(f[2 * i], f[2 * i + 1]);
    w[i] = *reinterpret_cast<uint32_t*>(&h);
  }
  *reinterpret_cast<uint4*>(p) = make_uint4(w[0], w[1], w[2], w[3]);
}

// ---------------------------------------------------------------------------
// Key-tile schedule of one query block, built by one full warp into shared
// memory: the causal own block first (tile 0: it needs no selection, so its
// K/V can be requested before the selection is read), then the valid
// selected groups in their (ascending) order, 8 per tile, the last routed
// tile padded with the own block's first group (masked out by tile_mask).
// An index that is neither -1 nor an earlier group latches
// HGA_ERR_DEVICE_CHECK and is skipped.  All of the row's loads are issued
// before the first is used (topk_groups <= 256: 8 per lane).
// ---------------------------------------------------------------------------
template <typename SH>
__device__ __forceinline__ void build_tile_schedule(SH& sh, const int32_t* srow, int topk_groups,
                                                    int64_t own_blk, int lane) {
  constexpr int kRounds = 8;
  int gv[kRounds];
#pragma unroll
  for (int i = 0; i < kRounds; ++i) {
    const int idx = i * 32 + lane;
    gv[i] = idx < topk_groups ? srow[idx] : -1;
  }
  const int own0 = int(own_blk * kGroupsPerBlock);
  int* routed = sh.grp + kGroupsPerBlock;
  int n_valid = 0;
#pragma unroll
  for (int i = 0; i < kRounds; ++i) {
    const int idx = i * 32 + lane, g = gv[i];
    bool ok = false;
    if (idx < topk_groups && g != -1) {
      ok = g >= 0 && int64_t(g) < own_blk * kGroupsPerBlock;
      if (!ok) latch_status(HGA_ERR_DEVICE_CHECK);
    }
    const unsigned ball = __ballot_sync(0xffffffffu, ok);
    if (ok) routed[n_valid + __popc(ball & ((1u << lane) - 1u))] = g;
    n_valid += __popc(ball);
  }
  __syncwarp();
  const int n_rt = (n_valid + 7) / 8;
  for (int i = n_valid + lane; i < n_rt * 8; i += 32) routed[i] = own0;
  for (int t = lane; t < n_rt; t += 32) {
    const int left = n_valid - 8 * t;
    sh.tile_mask[1 + t] = left >= 8 ? 0xffu : uint8_t((1u << left) - 1u);
  }
  for (int i = lane; i < kGroupsPerBlock; i += 32) sh.grp[i] = own0 + i;
  if (lane == 0) {
    sh.tile_mask[0] = 0xffu;
    sh.n_tiles = n_rt + 1;
  }
}

// ---------------------------------------------------------------------------
// order-preserving float -> uint32 key (larger float -> larger key; -0 == +0)
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t ordered_key(float f) {
  uint32_t u = __float_as_uint(f);
  if ((u & 0x7fffffffu) == 0u) u = 0u;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// ---------------------------------------------------------------------------
// block-wide, order-preserving enumeration of a predicate over [0, n):
// calls f(i, rank) for each i with pred(i), rank = number of earlier i with
// pred.  Each thread owns a contiguous chunk, so ranks follow index order.
// Needs `scratch` of at least (blockDim.x/32 + 1) ints in shared memory.
// Returns the total count (same value in every thread).
// ---------------------------------------------------------------------------
template <typename Pred, typename Fn>
__device__ int block_enumerate(int n, Pred pred, Fn f, int* scratch) {
  const int nt = blockDim.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nwarps = nt >> 5;
  const int chunk = (n + nt - 1) / nt;
  const int lo = min(n, tid * chunk), hi = min(n, lo + chunk);
  int cnt = 0;
  for (int i = lo; i < hi; ++i) cnt += pred(i) ? 1 : 0;
  int incl = cnt;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  if (lane == 31) scratch[warp] = incl;
  __syncthreads();
  if (tid == 0) {
    int run = 0;
    for (int w = 0; w < nwarps; ++w) {
      int v = scratch[w];
      scratch[w] = run;
      run += v;
    }
    scratch[nwarps] = run;
  }
  __syncthreads();
  int rank = scratch[warp] + incl - cnt;
  for (int i = lo; i < hi; ++i) {
    if (pred(i)) f(i, rank++);
  }
  int total = scratch[nwarps];
  __syncthreads();
  return total;
}

// The same contract for short ranges (a few times the block size): element
// i goes to thread i % blockDim.x in round i / blockDim.x, and its rank is
// the count of earlier predicates in that round (warp ballots, one table of
// per-warp counts) plus the counts of the earlier rounds.  Needs `scratch` of
// blockDim.x/32 ints.
template <typename Pred, typename Fn>
__device__ int block_enumerate_rounds(int n, Pred pred, Fn f, int* scratch) {
  const int nt = blockDim.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nwarps = nt >> 5;
  int done = 0;
  for (int base = 0; base < n; base += nt) {
    const int i = base + tid;
    const bool p = i < n && pred(i);
    const unsigned ball = __ballot_sync(0xffffffffu, p);
    if (lane == 0) scratch[warp] = __popc(ball);
    __syncthreads();
    int before = done, total = done;
    for (int w = 0; w < nwarps; ++w) {
      const int c = scratch[w];
      before += w < warp ? c : 0;
      total += c;
    }
    if (p) f(i, before + __popc(ball & ((1u << lane) - 1u)));
    done = total;
    __syncthreads();
  }
  return done;
}

// block_enumerate or block_enumerate_rounds, whichever takes fewer barriers
template <typename Pred, typename Fn>
__device__ int block_enumerate_any(int n, Pred pred, Fn f, int* scratch) {
  if (n <= 2 * int(blockDim.x)) return block_enumerate_rounds(n, pred, f, scratch);
  return block_enumerate(n, pred, f, scratch);
}

// ---------------------------------------------------------------------------
// block-wide top-k of n distinct-or-not uint32 keys held in shared memory:
// sets sel[i] = 1 for the k largest keys, ties broken toward the lower index.
// Up to blockDim.x keys: rank counting (below).  Otherwise a radix select on 8-bit
// digits (MSB first) finds the k-th largest key T; keys above T are taken,
// and among keys equal to T the lowest indices fill the remaining slots.
// Needs hist[256] and scratch (see block_enumerate).
// ---------------------------------------------------------------------------
__device__ void block_topk(const uint32_t* key, int n, int k, uint8_t* sel, int* hist,
                           int* scratch) {
  const int nt = blockDim.x, tid = threadIdx.x;
  if (k >= n) {
    for (int i = tid; i < n; i += nt) sel[i] = 1;
    __syncthreads();
    return;
  }
  if (n <= nt) {
    // rank by counting: rank(i) = #{keys above key[i]} + #{equal keys before i};
    // the k smallest ranks are the k largest keys, ties to the lower index.
    // P consecutive lanes share a key (P = the largest power of two, at most
    // 32, with P * n <= threads), each counting over a quarter-aligned slice
    // of the keys with broadcast 16-byte shared-memory reads (`key` is
    // 16-byte aligned); the slices' counts are added by shuffles.  No barrier
    // until the flags are written.
    int P = 1;
    while (P < 32 && 2 * P * n <= nt) P *= 2;
    const int i = tid / P, part = tid % P;
    const int chunk = (((n + P - 1) / P) + 3) & ~3;
    const int j0 = part * chunk < n ? part * chunk : n;
    const int j1 = j0 + chunk < n ? j0 + chunk : n;
    const uint32_t ki = i < n ? key[i] : 0u;
    int rank = 0;
    if (i < n) {
      const uint4* key4 = reinterpret_cast<const uint4*>(key);
      const int q1 = j0 + ((j1 - j0) & ~3);
#pragma unroll 4
      for (int jj = j0; jj < q1; jj += 4) {
        const uint4 v = key4[jj >> 2];
        rank += (v.x > ki) || (v.x == ki && jj < i);
        rank += (v.y > ki) || (v.y == ki && jj + 1 < i);
        rank += (v.z > ki) || (v.z == ki && jj + 2 < i);
        rank += (v.w > ki) || (v.w == ki && jj + 3 < i);
      }
      for (int jj = q1; jj < j1; ++jj) {
        const uint32_t kj = key[jj];
        rank += (kj > ki) || (kj == ki && jj < i);
      }
    }
    for (int o = 1; o < P; o <<= 1) rank += __shfl_xor_sync(0xffffffffu, rank, o);
    if (i < n && part == 0) sel[i] = rank < k ? 1 : 0;
    __syncthreads();
    return;
  }
  __shared__ uint32_t s_prefix, s_mask;
  __shared__ int s_remaining;
  if (tid == 0) { s_prefix = 0u; s_mask = 0u; s_remaining = k; }
  __syncthreads();
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
    for (int i = tid; i < 256; i += nt) hist[i] = 0;
    __syncthreads();
    const uint32_t prefix = s_prefix, mask = s_mask;
    // warp-aggregated: the lanes holding the same digit add their count once
    // (the top digits of nearby scores are mostly equal)
    for (int base = 0; base < n; base += nt) {
      const int i = base + tid;
      const uint32_t kk = i < n ? key[i] : 0u;
      const bool act = i < n && (kk & mask) == prefix;
      const unsigned am = __ballot_sync(0xffffffffu, act);
      if (act) {
        const uint32_t dg = (kk >> shift) & 255u;
        const unsigned peers = __match_any_sync(am, dg);
        if ((tid & 31) == __ffs(peers) - 1) atomicAdd(&hist[dg], __popc(peers));
      }
    }
    __syncthreads();
    if (tid < 32) {
      // lane l owns digits 255-8l .. 248-8l (descending); find the digit where
      // the running count from the top first reaches `remaining`.
      const int lane = tid;
      int local = 0;
#pragma unroll
      for (int t = 0; t < 8; ++t) local += hist[255 - 8 * lane - t];
      int incl = local;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        int v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
      }
      const int remaining = s_remaining;
      const int excl = incl - local;
      const bool mine = excl < remaining && incl >= remaining;
      const unsigned ball = __ballot_sync(0xffffffffu, mine);
      const int owner = __ffs(ball) - 1;
      if (lane == owner) {
        int above = excl;
        for (int t = 0; t < 8; ++t) {
          const int dgt = 255 - 8 * lane - t;
          const int c = hist[dgt];
          if (above + c >= remaining) {
            s_prefix = prefix | (uint32_t(dgt) << shift);
            s_mask = mask | (255u << shift);
            s_remaining = remaining - above;
            break;
          }
          above += c;
        }
      }
    }
    __syncthreads();
  }
  const uint32_t thr = s_prefix;
  const int need_equal = s_remaining;  // how many keys equal to thr are taken
  for (int i = tid; i < n; i += nt) sel[i] = key[i] > thr ? 1 : 0;
  __syncthreads();
  block_enumerate_any(
      n, [&](int i) { return key[i] == thr; },
      [&](int i, int rank) {
        if (rank < need_equal) sel[i] = 1;
      },
      scratch);
  __syncthreads();
}

// The float score behind an ordered key (inverse of ordered_key).
__device__ __forceinline__ float key_score(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}

// After block_topk: out[0] = the k-th largest score (the smallest chosen
// key), out[1] = the (k+1)-th (the largest key not chosen), both times
// `scale`; -inf where there is none (k = 0, or every key chosen; padding key
// 0 counts as none).  Every thread calls it; thread 0 writes out.
__device__ void kth_scores(const uint32_t* key, const uint8_t* sel, int n, float scale,
                           float* out) {
  __shared__ uint32_t s_lo, s_hi;
  if (threadIdx.x == 0) {
    s_lo = 0xffffffffu;
    s_hi = 0u;
  }
  __syncthreads();
  uint32_t lo = 0xffffffffu, hi = 0u;
  for (int i = threadIdx.x; i < n; i += blockDim.x) {
    const uint32_t k = key[i];
    if (sel[i]) lo = k < lo ? k : lo;
    else hi = k > hi ? k : hi;
  }
  if (lo != 0xffffffffu) atomicMin(&s_lo, lo);
  if (hi != 0u) atomicMax(&s_hi, hi);
  __syncthreads();
  if (threadIdx.x == 0 && out) {
    out[0] = s_lo == 0xffffffffu || s_lo == 0u ? -INFINITY : key_score(s_lo) * scale;
    out[1] = s_hi == 0u ? -INFINITY : key_score(s_hi) * scale;
  }
  __syncthreads();
}

// block_topk followed by the ascending list of the chosen indices:
// out[r] = the r-th smallest index among the top-k of key[0, n) (k <= n).
// Kept out of line: a kernel that selects several times runs one copy of
// this code, which stays in the instruction cache.
__device__ __noinline__ void block_topk_indices(const uint32_t* key, int n, int k, int* out,
                                                uint8_t* sel, int* hist, int* scratch,
                                                float scale = 0.f, float* scores = nullptr) {
  block_topk(key, n, k, sel, hist, scratch);
  if (scores) kth_scores(key, sel, n, scale, scores);
  block_enumerate_any(
      n, [&](int i) { return sel[i] != 0; }, [&](int i, int r) { out[r] = i; }, scratch);
  __syncthreads();
}

}  // namespace hga
