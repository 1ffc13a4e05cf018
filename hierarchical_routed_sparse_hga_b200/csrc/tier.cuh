// Step a7: the host tier.  History K/V live in pinned host memory (the
// adnankhan.ai notes, section "Raw Abstract / Excerpt": older KV is detached
// into RAM or NVMe and HGA loads a bounded set of exact historical tokens per
// query block; seventnews "BMW如何…" intro: old keys and values move to RAM).
//
// Per segment and (batch, KV head) the groups that any query block of the
// segment selected from the history are deduplicated, copied over PCIe into a
// compact HBM staging buffer, and the selection is rewritten to staging-local
// indices, so the unchanged attention kernels run on the staging buffer:
//
//   staging rows [0, 8U)                    the U unique history groups, in
//                                           ascending global order
//   staging rows [stage_cap - s_len, ...)   the active segment (placed there by
//                                           the caller)
//
// tier_dedup_kernel  one CTA per (b, h): marks the selected history groups in
//                    a shared-memory bitmap, ranks them with a block scan
//                    (slot = number of marked groups below it), writes the
//                    remapped selection and the slot -> group list;
// tier_copy_kernel   one warp per group: 2 KiB of K and 2 KiB of V read from
//                    pinned host memory (zero-copy, 16-byte loads, all issued
//                    before the stores) and written to the staging slot.
#pragma once

#include "hga_common.cuh"

namespace hga {

constexpr int kTierThreads = 512;
constexpr int kTierCopyWarps = 8;

// Remapped value for a selection entry that is not a valid routed group;
// the attention kernels reject it (and latch HGA_ERR_DEVICE_CHECK).
constexpr int32_t kTierInvalid = -2;

template <int D>
__global__ void __launch_bounds__(kTierThreads)
    tier_dedup_kernel(const int32_t* __restrict__ sel_grp, int n_kv_heads, int n_qb,
                      int topk_groups, int64_t q_begin, int64_t stage_cap, int s_len,
                      int32_t* __restrict__ sel_stage, int32_t* __restrict__ slot_group,
                      int32_t* __restrict__ n_unique, int64_t slot_cap) {
  extern __shared__ uint32_t bitmap[];  // one bit per history group
  __shared__ int scratch[kTierThreads / 32 + 1];
  const int h = blockIdx.x, b = blockIdx.y;
  const int64_t head = int64_t(b) * n_kv_heads + h;
  const int64_t n_hist = q_begin / kGroup;             // history groups
  const int n_words = int((n_hist + 31) / 32);
  const int64_t act0 = (stage_cap - s_len) / kGroup;   // staging group of the segment start
  const int64_t seg0 = q_begin / kGroup;
  const int32_t* sel = sel_grp + head * n_qb * topk_groups;
  int32_t* out = sel_stage + head * n_qb * topk_groups;
  const int n = n_qb * topk_groups;

  for (int w = threadIdx.x; w < n_words; w += blockDim.x) bitmap[w] = 0u;
  __syncthreads();
  for (int i = threadIdx.x; i < n; i += blockDim.x) {
    const int g = sel[i];
    if (g >= 0 && g < n_hist) atomicOr(&bitmap[g >> 5], 1u << (g & 31));
  }
  __syncthreads();
  // exclusive prefix of the per-word popcounts, in word order: word_off[w]
  // is the slot of the lowest marked group of word w
  int* word_off = reinterpret_cast<int*>(bitmap + n_words);
  {
    const int nt = blockDim.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int chunk = (n_words + nt - 1) / nt;
    const int lo = min(n_words, tid * chunk), hi = min(n_words, lo + chunk);
    int cnt = 0;
    for (int w = lo; w < hi; ++w) cnt += __popc(bitmap[w]);
    int incl = cnt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    if (lane == 31) scratch[warp] = incl;
    __syncthreads();
    if (tid == 0) {
      int run = 0;
      for (int w = 0; w < nt / 32; ++w) {
        const int v = scratch[w];
        scratch[w] = run;
        run += v;
      }
      scratch[nt / 32] = run;
    }
    __syncthreads();
    int run = scratch[warp] + incl - cnt;
    for (int w = lo; w < hi; ++w) {
      word_off[w] = run;
      run += __popc(bitmap[w]);
    }
  }
  __syncthreads();
  const int U = scratch[blockDim.x / 32];
  if (threadIdx.x == 0 && n_unique) n_unique[head] = U;
  // slot -> group list
  int32_t* slots = slot_group + head * slot_cap;
  for (int w = threadIdx.x; w < n_words; w += blockDim.x) {
    uint32_t bits = bitmap[w];
    int s = word_off[w];
    while (bits) {
      const int bit = __ffs(bits) - 1;
      bits &= bits - 1u;
      slots[s++] = w * 32 + bit;
    }
  }
  // remapped selection
  for (int i = threadIdx.x; i < n; i += blockDim.x) {
    const int g = sel[i];
    const int jj = i / topk_groups;
    const int64_t own_grp = (q_begin / kBlock + jj) * kGroupsPerBlock;
    int32_t r;
    if (g == -1) {
      r = -1;
    } else if (g >= 0 && g < n_hist) {
      const uint32_t below = bitmap[g >> 5] & ((1u << (g & 31)) - 1u);
      r = word_off[g >> 5] + __popc(below);
    } else if (g >= n_hist && g < own_grp) {
      r = int32_t(act0 + (g - seg0));
    } else {
      latch_status(HGA_ERR_DEVICE_CHECK);
      r = kTierInvalid;
    }
    out[i] = r;
  }
}

// grid (ceil(slot_cap / (8 * kTierCopyWarps)), Hkv, B); 8 groups per warp-loop
template <typename T, int D>
__global__ void __launch_bounds__(kTierCopyWarps * 32)
    tier_copy_kernel(const T* __restrict__ k_host, const T* __restrict__ v_host, int64_t ctx_cap,
                     int n_kv_heads, const int32_t* __restrict__ slot_group,
                     const int32_t* __restrict__ n_unique, int64_t slot_cap,
                     T* __restrict__ k_stage, T* __restrict__ v_stage, int64_t stage_cap) {
  constexpr int kRowBytes = D * int(sizeof(T));
  constexpr int kGroupVec = kGroup * kRowBytes / 16;  // uint4 per group per tensor
  constexpr int kPerLane = (kGroupVec + 31) / 32;
  const int h = blockIdx.y, b = blockIdx.z;
  const int64_t head = int64_t(b) * n_kv_heads + h;
  const int U = n_unique[head];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int per_cta = 8 * kTierCopyWarps;
  for (int u = 0; u < 8; ++u) {
    const int s = blockIdx.x * per_cta + u * kTierCopyWarps + warp;
    if (s >= U) break;
    const int64_t g = slot_group[head * slot_cap + s];
    const uint4* ks = reinterpret_cast<const uint4*>(k_host + (head * ctx_cap + g * kGroup) * D);
    const uint4* vs = reinterpret_cast<const uint4*>(v_host + (head * ctx_cap + g * kGroup) * D);
    uint4* kd = reinterpret_cast<uint4*>(k_stage + (head * stage_cap + int64_t(s) * kGroup) * D);
    uint4* vd = reinterpret_cast<uint4*>(v_stage + (head * stage_cap + int64_t(s) * kGroup) * D);
    uint4 kr[kPerLane], vr[kPerLane];
#pragma unroll
    for (int i = 0; i < kPerLane; ++i) {
      const int e = lane + 32 * i;
      if (e < kGroupVec) {
        kr[i] = ks[e];
        vr[i] = vs[e];
      }
    }
#pragma unroll
    for (int i = 0; i < kPerLane; ++i) {
      const int e = lane + 32 * i;
      if (e < kGroupVec) {
        kd[e] = kr[i];
        vd[e] = vr[i];
      }
    }
  }
}

}  // namespace hga
