// Step a1: group (8-token) and block (64-token) summaries of the keys, the
// mean of the post-RoPE keys per KV head ("BMW如何通过重新设计注意力机制…",
// section "HGA的不同之处": one compact summary per 64-token block kept on the
// GPU, blocks opened at 8-token-group level; gist.science retelling, section
// "解决方案": block summary cards and an 8-token group summary cache).
//
// HBM-bound streaming reduction.  One CTA per (64-token block, KV head, batch)
// with D threads = 8 groups x D/8 column chunks of 8 elements: for one key row
// the D/8 threads of a group read one contiguous row (256 B at bf16, d=128),
// so every load instruction is fully coalesced; each thread keeps 8 float32
// column sums of its group, writes the group mean, and the 8 group sums are
// combined through shared memory into the block mean.
#pragma once

#include "hga_common.cuh"

namespace hga {

// K rows of head (b, h): k + ((b * Hkv + h) * k_rows + row) * D, where block
// blk0 + i starts at row k_first + 64 i (k_rows = ctx_cap, k_first = 64 blk0
// for a whole-context buffer; k_rows = segment capacity, k_first = 0 for a
// segment-local one).  Summaries are indexed by global group / block.
template <typename T, int D>
__global__ void __launch_bounds__(D) summaries_kernel(const T* __restrict__ k, int64_t k_rows,
                                                      int64_t k_first, int64_t ctx_cap,
                                                      int64_t blk0, int n_kv_heads,
                                                      float* __restrict__ gsum,
                                                      float* __restrict__ bsum) {
  // nothing this kernel reads is written by the kernel before it on the
  // stream (only the keys of the new blocks, written before that kernel
  // started): run alongside its tail, but complete only after it, so the
  // kernels after this one see both complete
  pdl_launch_dependents();
  constexpr int CH = D / 8;  // column chunks per row
  __shared__ float part[kGroupsPerBlock][D];
  const int64_t c = blk0 + blockIdx.x;  // global block index
  const int h = blockIdx.y, b = blockIdx.z;
  const int gi = threadIdx.x / CH, ch = threadIdx.x % CH;
  const int64_t head = int64_t(b) * n_kv_heads + h;
  const T* src =
      k + (head * k_rows + k_first + int64_t(blockIdx.x) * kBlock + gi * kGroup) * D + ch * 8;

  float acc[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[e] = 0.f;
  float row[kGroup][8];
#pragma unroll
  for (int r = 0; r < kGroup; ++r) load8(src + int64_t(r) * D, row[r]);
#pragma unroll
  for (int r = 0; r < kGroup; ++r)
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] += row[r][e];

  float mean[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    mean[e] = acc[e] * (1.0f / kGroup);
    part[gi][ch * 8 + e] = acc[e];
  }
  store8(gsum + (head * (ctx_cap / kGroup) + c * kGroupsPerBlock + gi) * D + ch * 8, mean);
  __syncthreads();
  for (int e = threadIdx.x; e < D; e += blockDim.x) {
    float s = 0.f;
#pragma unroll
    for (int g = 0; g < kGroupsPerBlock; ++g) s += part[g][e];
    bsum[(head * (ctx_cap / kBlock) + c) * D + e] = s * (1.0f / kBlock);
  }
  pdl_wait();
}

}  // namespace hga
