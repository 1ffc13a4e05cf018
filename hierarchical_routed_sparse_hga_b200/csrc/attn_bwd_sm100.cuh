// Step a5 on the 5th-generation tensor cores: the backward of the exact-token
// attention under segment-wise backprop ("BMW如何通过重新设计注意力机制…",
// section "HGA的不同之处", last paragraph: forward and backward per segment,
// no gradient across the segment boundary, later segments still attend to
// earlier exact tokens).  History keys give dQ only; keys of the active
// segment also receive dK and dV.  P is recomputed from the saved LSE.
//
// Two kernels, both deterministic (no atomics on the gradients):
//
// attn_bwd_dq_tc_kernel -- one CTA per (batch, KV head, query block), the G
//   heads stacked into M = 64 G rows as in the forward.  Per key tile (the
//   same tiles as the forward): S = Q K^T and dP = dO V^T into TMEM, then one
//   thread per row forms P = exp2(S c - LSE2), dS = P (dP - D) (bf16 into
//   shared memory), and dQ += dS K accumulates in TMEM; dQ = scale * dQ at the
//   end.  D = rowsum(dO * O) is computed here and saved for the next kernel.
//
// attn_bwd_dkdv_tc_kernel -- one CTA per (batch, KV head, 64-key block of the
//   active segment).  It visits, in increasing order, every query block of the
//   segment that attends to the block (its own block causally, later blocks
//   through the groups of it they selected) and accumulates the transposed
//   gradients dV^T += dO^T P and dK^T += Q^T dS in TMEM (M = head_dim = 128,
//   N = 64 keys, K = the 64 G query rows, so the sum over the GQA heads falls
//   out of the contraction).
#pragma once

#include <cuda.h>
#include <math.h>

#include "hga_common.cuh"
#include "sm100_ptx.cuh"

namespace hga {
namespace bwdtc {

using namespace sm100;

constexpr int kD = 128;
constexpr int kMaxTiles = 33;

// ------------------------------------------------------------------------
// dQ kernel
// ------------------------------------------------------------------------
template <int MT>
struct DqLayout {
  static constexpr uint32_t kQ = 0;                              // [MT][2][128][128 B]
  static constexpr uint32_t kDO = MT * 32768;                    // same layout
  static constexpr uint32_t kKV = 2 * MT * 32768;                // [2 stages][K | V]
  static constexpr uint32_t kStages = 2;
  static constexpr uint32_t kStageBytes = 32768;
  static constexpr uint32_t kDS = kKV + kStages * kStageBytes;   // [MT][128][128 B]
  static constexpr uint32_t kBytes = kDS + MT * 16384;
  static constexpr uint32_t kDynSmem = kBytes + 1024;
  static constexpr uint32_t kThreads = 128 + 128 * MT;
  static constexpr uint32_t kTmemCols = MT == 2 ? 512 : 256;
  // TMEM columns: S_m, dP_m (64 each), dQ_m (128)
  static constexpr uint32_t colS(int m) { return m * 64; }
  static constexpr uint32_t colDP(int m) { return MT * 64 + m * 64; }
  static constexpr uint32_t colDQ(int m) { return MT * 128 + m * 128; }
};

struct DqShared {
  uint64_t q_full;
  uint64_t kv_full[2];
  uint64_t kv_empty[2];
  uint64_t sdp_full[2];
  uint64_t sdp_free[2];
  uint64_t ds_full[2];
  uint64_t ds_done[2];
  uint64_t mma_done;
  uint32_t tmem_base;
  int abort;
  int n_tiles;
  int grp[kMaxTiles * 8];
  uint8_t tile_mask[kMaxTiles];
};

// Builds the key-tile schedule of query block j exactly as the forward does:
// valid selected groups in order, last routed tile padded with the first
// valid group (masked), then the own block.  Executed by one full warp.
template <typename SH>
__device__ __forceinline__ void build_schedule(SH& sh, const int32_t* srow, int topk_groups,
                                               int64_t own_blk, int lane) {
  int n_valid = 0;
  for (int c0 = 0; c0 < topk_groups; c0 += 32) {
    const int idx = c0 + lane;
    const int g = idx < topk_groups ? srow[idx] : -1;
    bool ok = false;
    if (idx < topk_groups && g != -1) {
      ok = g >= 0 && int64_t(g) < own_blk * kGroupsPerBlock;
      if (!ok) latch_status(HGA_ERR_DEVICE_CHECK);
    }
    const unsigned ball = __ballot_sync(0xffffffffu, ok);
    if (ok) sh.grp[n_valid + __popc(ball & ((1u << lane) - 1u))] = g;
    n_valid += __popc(ball);
  }
  __syncwarp();
  const int n_rt = (n_valid + 7) / 8;
  for (int i = n_valid + lane; i < n_rt * 8; i += 32) sh.grp[i] = sh.grp[0];
  for (int t = lane; t < n_rt; t += 32) {
    const int left = n_valid - 8 * t;
    sh.tile_mask[t] = left >= 8 ? 0xffu : uint8_t((1u << left) - 1u);
  }
  for (int i = lane; i < 8; i += 32) sh.grp[n_rt * 8 + i] = int(own_blk * kGroupsPerBlock + i);
  if (lane == 0) {
    sh.tile_mask[n_rt] = 0xffu;
    sh.n_tiles = n_rt + 1;
  }
}

template <int MT>
__global__ void __launch_bounds__(DqLayout<MT>::kThreads, 1)
    attn_bwd_dq_tc_kernel(const __grid_constant__ CUtensorMap tm_q,
                          const __grid_constant__ CUtensorMap tm_do,
                          const __grid_constant__ CUtensorMap tm_k,
                          const __grid_constant__ CUtensorMap tm_v, int64_t ctx_cap,
                          int64_t q_begin, int s_len, int n_q_heads, int n_kv_heads,
                          int topk_groups, const int32_t* __restrict__ sel_grp, float scale,
                          float scale_log2, const __nv_bfloat16* __restrict__ o,
                          const __nv_bfloat16* __restrict__ d_o, const float* __restrict__ lse,
                          __nv_bfloat16* __restrict__ dq, float* __restrict__ dvec) {
  using L = DqLayout<MT>;
  constexpr int G = 2 * MT;
  extern __shared__ uint8_t dsmem_raw[];
  __shared__ DqShared sh;
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(dsmem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sQ = smem_u32(smem + L::kQ), sDO = smem_u32(smem + L::kDO);
  const uint32_t sKV = smem_u32(smem + L::kKV), sDS = smem_u32(smem + L::kDS);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int j = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int n_qb = s_len / kQBlock;
  const int64_t own_blk = (q_begin + int64_t(j) * kQBlock) / kBlock;
  volatile int* abort = &sh.abort;

  if (tid == 0) {
    mbar_init(&sh.q_full, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&sh.kv_full[s], 1);
      mbar_init(&sh.kv_empty[s], 1);
    }
    for (int m = 0; m < 2; ++m) {
      mbar_init(&sh.sdp_full[m], 1);
      mbar_init(&sh.sdp_free[m], 128);
      mbar_init(&sh.ds_full[m], 128);
      mbar_init(&sh.ds_done[m], 1);
    }
    mbar_init(&sh.mma_done, 1);
    sh.abort = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(&sh.tmem_base, L::kTmemCols);
    tmem_relinquish();
  }
  if (warp == 0)
    build_schedule(sh, sel_grp + ((int64_t(b) * n_kv_heads + h) * n_qb + j) * topk_groups,
                   topk_groups, own_blk, lane);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sh.tmem_base;
  const int n_tiles = sh.n_tiles;

  if (warp == 0) {
    if (lane == 0) {
      prefetch_tmap(&tm_q);
      prefetch_tmap(&tm_do);
      prefetch_tmap(&tm_k);
      prefetch_tmap(&tm_v);
      mbar_arrive_expect_tx(&sh.q_full, MT * 65536);
      for (int g = 0; g < G; ++g) {
        const int32_t row = int32_t((int64_t(b) * n_q_heads + h * G + g) * s_len + j * kQBlock);
        for (int hf = 0; hf < 2; ++hf) {
          const uint32_t off = (g >> 1) * 32768 + hf * 16384 + (g & 1) * 8192;
          tma_load_2d(smem + L::kQ + off, &tm_q, &sh.q_full, hf * 64, row);
          tma_load_2d(smem + L::kDO + off, &tm_do, &sh.q_full, hf * 64, row);
        }
      }
      const int64_t kv_row0 = (int64_t(b) * n_kv_heads + h) * ctx_cap;
      int issued = 0;
      for (int t = 0; t < n_tiles; ++t) {
        const int st = t & 1;
        if (t >= 2 && !mbar_wait(&sh.kv_empty[st], ((t >> 1) - 1) & 1, abort)) break;
        mbar_arrive_expect_tx(&sh.kv_full[st], L::kStageBytes);
        uint8_t* kdst = smem + L::kKV + st * L::kStageBytes;
        for (int gi = 0; gi < 8; ++gi) {
          const int32_t row = int32_t(kv_row0 + int64_t(sh.grp[t * 8 + gi]) * kGroup);
          for (int hf = 0; hf < 2; ++hf) {
            tma_load_2d(kdst + hf * 8192 + gi * 1024, &tm_k, &sh.kv_full[st], hf * 64, row);
            tma_load_2d(kdst + 16384 + hf * 8192 + gi * 1024, &tm_v, &sh.kv_full[st], hf * 64,
                        row);
          }
        }
        issued = t + 1;
      }
      int never = 0;
      mbar_wait(&sh.q_full, 0, &never);
      for (int t = issued - 1; t >= 0 && t >= issued - 2; --t)
        mbar_wait(&sh.kv_full[t & 1], (t >> 1) & 1, &never);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16_f32(128, 64, 0, 0);
      constexpr uint32_t idesc_dq = idesc_bf16_f32(128, kD, 0, 1);
      bool ok = mbar_wait(&sh.q_full, 0, abort);
      bool issued_any = false;
      tc_fence_after();
      for (int t = 0; ok && t <= n_tiles; ++t) {
        if (t < n_tiles) {
          const int st = t & 1;
          if (!(ok = mbar_wait(&sh.kv_full[st], (t >> 1) & 1, abort))) break;
          for (int m = 0; m < MT && ok; ++m)
            if (t >= 1) ok = mbar_wait(&sh.sdp_free[m], (t - 1) & 1, abort);
          if (!ok) break;
          tc_fence_after();
          const uint32_t kb = sKV + st * L::kStageBytes;
          for (int m = 0; m < MT; ++m) {
#pragma unroll
            for (int k = 0; k < 8; ++k) {
              const uint32_t ko = (k >> 2) * 16384 + (k & 3) * 32;
              const uint32_t bo = (k >> 2) * 8192 + (k & 3) * 32;
              mma_bf16(tmem + L::colS(m), smem_desc_sw128(sQ + m * 32768 + ko, 16, 1024),
                       smem_desc_sw128(kb + bo, 16, 1024), idesc_s, k > 0);
              mma_bf16(tmem + L::colDP(m), smem_desc_sw128(sDO + m * 32768 + ko, 16, 1024),
                       smem_desc_sw128(kb + 16384 + bo, 16, 1024), idesc_s, k > 0);
            }
            mma_commit(&sh.sdp_full[m]);
          }
          issued_any = true;
        }
        if (t >= 1) {
          const int tt = t - 1, st = tt & 1;
          const uint32_t kb = sKV + st * L::kStageBytes;
          for (int m = 0; m < MT; ++m) {
            if (!(ok = mbar_wait(&sh.ds_full[m], tt & 1, abort))) break;
            tc_fence_after();
#pragma unroll
            for (int k = 0; k < 4; ++k)
              mma_bf16(tmem + L::colDQ(m), smem_desc_sw128(sDS + m * 16384 + k * 32, 16, 1024),
                       smem_desc_sw128(kb + k * 2048, 8192, 1024), idesc_dq,
                       (tt > 0 || k > 0) ? 1u : 0u);
            mma_commit(&sh.ds_done[m]);
          }
          if (!ok) break;
          mma_commit(&sh.kv_empty[st]);
        }
      }
      if (issued_any) {
        int never = 0;
        mma_commit(&sh.mma_done);
        mbar_wait(&sh.mma_done, 0, &never);
      }
    }
  } else if (warp >= 4) {
    const int m = (warp - 4) >> 2, wq = (warp - 4) & 3;
    const int row = wq * 32 + lane;
    const int grow = m * 128 + row, g = grow >> 6, r = grow & 63;
    const uint32_t lane_addr = uint32_t(wq * 32) << 16;
    const int hq = h * G + g;
    const int64_t rix = (int64_t(b) * n_q_heads + hq) * s_len + int64_t(j) * kQBlock + r;
    // D = rowsum(dO * O), saved for the dK/dV kernel
    float dsum = 0.f;
    for (int c = 0; c < kD; c += 8) {
      float a[8], bb[8];
      load8(d_o + rix * kD + c, a);
      load8(o + rix * kD + c, bb);
#pragma unroll
      for (int i = 0; i < 8; ++i) dsum = fmaf(a[i], bb[i], dsum);
    }
    dvec[rix] = dsum;
    const float lse2 = lse[rix] * 1.4426950408889634f;
    bool ok = true;
    uint8_t* drow = smem + L::kDS + m * 16384 + row * 128;
    for (int t = 0; t < n_tiles && ok; ++t) {
      if (!(ok = mbar_wait(&sh.sdp_full[m], t & 1, abort))) break;
      tc_fence_after();
      const bool own = t == n_tiles - 1;
      const uint32_t mask = sh.tile_mask[t];
      uint32_t packed[32];
#pragma unroll
      for (int hb = 0; hb < 2; ++hb) {
        float sv[32], dp[32];
        tmem_ld32(tmem + lane_addr + L::colS(m) + hb * 32, sv);
        tmem_ld32(tmem + lane_addr + L::colDP(m) + hb * 32, dp);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; i += 2) {
          float ds2[2];
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            const int key = hb * 32 + i + u;
            const bool valid = ((mask >> (key >> 3)) & 1u) && (!own || key <= r);
            const float p = valid ? exp2f(sv[i + u] * scale_log2 - lse2) : 0.f;
            ds2[u] = p * (dp[i + u] - dsum);
          }
          __nv_bfloat162 pr = __floats2bfloat162_rn(ds2[0], ds2[1]);
          packed[hb * 16 + i / 2] = *reinterpret_cast<uint32_t*>(&pr);
        }
      }
      tc_fence_before();
      mbar_arrive(&sh.sdp_free[m]);
      if (t > 0 && !(ok = mbar_wait(&sh.ds_done[m], (t - 1) & 1, abort))) break;
#pragma unroll
      for (int c = 0; c < 8; ++c)
        *reinterpret_cast<uint4*>(drow + ((c ^ (row & 7)) << 4)) =
            make_uint4(packed[4 * c], packed[4 * c + 1], packed[4 * c + 2], packed[4 * c + 3]);
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(&sh.ds_full[m]);
    }
    if (ok) ok = mbar_wait(&sh.ds_done[m], (n_tiles - 1) & 1, abort);
    if (ok) {
      tc_fence_after();
      __nv_bfloat16* dst = dq + rix * kD;
      for (int c = 0; c < kD; c += 32) {
        float v[32];
        tmem_ld32(tmem + lane_addr + L::colDQ(m) + c, v);
        tmem_wait_ld();
#pragma unroll
        for (int q8 = 0; q8 < 4; ++q8) {
          float f[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) f[i] = v[8 * q8 + i] * scale;
          store8(dst + c + 8 * q8, f);
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, L::kTmemCols);
  }
}

// ------------------------------------------------------------------------
// dK / dV kernel
// ------------------------------------------------------------------------
template <int MT>
struct KvLayout {
  static constexpr uint32_t kK = 0;                  // [2 halves][64][128 B]
  static constexpr uint32_t kV = 16384;
  static constexpr uint32_t kQ = 32768;              // [MT][2][128][128 B]
  static constexpr uint32_t kDO = kQ + MT * 32768;
  static constexpr uint32_t kP = kDO + MT * 32768;   // [MT][128][128 B]
  static constexpr uint32_t kDS = kP + MT * 16384;
  static constexpr uint32_t kBytes = kDS + MT * 16384;
  static constexpr uint32_t kDynSmem = kBytes + 1024;
  static constexpr uint32_t kThreads = 128 + 128 * MT;
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t colS(int m) { return m * 64; }
  static constexpr uint32_t colDP(int m) { return MT * 64 + m * 64; }
  static constexpr uint32_t kColDV = MT * 128;
  static constexpr uint32_t kColDK = MT * 128 + 64;
};

struct KvShared {
  uint64_t kv_full;
  uint64_t qd_full;
  uint64_t qd_empty;
  uint64_t sdp_full[2];
  uint64_t pds_full;
  uint64_t mma_done;
  uint32_t tmem_base;
  int abort;
  int n_iter;
  int masks[64];
  int js[64];
};

template <int MT>
__global__ void __launch_bounds__(KvLayout<MT>::kThreads, 1)
    attn_bwd_dkdv_tc_kernel(const __grid_constant__ CUtensorMap tm_q,
                            const __grid_constant__ CUtensorMap tm_do,
                            const __grid_constant__ CUtensorMap tm_k,
                            const __grid_constant__ CUtensorMap tm_v, int64_t ctx_cap,
                            int64_t q_begin, int s_len, int n_q_heads, int n_kv_heads,
                            int topk_groups, const int32_t* __restrict__ sel_grp, float scale,
                            float scale_log2, const float* __restrict__ lse,
                            const float* __restrict__ dvec, __nv_bfloat16* __restrict__ dk,
                            __nv_bfloat16* __restrict__ dv) {
  using L = KvLayout<MT>;
  constexpr int G = 2 * MT;
  extern __shared__ uint8_t dsmem_raw[];
  __shared__ KvShared sh;
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(dsmem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sK = smem_u32(smem + L::kK), sV = smem_u32(smem + L::kV);
  const uint32_t sQ = smem_u32(smem + L::kQ), sDO = smem_u32(smem + L::kDO);
  const uint32_t sP = smem_u32(smem + L::kP), sDS = smem_u32(smem + L::kDS);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int kb = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int n_qb = s_len / kQBlock;
  const int64_t gblk = q_begin / kBlock + kb;  // global index of this key block
  volatile int* abort = &sh.abort;

  for (int i = tid; i < 64; i += blockDim.x) sh.masks[i] = (i == kb) ? 0xff : 0;
  if (tid == 0) {
    mbar_init(&sh.kv_full, 1);
    mbar_init(&sh.qd_full, 1);
    mbar_init(&sh.qd_empty, 1);
    mbar_init(&sh.sdp_full[0], 1);
    mbar_init(&sh.sdp_full[1], 1);
    mbar_init(&sh.pds_full, 128 * MT);
    mbar_init(&sh.mma_done, 1);
    sh.abort = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(&sh.tmem_base, L::kTmemCols);
    tmem_relinquish();
  }
  __syncthreads();
  // which later query blocks of the segment selected groups of this block
  const int32_t* sel_bh = sel_grp + (int64_t(b) * n_kv_heads + h) * n_qb * topk_groups;
  for (int idx = tid; idx < n_qb * topk_groups; idx += blockDim.x) {
    const int jj = idx / topk_groups;
    if (jj <= kb) continue;
    const int g = sel_bh[idx];
    const int64_t own_jj = q_begin / kBlock + jj;
    if (g >= 0 && int64_t(g) < own_jj * kGroupsPerBlock && int64_t(g) / kGroupsPerBlock == gblk)
      atomicOr(&sh.masks[jj], 1 << (g % kGroupsPerBlock));
  }
  __syncthreads();
  if (warp == 0) {
    int n = 0;
    for (int c0 = 0; c0 < n_qb; c0 += 32) {
      const int jj = c0 + lane;
      const bool on = jj < n_qb && jj >= kb && sh.masks[jj] != 0;
      const unsigned ball = __ballot_sync(0xffffffffu, on);
      if (on) sh.js[n + __popc(ball & ((1u << lane) - 1u))] = jj;
      n += __popc(ball);
    }
    if (lane == 0) sh.n_iter = n;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sh.tmem_base;
  const int n_iter = sh.n_iter;

  if (warp == 0) {
    if (lane == 0) {
      prefetch_tmap(&tm_q);
      prefetch_tmap(&tm_do);
      prefetch_tmap(&tm_k);
      prefetch_tmap(&tm_v);
      const int32_t krow = int32_t((int64_t(b) * n_kv_heads + h) * ctx_cap + gblk * kBlock);
      mbar_arrive_expect_tx(&sh.kv_full, 32768);
      for (int gi = 0; gi < 8; ++gi)
        for (int hf = 0; hf < 2; ++hf) {
          tma_load_2d(smem + L::kK + hf * 8192 + gi * 1024, &tm_k, &sh.kv_full, hf * 64,
                      krow + gi * kGroup);
          tma_load_2d(smem + L::kV + hf * 8192 + gi * 1024, &tm_v, &sh.kv_full, hf * 64,
                      krow + gi * kGroup);
        }
      int issued = 0;
      for (int it = 0; it < n_iter; ++it) {
        if (it > 0 && !mbar_wait(&sh.qd_empty, (it - 1) & 1, abort)) break;
        const int jj = sh.js[it];
        mbar_arrive_expect_tx(&sh.qd_full, MT * 65536);
        for (int g = 0; g < G; ++g) {
          const int32_t row =
              int32_t((int64_t(b) * n_q_heads + h * G + g) * s_len + jj * kQBlock);
          for (int hf = 0; hf < 2; ++hf) {
            const uint32_t off = (g >> 1) * 32768 + hf * 16384 + (g & 1) * 8192;
            tma_load_2d(smem + L::kQ + off, &tm_q, &sh.qd_full, hf * 64, row);
            tma_load_2d(smem + L::kDO + off, &tm_do, &sh.qd_full, hf * 64, row);
          }
        }
        issued = it + 1;
      }
      int never = 0;
      mbar_wait(&sh.kv_full, 0, &never);
      if (issued > 0) mbar_wait(&sh.qd_full, (issued - 1) & 1, &never);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16_f32(128, 64, 0, 0);
      constexpr uint32_t idesc_t = idesc_bf16_f32(128, 64, 1, 1);
      bool ok = mbar_wait(&sh.kv_full, 0, abort);
      bool issued_any = false;
      for (int it = 0; ok && it < n_iter; ++it) {
        if (!(ok = mbar_wait(&sh.qd_full, it & 1, abort))) break;
        tc_fence_after();
        for (int m = 0; m < MT; ++m) {
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            const uint32_t ao = m * 32768 + (k >> 2) * 16384 + (k & 3) * 32;
            const uint32_t bo = (k >> 2) * 8192 + (k & 3) * 32;
            mma_bf16(tmem + L::colS(m), smem_desc_sw128(sQ + ao, 16, 1024),
                     smem_desc_sw128(sK + bo, 16, 1024), idesc_s, k > 0);
            mma_bf16(tmem + L::colDP(m), smem_desc_sw128(sDO + ao, 16, 1024),
                     smem_desc_sw128(sV + bo, 16, 1024), idesc_s, k > 0);
          }
          mma_commit(&sh.sdp_full[m]);
        }
        issued_any = true;
        if (!(ok = mbar_wait(&sh.pds_full, it & 1, abort))) break;
        tc_fence_after();
        // dV^T += dO^T P and dK^T += Q^T dS: K runs over the MT*128 query rows
        for (int s = 0; s < MT * 8; ++s) {
          const int m = s >> 3;
          const uint32_t ro = (s & 7) * 2048;
          const uint32_t acc = (it > 0 || s > 0) ? 1u : 0u;
          mma_bf16(tmem + L::kColDV, smem_desc_sw128(sDO + m * 32768 + ro, 16384, 1024),
                   smem_desc_sw128(sP + m * 16384 + ro, 8192, 1024), idesc_t, acc);
          mma_bf16(tmem + L::kColDK, smem_desc_sw128(sQ + m * 32768 + ro, 16384, 1024),
                   smem_desc_sw128(sDS + m * 16384 + ro, 8192, 1024), idesc_t, acc);
        }
        mma_commit(&sh.qd_empty);
      }
      if (issued_any) {
        int never = 0;
        mma_commit(&sh.mma_done);
        mbar_wait(&sh.mma_done, 0, &never);
      }
    }
  } else if (warp >= 4) {
    const int m = (warp - 4) >> 2, wq = (warp - 4) & 3;
    const int row = wq * 32 + lane;
    const int grow = m * 128 + row, g = grow >> 6, r = grow & 63;
    const uint32_t lane_addr = uint32_t(wq * 32) << 16;
    const int hq = h * G + g;
    bool ok = true;
    uint8_t* prow = smem + L::kP + m * 16384 + row * 128;
    uint8_t* drow = smem + L::kDS + m * 16384 + row * 128;
    for (int it = 0; it < n_iter && ok; ++it) {
      const int jj = sh.js[it];
      const bool own = jj == kb;
      const uint32_t mask = sh.masks[jj];
      const int64_t rix = (int64_t(b) * n_q_heads + hq) * s_len + int64_t(jj) * kQBlock + r;
      const float lse2 = lse[rix] * 1.4426950408889634f;
      const float dsum = dvec[rix];
      if (!(ok = mbar_wait(&sh.sdp_full[m], it & 1, abort))) break;
      // the previous iteration's dV/dK MMAs must be done reading P and dS (this
      // phase already completed: the producer waited for it before loading the
      // Q/dO tiles that this iteration's S and dP were computed from)
      if (it > 0 && !(ok = mbar_wait(&sh.qd_empty, (it - 1) & 1, abort))) break;
      tc_fence_after();
#pragma unroll
      for (int hb = 0; hb < 2; ++hb) {
        float sv[32], dp[32];
        tmem_ld32(tmem + lane_addr + L::colS(m) + hb * 32, sv);
        tmem_ld32(tmem + lane_addr + L::colDP(m) + hb * 32, dp);
        tmem_wait_ld();
        uint32_t pk[16], dk2[16];
#pragma unroll
        for (int i = 0; i < 32; i += 2) {
          float p2[2], d2[2];
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            const int key = hb * 32 + i + u;
            const bool valid = ((mask >> (key >> 3)) & 1u) && (!own || key <= r);
            p2[u] = valid ? exp2f(sv[i + u] * scale_log2 - lse2) : 0.f;
            d2[u] = p2[u] * (dp[i + u] - dsum);
          }
          __nv_bfloat162 pp = __floats2bfloat162_rn(p2[0], p2[1]);
          __nv_bfloat162 dd = __floats2bfloat162_rn(d2[0], d2[1]);
          pk[i / 2] = *reinterpret_cast<uint32_t*>(&pp);
          dk2[i / 2] = *reinterpret_cast<uint32_t*>(&dd);
        }
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
          const int c = hb * 4 + cc;
          const int off = (c ^ (row & 7)) << 4;
          *reinterpret_cast<uint4*>(prow + off) =
              make_uint4(pk[4 * cc], pk[4 * cc + 1], pk[4 * cc + 2], pk[4 * cc + 3]);
          *reinterpret_cast<uint4*>(drow + off) =
              make_uint4(dk2[4 * cc], dk2[4 * cc + 1], dk2[4 * cc + 2], dk2[4 * cc + 3]);
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(&sh.pds_full);
    }
    // epilogue: warp group 0 owns TMEM lanes 0..127 = the 128 head dims
    if (m == 0) {
      if (ok && n_iter > 0) ok = mbar_wait(&sh.qd_empty, (n_iter - 1) & 1, abort);
      if (ok) {
        tc_fence_after();
        const int dcol = row;
        const int64_t base = ((int64_t(b) * n_kv_heads + h) * s_len + int64_t(kb) * kBlock) * kD;
        for (int c = 0; c < 64; c += 32) {
          float vv[32], kk[32];
          tmem_ld32(tmem + lane_addr + L::kColDV + c, vv);
          tmem_ld32(tmem + lane_addr + L::kColDK + c, kk);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const int64_t at = base + int64_t(c + i) * kD + dcol;
            dv[at] = __float2bfloat16_rn(n_iter > 0 ? vv[i] : 0.f);
            dk[at] = __float2bfloat16_rn(n_iter > 0 ? kk[i] * scale : 0.f);
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, L::kTmemCols);
  }
}

}  // namespace bwdtc
}  // namespace hga
