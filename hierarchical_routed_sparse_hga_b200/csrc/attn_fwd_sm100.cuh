// Step a4 on the 5th-generation tensor cores: exact-token attention of one
// query block over its selected 8-token groups plus its causal own block
// ("BMW如何通过重新设计注意力机制…", section "HGA的不同之处": only the selected
// groups' exact K/V enter the attention; the summaries only steer selection).
//
// One CTA per (batch, KV head, query block, set of 2*MT query heads): the G
// query heads sharing a KV head share the selection, so up to four of them
// are stacked into MT tiles of M = 128 rows and every gathered K/V tile feeds
// all of them.
//
// Roles (128 + 128*MT threads, one CTA per SM):
//   warp 0      TMA producer: Q once (64 x 64 boxes); then per key tile the
//               8 selected groups of K and V, each group (a contiguous 2 KiB
//               run of [B,Hkv,T,d]) one 3-D box of 64 columns x 8 rows x 2
//               column halves, into a 4-stage ring laid
//               out [group][d half][8 rows][128 B] (128-byte swizzle; UMMA
//               stride 2048 B between 8-row groups);
//   warp 1      TMEM owner and S issuer: S = Q K^T into double-buffered
//               TMEM, in a fixed order with blocking waits;
//   warp 3      PV issuer: O += P V with P read straight from TMEM (A
//               operand in tensor memory), as soon as the softmax wrote it;
//   warps 4..   softmax, one warp group per M tile, one thread per row (TMEM
//               lane): masks (padding slots, causal own block; skipped for
//               full routed tiles), online softmax in the log2 domain with
//               packed f32x2 arithmetic and lazy rescaling (O is rescaled only
//               when the running max grows by more than 2^8), P written back as
//               bf16 over its own S columns; epilogue O / l (through shared
//               memory, TMA stores) and LSE.
// The producer and issuer loops run in all 32 lanes of their warp, so loop
// state and operand descriptors are warp-uniform; one elected lane issues.
// Every wait is bounded; a timeout latches HGA_ERR_TIMEOUT, raises a shared
// abort flag, drains the copies and MMAs in flight and frees TMEM.
#pragma once

#include <cuda.h>
#include <math.h>

#include "hga_common.cuh"
#include "sm100_ptx.cuh"

namespace hga {
namespace fwdtc {

using namespace sm100;

constexpr int kD = 128;
constexpr int kStages = 4;
constexpr int kMaxTiles = 33;  // 256 groups / 8 + own block

template <int MT>
struct Layout {
  static constexpr uint32_t kQ = 0;                                // [MT][2 halves][128][128 B]
  static constexpr uint32_t kKV = MT * 32768;                      // [stage][K 16 KB | V 16 KB]
  static constexpr uint32_t kStageBytes = 32768;
  static constexpr uint32_t kBytes = kKV + kStages * kStageBytes;
  static constexpr uint32_t kDynSmem = kBytes + 1024;              // + alignment slack
  static constexpr uint32_t kThreads = 128 + 128 * MT;
  static constexpr uint32_t kTmemCols = MT == 2 ? 512 : 256;
  static constexpr uint32_t colS(int m, int buf) { return (m * 2 + buf) * 64; }
  static constexpr uint32_t colO(int m) { return MT * 128 + m * kD; }
};

struct Shared {
  uint64_t q_full;
  uint64_t kv_full[kStages];
  uint64_t kv_empty[kStages];
  // [M tile][tile & 1]: per-buffer barriers, so no waiter can ever fall two
  // phases behind (that would need a tile whose S buffer is still in use)
  uint64_t s_full[2][2];
  uint64_t p_full[2][2];
  uint64_t pv_done[2][2];
  uint64_t mma_done[2];  // every MMA of issuer 0 (S) / issuer 1 (PV) has completed
  uint32_t tmem_base;
  int abort;
  int n_tiles;
  int grp[kMaxTiles * 8];
  uint8_t tile_mask[kMaxTiles];
};

constexpr uint32_t kTestDropFirstTile = 0x80000000u;  // test hook, see hga.h

// grid (n_qb * G / (2 MT), Hkv, B)
template <int MT>
__global__ void __launch_bounds__(Layout<MT>::kThreads, 1)
    attn_fwd_tc_kernel(const __grid_constant__ CUtensorMap tm_q,
                       const __grid_constant__ CUtensorMap tm_k,
                       const __grid_constant__ CUtensorMap tm_v,
                       const __grid_constant__ CUtensorMap tm_o, int64_t ctx_cap, int64_t q_begin,
                       int s_len, int n_q_heads, int n_kv_heads, int topk_groups,
                       const int32_t* __restrict__ sel_grp, float scale_log2,
                       float* __restrict__ lse, uint32_t flags,
                       const int* __restrict__ route_done, int* __restrict__ done,
                       uint32_t token) {
  using L = Layout<MT>;
  extern __shared__ uint8_t dsmem_raw[];
  __shared__ Shared sh;
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(dsmem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sQ = smem_u32(smem + L::kQ);
  const uint32_t sKV = smem_u32(smem + L::kKV);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = n_q_heads / n_kv_heads, n_sets = G / (2 * MT);
  const int j = blockIdx.x / n_sets, hs = blockIdx.x % n_sets;
  const int h = blockIdx.y, b = blockIdx.z;
  const int head0 = h * G + hs * 2 * MT;       // first query head of this CTA
  const int n_qb = s_len / kQBlock;
  const int64_t own_blk = (q_begin + int64_t(j) * kQBlock) / kBlock;
  volatile int* abort = &sh.abort;

  // ---- set-up: barriers, the Q load, TMEM, the tile schedule -------------
  if (tid == 0) {
    mbar_init(&sh.q_full, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&sh.kv_full[s], 1);
      mbar_init(&sh.kv_empty[s], 2);  // the last S and the last PV of the tile
    }
    for (int m = 0; m < 2; ++m)
      for (int u = 0; u < 2; ++u) {
        mbar_init(&sh.s_full[m][u], 1);
        mbar_init(&sh.p_full[m][u], 128);
        mbar_init(&sh.pv_done[m][u], 1);
      }
    mbar_init(&sh.mma_done[0], 1);
    mbar_init(&sh.mma_done[1], 1);
    sh.abort = 0;
    fence_barrier_init();
  }
  // the previous kernel may still hold this SM's tensor memory or write
  // this kernel's inputs: wait for it before allocating or reading.  In a
  // chained segment call the previous kernel is the routing, which has no
  // tensor memory and let this grid start only once everything before it
  // had completed: only this item's selection is waited for (route_done).
  if (!route_done) pdl_wait();
  if (tid == 0) {
    // Q first: it does not depend on the selection
    prefetch_tmap(&tm_q);
    prefetch_tmap(&tm_k);
    prefetch_tmap(&tm_v);
    mbar_arrive_expect_tx(&sh.q_full, MT * 32768);
    for (int g = 0; g < 2 * MT; ++g) {
      const int32_t row = int32_t((int64_t(b) * n_q_heads + head0 + g) * s_len + j * kQBlock);
      for (int hf = 0; hf < 2; ++hf) {
        uint8_t* dst = smem + L::kQ + (g >> 1) * 32768 + hf * 16384 + (g & 1) * 8192;
        tma_load_2d(dst, &tm_q, &sh.q_full, hf * 64, row);
      }
    }
    // and tile 0, the causal own block, which does not depend on it either
    if (!(flags & kTestDropFirstTile)) {
      mbar_arrive_expect_tx(&sh.kv_full[0], L::kStageBytes);
      const int64_t own_row0 =
          (int64_t(b) * n_kv_heads + h) * ctx_cap + own_blk * kBlock;
      uint8_t* kdst = smem + L::kKV;
#pragma unroll
      for (int gi = 0; gi < 8; ++gi) {
        const int32_t row = int32_t(own_row0 + gi * kGroup);
        tma_load_3d(kdst + gi * 2048, &tm_k, &sh.kv_full[0], 0, row, 0);
        tma_load_3d(kdst + gi * 2048 + 16384, &tm_v, &sh.kv_full[0], 0, row, 0);
      }
    }
  }
  if (warp == 1) {
    tmem_alloc(&sh.tmem_base, L::kTmemCols);
    tmem_relinquish();
  }
  if (warp == 0) {
    if (route_done)
      flag_wait(route_done + blockIdx.x + gridDim.x * (blockIdx.y + gridDim.y * blockIdx.z),
                token, abort);
    build_tile_schedule(sh, sel_grp + ((int64_t(b) * n_kv_heads + h) * n_qb + j) * topk_groups,
                        topk_groups, own_blk, lane);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // the next kernel may be scheduled from here on (this item's selection,
  // and everything the routing waited for, are complete)
  pdl_launch_dependents();
  const uint32_t tmem = sh.tmem_base;
  const int n_tiles = sh.n_tiles;

  if (warp == 0) {
    // ---------------- TMA producer (whole warp; one elected lane issues) ----
    // K/V tile layout: group gi at gi * 2048: [d half][8 rows][128 B], one
    // 3-D box (64 columns x 8 rows x 2 halves) per group and tensor (Q was
    // issued during set-up)
    const int64_t kv_row0 = (int64_t(b) * n_kv_heads + h) * ctx_cap;
    // tile 0 (the own block) was requested during set-up; with the test
    // hook it is never armed, so its consumers must time out
    int issued = (flags & kTestDropFirstTile) ? 0 : 1;
    for (int t = 1; t < n_tiles; ++t) {
      const int st = t % kStages;
      const bool free_ok =
          t < kStages || mbar_wait(&sh.kv_empty[st], ((t / kStages) - 1) & 1, abort);
      if (!__all_sync(kFullMask, free_ok)) break;
      if (elect_one()) {
        mbar_arrive_expect_tx(&sh.kv_full[st], L::kStageBytes);
        uint8_t* kdst = smem + L::kKV + st * L::kStageBytes;
#pragma unroll
        for (int gi = 0; gi < 8; ++gi) {
          const int32_t row = int32_t(kv_row0 + int64_t(sh.grp[t * 8 + gi]) * kGroup);
          tma_load_3d(kdst + gi * 2048, &tm_k, &sh.kv_full[st], 0, row, 0);
          tma_load_3d(kdst + gi * 2048 + 16384, &tm_v, &sh.kv_full[st], 0, row, 0);
        }
      }
      __syncwarp();
      issued = t + 1;
    }
    // drain: wait (bounded, independent of abort) for the copies in flight
    if (lane == 0) {
      int never = 0;
      mbar_wait(&sh.q_full, 0, &never);
      for (int t = issued - 1; t >= 0 && t >= issued - kStages; --t) {
        if ((flags & kTestDropFirstTile) && t == 0) continue;
        mbar_wait(&sh.kv_full[t % kStages], (t / kStages) & 1, &never);
      }
    }
  } else if (warp == 1 || warp == 3) {
    // ---------------- MMA issuers (whole warp each, one lane issues) --------
    // Warp 1 issues S(t, m) = Q_m K_t^T once K/V of tile t are in and, for
    // t >= 2, PV(t-2, m) has completed (S(t, m) reuses the TMEM columns that
    // hold P(t-2, m) until PV(t-2, m) has read them); warp 3 issues
    // PV(t, m): O_m += P(t, m) V_t once the softmax has written P(t, m).  Two
    // issuers, so that a ready PV never queues behind the sixteen S MMAs of
    // the next tile.  The stage of tile t is free once its last S and its
    // last PV have completed (two commits on kv_empty).  The waits block
    // (the warp is parked until the phase completes), which leaves the issue
    // slots of its sub-partition to the softmax warps.
    const int iss = warp == 1 ? 0 : 1;
    constexpr uint32_t idesc_qk = idesc_bf16_f32(128, 64, 0, 0);
    constexpr uint32_t idesc_pv = idesc_bf16_f32(128, kD, 0, 1);
    bool issued_any = false;
    bool ok = __all_sync(kFullMask, mbar_wait(&sh.q_full, 0, abort));
    for (int t = 0; ok && t < n_tiles; ++t) {
      const int st = t % kStages, buf = t & 1;
      for (int m = 0; ok && m < MT; ++m) {
        if (iss == 0) {
          bool ready = m > 0 || mbar_wait(&sh.kv_full[st], (t / kStages) & 1, abort);
          if (t >= 2) ready = ready && mbar_wait(&sh.pv_done[m][buf], ((t - 2) >> 1) & 1, abort);
          if (!(ok = __all_sync(kFullMask, ready))) break;
          tc_fence_after();
          const uint32_t kbase = sKV + st * L::kStageBytes;
          if (elect_one()) {
#pragma unroll
            for (int k = 0; k < 8; ++k) {
              const uint64_t a =
                  smem_desc_sw128(sQ + m * 32768 + (k >> 2) * 16384 + (k & 3) * 32, 16, 1024);
              const uint64_t bd =
                  smem_desc_sw128(kbase + (k >> 2) * 1024 + (k & 3) * 32, 16, 2048);
              mma_bf16(tmem + L::colS(m, buf), a, bd, idesc_qk, k > 0);
            }
            mma_commit(&sh.s_full[m][buf]);
            if (m == MT - 1) mma_commit(&sh.kv_empty[st]);
          }
        } else {
          if (!(ok = __all_sync(kFullMask, mbar_wait(&sh.p_full[m][buf], (t >> 1) & 1, abort))))
            break;
          const uint32_t vbase = sKV + st * L::kStageBytes + 16384;
          tc_fence_after();
          if (elect_one()) {
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const uint64_t bd = smem_desc_sw128(vbase + k * 4096, 1024, 2048);
              mma_bf16_tmem_a(tmem + L::colO(m), tmem + L::colS(m, buf) + k * 8, bd, idesc_pv,
                              (t > 0 || k > 0) ? 1u : 0u);
            }
            mma_commit(&sh.pv_done[m][buf]);
            if (m == MT - 1) mma_commit(&sh.kv_empty[st]);
          }
        }
        __syncwarp();
        issued_any = true;
      }
    }
    if (issued_any) {
      // every MMA this warp issued must finish before TMEM is freed
      if (elect_one()) mma_commit(&sh.mma_done[iss]);
      __syncwarp();
      int never = 0;
      mbar_wait(&sh.mma_done[iss], 0, &never);
    }
  } else if (warp >= 4) {
    // ---------------- softmax / epilogue ----------------
    const int m = (warp - 4) >> 2, wq = warp & 3;
    const int row = wq * 32 + lane;          // row in the M tile = TMEM lane
    const int grow = m * 128 + row;          // row in the CTA: head, token
    const int g = grow >> 6, r = grow & 63;
    const uint32_t lane_addr = uint32_t(wq * 32) << 16;
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true;
    for (int t = 0; t < n_tiles && ok; ++t) {
      const int buf = t & 1;
      if (!(ok = mbar_wait(&sh.s_full[m][buf], (t >> 1) & 1, abort))) break;
      tc_fence_after();
      float s[64];
      tmem_ld32(tmem + lane_addr + L::colS(m, buf), s);
      tmem_ld32(tmem + lane_addr + L::colS(m, buf) + 32, s + 32);
      tmem_wait_ld();
      const bool own = t == 0;
      const uint32_t mask = sh.tile_mask[t];
      if (own || mask != 0xffu) {
#pragma unroll
        for (int i = 0; i < 64; ++i) {
          const bool valid = ((mask >> (i >> 3)) & 1u) && (!own || i <= r);
          if (!valid) s[i] = -INFINITY;
        }
      }
      float m0 = fmax3(s[0], s[1], s[2]), m1 = fmax3(s[3], s[4], s[5]);
#pragma unroll
      for (int i = 6; i < 62; i += 4) {
        m0 = fmax3(m0, s[i], s[i + 1]);
        m1 = fmax3(m1, s[i + 2], s[i + 3]);
      }
      const float tmax = fmax3(m0, m1, fmaxf(s[62], s[63])) * scale_log2;
      if (t == 0) {
        m_run = tmax;
      } else if (tmax > m_run + 8.f) {
        // lazy rescale: only when the running max grows by more than 2^8
        if (!(ok = mbar_wait(&sh.pv_done[m][(t - 1) & 1], ((t - 1) >> 1) & 1, abort))) break;
        tc_fence_after();
        const float alpha = ex2_approx(m_run - tmax);
        l_run *= alpha;
        for (int c = 0; c < kD; c += 32) {
          float ov[32];
          tmem_ld32(tmem + lane_addr + L::colO(m) + c, ov);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) ov[i] *= alpha;
          tmem_st32(tmem + lane_addr + L::colO(m) + c, ov);
        }
        tmem_wait_st();
        m_run = tmax;
      }
      // p = 2^(s c - m): one packed FMA per pair, then the exponential
      const float2 c2 = make_float2(scale_log2, scale_log2);
      const float2 nm = make_float2(-m_run, -m_run);
      uint32_t pk[32];
      float2 acc = make_float2(0.f, 0.f);
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        float2 x = __ffma2_rn(make_float2(s[2 * i], s[2 * i + 1]), c2, nm);
        x.x = ex2_approx(x.x);
        x.y = ex2_approx(x.y);
        acc = __fadd2_rn(acc, x);
        pk[i] = pack_bf16x2(x.x, x.y);
      }
      l_run += acc.x + acc.y;
      // P(t) goes over the first 32 columns of its own S buffer
      tmem_st32_u(tmem + lane_addr + L::colS(m, buf), pk);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&sh.p_full[m][buf]);
    }
    if (ok)
      ok = mbar_wait(&sh.pv_done[m][(n_tiles - 1) & 1], ((n_tiles - 1) >> 1) & 1, abort);
    // O of this M tile goes out through shared memory, over its own Q tile
    // (every MMA that reads it has completed), in the layout Q came in:
    // [head][column half][64 rows][128 B], 128-byte swizzle; one TMA store
    // per head and column half
    uint8_t* stage = smem + L::kQ + m * 32768 + (row >> 6) * 8192 + r * 128;
    if (ok) {
      tc_fence_after();
      const float inv = 1.f / l_run;
      for (int c = 0; c < kD; c += 32) {
        float ov[32];
        tmem_ld32(tmem + lane_addr + L::colO(m) + c, ov);
        tmem_wait_ld();
#pragma unroll
        for (int q8 = 0; q8 < 4; ++q8) {
          const int ch = c / 8 + q8;
          const float* f = ov + 8 * q8;
          *reinterpret_cast<uint4*>(stage + (ch >> 3) * 16384 + (((ch & 7) ^ (r & 7)) << 4)) =
              make_uint4(pack_bf16x2(f[0] * inv, f[1] * inv), pack_bf16x2(f[2] * inv, f[3] * inv),
                         pack_bf16x2(f[4] * inv, f[5] * inv), pack_bf16x2(f[6] * inv, f[7] * inv));
        }
      }
      const int64_t orow =
          (int64_t(b) * n_q_heads + head0 + g) * s_len + int64_t(j) * kQBlock + r;
      lse[orow] = (m_run + log2f(l_run)) * 0.69314718055994530942f;
      fence_proxy_async_smem();
    }
    if (m == 0)
      named_barrier<1, 128>();
    else
      named_barrier<2, 128>();
    if (ok && row == 0) {
      for (int gg = 0; gg < 2; ++gg) {
        const int32_t orow0 =
            int32_t((int64_t(b) * n_q_heads + head0 + 2 * m + gg) * s_len + j * kQBlock);
        for (int hf = 0; hf < 2; ++hf)
          tma_store_2d(&tm_o, smem + L::kQ + m * 32768 + hf * 16384 + gg * 8192, hf * 64, orow0);
      }
      bulk_commit_group();
      // a chained dQ kernel reads O once this item's flag is set: the stores
      // must have completed, not only read shared memory
      if (done) {
        bulk_wait_all();
        fence_proxy_async_global();
      } else {
        bulk_wait_read_all();
      }
    }
    if (done) __threadfence();  // O and LSE before this item's completion flag
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, L::kTmemCols);
  }
  // fused forward + backward: this item's O and LSE are written
  if (done && tid == 0 && !*abort)
    flag_release(done + blockIdx.x + gridDim.x * (blockIdx.y + gridDim.y * blockIdx.z), token);
  // chained: this grid completes only after the routing grid has
  if (route_done) pdl_wait();
}

}  // namespace fwdtc
}  // namespace hga
