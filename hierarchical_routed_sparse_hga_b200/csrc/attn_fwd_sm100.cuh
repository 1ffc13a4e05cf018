// Step a4 on the 5th-generation tensor cores: exact-token attention of one
// query block over its selected 8-token groups plus its causal own block
// ("BMW如何通过重新设计注意力机制…", section "HGA的不同之处": only the selected
// groups' exact K/V enter the attention; the summaries only steer selection).
//
// One CTA per (batch, KV head, query block).  The G query heads that share
// the KV head share the selection, so the CTA stacks them into M = 64*G rows
// (MT = G/2 tiles of 128 rows) and every gathered K/V tile feeds all of them.
//
// Roles (warp-specialised, one CTA per SM: 192 KB of shared memory at MT=2):
//   warp 0      TMA producer: Q once (64 x 64 boxes), then per key tile the
//               8 selected groups of K and V as 8-row boxes (a group is a
//               contiguous 2 KiB run of [B,Hkv,T,d]) into a 3-stage ring;
//   warp 1      TMEM owner and MMA issuer: S = Q K^T into double-buffered TMEM
//               (per M tile), then O += P V with P from shared memory;
//   warps 4..   softmax, one warp group (4 warps = 128 TMEM lanes) per M
//               tile, one thread per row: masks (padding slots, causal own
//               block), online softmax in the log2 domain with lazy
//               rescaling (O in TMEM is rescaled only when the running max
//               grows by more than 2^8), P to shared memory (bf16, 128-byte
//               swizzle), epilogue O / l and LSE.
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
constexpr int kStages = 3;
constexpr int kMaxTiles = 33;  // 256 groups / 8 + own block

template <int MT>
struct Layout {
  static constexpr uint32_t kQ = 0;                                // [MT][2 halves][128][128 B]
  static constexpr uint32_t kKV = MT * 32768;                      // [stage][K 16 KB | V 16 KB]
  static constexpr uint32_t kStageBytes = 32768;
  static constexpr uint32_t kP = kKV + kStages * kStageBytes;      // [MT][128][128 B]
  static constexpr uint32_t kBytes = kP + MT * 16384;
  static constexpr uint32_t kDynSmem = kBytes + 1024;              // + alignment slack
  static constexpr uint32_t kThreads = 128 + 128 * MT;
  static constexpr uint32_t kTmemCols = MT == 2 ? 512 : 256;
  static constexpr uint32_t kColO = MT * 128;                      // S buffers first
};

struct Shared {
  uint64_t q_full;
  uint64_t kv_full[kStages];
  uint64_t kv_empty[kStages];
  uint64_t s_full[2][2];
  uint64_t s_free[2][2];
  uint64_t p_full[2];
  uint64_t pv_done[2];
  uint64_t mma_done;
  uint32_t tmem_base;
  int abort;
  int n_tiles;
  int grp[kMaxTiles * 8];
  uint8_t tile_mask[kMaxTiles];
};

constexpr uint32_t kTestDropFirstTile = 0x80000000u;  // test hook, see hga.h

template <int MT>
__global__ void __launch_bounds__(Layout<MT>::kThreads, 1)
    attn_fwd_tc_kernel(const __grid_constant__ CUtensorMap tm_q,
                       const __grid_constant__ CUtensorMap tm_k,
                       const __grid_constant__ CUtensorMap tm_v, int64_t ctx_cap,
                       int64_t q_begin, int s_len, int n_q_heads, int n_kv_heads,
                       int topk_groups, const int32_t* __restrict__ sel_grp, float scale_log2,
                       __nv_bfloat16* __restrict__ o, float* __restrict__ lse, uint32_t flags) {
  using L = Layout<MT>;
  constexpr int G = 2 * MT;
  extern __shared__ uint8_t dsmem_raw[];
  __shared__ Shared sh;
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(dsmem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sQ = smem_u32(smem + L::kQ);
  const uint32_t sKV = smem_u32(smem + L::kKV);
  const uint32_t sP = smem_u32(smem + L::kP);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int j = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int n_qb = s_len / kQBlock;
  const int64_t own_blk = (q_begin + int64_t(j) * kQBlock) / kBlock;
  volatile int* abort = &sh.abort;

  // ---- set-up: barriers, TMEM, the tile schedule -------------------------
  if (tid == 0) {
    mbar_init(&sh.q_full, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&sh.kv_full[s], 1);
      mbar_init(&sh.kv_empty[s], 1);
    }
    for (int m = 0; m < 2; ++m) {
      for (int u = 0; u < 2; ++u) {
        mbar_init(&sh.s_full[m][u], 1);
        mbar_init(&sh.s_free[m][u], 128);
      }
      mbar_init(&sh.p_full[m], 128);
      mbar_init(&sh.pv_done[m], 1);
    }
    mbar_init(&sh.mma_done, 1);
    sh.abort = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(&sh.tmem_base, L::kTmemCols);
    tmem_relinquish();
  }
  if (warp == 0) {
    // compact the valid selected groups (ascending order kept), pad the last
    // routed tile with copies of the first valid group (masked out later)
    const int32_t* srow = sel_grp + ((int64_t(b) * n_kv_heads + h) * n_qb + j) * topk_groups;
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
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sh.tmem_base;
  const int n_tiles = sh.n_tiles;

  if (warp == 0) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      prefetch_tmap(&tm_q);
      prefetch_tmap(&tm_k);
      prefetch_tmap(&tm_v);
      mbar_arrive_expect_tx(&sh.q_full, MT * 32768);
      for (int g = 0; g < G; ++g) {
        const int32_t row = int32_t((int64_t(b) * n_q_heads + h * G + g) * s_len + j * kQBlock);
        for (int hf = 0; hf < 2; ++hf) {
          uint8_t* dst = smem + L::kQ + (g >> 1) * 32768 + hf * 16384 + (g & 1) * 8192;
          tma_load_2d(dst, &tm_q, &sh.q_full, hf * 64, row);
        }
      }
      const int64_t kv_row0 = (int64_t(b) * n_kv_heads + h) * ctx_cap;
      int issued = 0;
      for (int t = 0; t < n_tiles; ++t) {
        const int st = t % kStages;
        if (t >= kStages && !mbar_wait(&sh.kv_empty[st], ((t / kStages) - 1) & 1, abort)) break;
        if ((flags & kTestDropFirstTile) && t == 0) continue;  // test hook: never armed
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
      // drain: wait (bounded, independent of abort) for the copies in flight
      int never = 0;
      mbar_wait(&sh.q_full, 0, &never, 2000000000LL);
      for (int t = issued - 1; t >= 0 && t >= issued - kStages; --t) {
        if ((flags & kTestDropFirstTile) && t == 0) continue;
        mbar_wait(&sh.kv_full[t % kStages], (t / kStages) & 1, &never, 2000000000LL);
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      constexpr uint32_t idesc_qk = idesc_bf16_f32(128, 64, 0, 0);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(128, kD, 0, 1);
      bool ok = mbar_wait(&sh.q_full, 0, abort);
      bool issued_any = false;
      tc_fence_after();
      for (int t = 0; ok && t <= n_tiles; ++t) {
        if (t < n_tiles) {
          const int st = t % kStages, buf = t & 1;
          if (!mbar_wait(&sh.kv_full[st], (t / kStages) & 1, abort)) break;
          for (int m = 0; m < MT && ok; ++m)
            if (t >= 2) ok = mbar_wait(&sh.s_free[m][buf], ((t >> 1) - 1) & 1, abort);
          if (!ok) break;
          tc_fence_after();
          const uint32_t kbase = sKV + st * L::kStageBytes;
          for (int m = 0; m < MT; ++m) {
            const uint32_t d = tmem + (m * 2 + buf) * 64;
#pragma unroll
            for (int k = 0; k < 8; ++k) {
              const uint64_t a =
                  smem_desc_sw128(sQ + m * 32768 + (k >> 2) * 16384 + (k & 3) * 32, 16, 1024);
              const uint64_t bd = smem_desc_sw128(kbase + (k >> 2) * 8192 + (k & 3) * 32, 16, 1024);
              mma_bf16(d, a, bd, idesc_qk, k > 0);
            }
            mma_commit(&sh.s_full[m][buf]);
          }
          issued_any = true;
        }
        if (t >= 1) {
          const int tt = t - 1, st = tt % kStages;
          const uint32_t vbase = sKV + st * L::kStageBytes + 16384;
          for (int m = 0; m < MT; ++m) {
            if (!(ok = mbar_wait(&sh.p_full[m], tt & 1, abort))) break;
            tc_fence_after();
            const uint32_t d = tmem + L::kColO + m * kD;
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const uint64_t a = smem_desc_sw128(sP + m * 16384 + k * 32, 16, 1024);
              const uint64_t bd = smem_desc_sw128(vbase + k * 2048, 8192, 1024);
              mma_bf16(d, a, bd, idesc_pv, (tt > 0 || k > 0) ? 1u : 0u);
            }
            mma_commit(&sh.pv_done[m]);
          }
          if (!ok) break;
          mma_commit(&sh.kv_empty[st]);
        }
      }
      if (issued_any) {
        // every MMA this thread issued must finish before TMEM is freed
        int never = 0;
        mma_commit(&sh.mma_done);
        mbar_wait(&sh.mma_done, 0, &never, 2000000000LL);
      }
    }
  } else if (warp >= 4) {
    // ---------------- softmax / epilogue ----------------
    const int m = (warp - 4) >> 2, wq = (warp - 4) & 3;
    const int row = wq * 32 + lane;          // row inside the M tile = TMEM lane
    const int grow = m * 128 + row;          // row inside the CTA: head g, token r
    const int g = grow >> 6, r = grow & 63;
    const uint32_t lane_addr = uint32_t(wq * 32) << 16;
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true;
    uint8_t* prow = smem + L::kP + m * 16384 + row * 128;
    for (int t = 0; t < n_tiles && ok; ++t) {
      const int buf = t & 1;
      if (!(ok = mbar_wait(&sh.s_full[m][buf], (t >> 1) & 1, abort))) break;
      tc_fence_after();
      float s[64];
      tmem_ld32(tmem + lane_addr + (m * 2 + buf) * 64, s);
      tmem_ld32(tmem + lane_addr + (m * 2 + buf) * 64 + 32, s + 32);
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(&sh.s_free[m][buf]);

      const bool own = t == n_tiles - 1;
      const uint32_t mask = sh.tile_mask[t];
      float tmax = -INFINITY;
#pragma unroll
      for (int i = 0; i < 64; ++i) {
        const bool valid = ((mask >> (i >> 3)) & 1u) && (!own || i <= r);
        s[i] = valid ? s[i] * scale_log2 : -INFINITY;
        tmax = fmaxf(tmax, s[i]);
      }
      if (t > 0 && !(ok = mbar_wait(&sh.pv_done[m], (t - 1) & 1, abort))) break;
      tc_fence_after();
      if (t == 0) {
        m_run = tmax;
      } else if (tmax > m_run + 8.f) {
        // lazy rescale: only when the running max grows by more than 2^8
        const float alpha = exp2f(m_run - tmax);
        l_run *= alpha;
        for (int c = 0; c < kD; c += 32) {
          float ov[32];
          tmem_ld32(tmem + lane_addr + L::kColO + m * kD + c, ov);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) ov[i] *= alpha;
          tmem_st32(tmem + lane_addr + L::kColO + m * kD + c, ov);
        }
        tmem_wait_st();
        m_run = tmax;
      }
      float psum = 0.f;
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        uint32_t w[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const float p0 = exp2f(s[8 * c + 2 * u] - m_run);
          const float p1 = exp2f(s[8 * c + 2 * u + 1] - m_run);
          psum += p0 + p1;
          __nv_bfloat162 pr = __floats2bfloat162_rn(p0, p1);
          w[u] = *reinterpret_cast<uint32_t*>(&pr);
        }
        *reinterpret_cast<uint4*>(prow + ((c ^ (row & 7)) << 4)) = make_uint4(w[0], w[1], w[2], w[3]);
      }
      l_run += psum;
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(&sh.p_full[m]);
    }
    if (ok) ok = mbar_wait(&sh.pv_done[m], (n_tiles - 1) & 1, abort);
    if (ok) {
      tc_fence_after();
      const float inv = 1.f / l_run;
      const int hq = h * G + g;
      const int64_t orow = (int64_t(b) * n_q_heads + hq) * s_len + int64_t(j) * kQBlock + r;
      __nv_bfloat16* odst = o + orow * kD;
      for (int c = 0; c < kD; c += 32) {
        float ov[32];
        tmem_ld32(tmem + lane_addr + L::kColO + m * kD + c, ov);
        tmem_wait_ld();
#pragma unroll
        for (int q8 = 0; q8 < 4; ++q8) {
          float f[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) f[i] = ov[8 * q8 + i] * inv;
          store8(odst + c + 8 * q8, f);
        }
      }
      lse[orow] = (m_run + log2f(l_run)) * 0.69314718055994530942f;
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

}  // namespace fwdtc
}  // namespace hga
