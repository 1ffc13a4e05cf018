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
//   same tiles as the forward, gathered by 3-D TMA boxes into a 3-stage ring) and
//   M tile: S = Q K^T and dP = dO V^T into one of two TMEM regions, then one
//   thread per row forms P = exp2(S c - LSE2), dS = P (dP - D) and stores it
//   as bf16 over the region's S columns, and dQ += dS K (A operand in tensor
//   memory) accumulates in TMEM; dQ = scale * dQ at the end.  D = rowsum(dO * O)
//   is computed here (warp shuffles) and saved for the next kernel.
//
// attn_bwd_dkdv_tc_kernel -- persistent: at most one CTA per SM, each taking
//   work units (batch, KV head, 64-key block of the active segment) from a
//   counter in the workspace (zeroed by the dQ kernel) until none is left,
//   the key blocks that the most query blocks can select first, so the
//   uneven units balance out over the SMs.  Per unit it visits, in
//   increasing order, every query block of the
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

// The dQ kernel visits the routed tiles first and the causal own block last
// (measured faster for it than the schedule's own-block-first order): its
// tile t is schedule tile t + 1, and its last tile is schedule tile 0.
__device__ __forceinline__ int sched_tile(int t, int n_tiles) {
  return t + 1 < n_tiles ? t + 1 : 0;
}

// ------------------------------------------------------------------------
// dQ kernel
// ------------------------------------------------------------------------
template <int MT>
struct DqLayout {
  static constexpr uint32_t kQ = 0;                              // [MT][2][128][128 B]
  static constexpr uint32_t kDO = MT * 32768;                    // same layout
  static constexpr uint32_t kKV = 2 * MT * 32768;                // [3 stages][K | V], group-major
  static constexpr uint32_t kStages = 3;
  static constexpr uint32_t kStageBytes = 32768;
  static constexpr uint32_t kBytes = kKV + kStages * kStageBytes;
  static constexpr uint32_t kDynSmem = kBytes + 1024;
  static constexpr uint32_t kThreads = 128 + 128 * MT;
  static constexpr uint32_t kTmemCols = 512;
  // TMEM columns: two S | dP regions (64 + 64 each); dS of an op, as bf16
  // pairs, goes over the first 32 columns of its own region once S and dP
  // are in registers; dQ of each M tile (128)
  static constexpr uint32_t colS(int r) { return r * 128; }
  static constexpr uint32_t colDP(int r) { return r * 128 + 64; }
  static constexpr uint32_t colDQ(int m) { return 256 + m * 128; }
};

struct DqShared {
  uint64_t q_full;
  uint64_t kv_full[3];
  uint64_t kv_empty[3];
  // [region]: op s = t * MT + m (tile t, M tile m) runs in region s & 1
  uint64_t sdp_full[2];   // S, dP of the op are in the region
  uint64_t ds_full[2];    // its dS is in the region
  uint64_t ds_done[2];    // dQ += dS K has completed: the region is free
  uint64_t mma_done[2];   // every MMA of issuer 0 (S, dP) / issuer 1 (dQ) has completed
  uint32_t tmem_base;
  int abort;
  int n_tiles;
  int d_arrived;          // rows whose D is written (fused forward + backward)
  int grp[kMaxTiles * 8];
  uint8_t tile_mask[kMaxTiles];
};



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
                          const __grid_constant__ CUtensorMap tm_dq, float* __restrict__ dvec,
                          int* __restrict__ unit_counter, const int* __restrict__ fwd_done,
                          int* __restrict__ d_done, uint32_t token, int* __restrict__ inv) {
  using L = DqLayout<MT>;
  // arrivals before this item's D flag: the softmax rows and warp 3's lanes
  constexpr int kArrive = 128 * MT + 32;
  constexpr int G = 2 * MT;
  constexpr int kSt = L::kStages;
  extern __shared__ uint8_t dsmem_raw[];
  __shared__ DqShared sh;
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(dsmem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sQ = smem_u32(smem + L::kQ), sDO = smem_u32(smem + L::kDO);
  const uint32_t sKV = smem_u32(smem + L::kKV);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int j = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int n_qb = s_len / kQBlock;
  const int64_t own_blk = (q_begin + int64_t(j) * kQBlock) / kBlock;
  const int item = j + n_qb * (h + gridDim.y * b);
  volatile int* abort = &sh.abort;

  if (tid == 0) {
    sh.d_arrived = 0;
    mbar_init(&sh.q_full, 1);
    for (int s = 0; s < kSt; ++s) {
      mbar_init(&sh.kv_full[s], 1);
      mbar_init(&sh.kv_empty[s], 2);  // the last S/dP and the last dQ of the tile
    }
    for (int r = 0; r < 2; ++r) {
      mbar_init(&sh.sdp_full[r], 1);
      mbar_init(&sh.ds_full[r], 128);
      mbar_init(&sh.ds_done[r], 1);
    }
    mbar_init(&sh.mma_done[0], 1);
    mbar_init(&sh.mma_done[1], 1);
    sh.abort = 0;
    fence_barrier_init();
  }
  // the previous kernel may still hold this SM's tensor memory or write
  // this kernel's inputs: wait for it before allocating or reading.  In a
  // fused forward + backward the previous kernel is that forward: this CTA
  // waits only for its own item's O and LSE (fwd_done), and everything the
  // forward waited for has completed (it let this grid start only then);
  // the two kernels' CTAs cannot share an SM (shared memory), so no forward
  // CTA holds this SM's tensor memory.
  if (!fwd_done) pdl_wait();
  // the dK/dV kernel that follows takes its work units from this counter
  if (tid == 0 && blockIdx.x == 0 && blockIdx.y == 0 && blockIdx.z == 0) {
    *unit_counter = 0;
    __threadfence();
  }
  if (tid == 0) {
    // Q and dO first: they do not depend on the selection
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
  }
  if (warp == 1) {
    tmem_alloc(&sh.tmem_base, L::kTmemCols);
    tmem_relinquish();
  }
  if (warp == 0)
    build_tile_schedule(sh, sel_grp + ((int64_t(b) * n_kv_heads + h) * n_qb + j) * topk_groups,
                        topk_groups, own_blk, lane);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  pdl_launch_dependents();  // after CTA 0 has zeroed the unit counter
  const uint32_t tmem = sh.tmem_base;
  const int n_tiles = sh.n_tiles;

  if (warp == 0) {
    // ---------------- TMA producer (whole warp; one elected lane issues) ----
    // 3-stage ring; stage layout [K | V], each [group][d half][8 rows][128 B]
    // (128-byte swizzle): one 3-D box (64 columns x 8 rows x 2 halves) per
    // group and tensor
    const int64_t kv_row0 = (int64_t(b) * n_kv_heads + h) * ctx_cap;
    int issued = 0;
    for (int t = 0; t < n_tiles; ++t) {
      const int st = t % kSt;
      const int si = sched_tile(t, n_tiles);
      const bool free_ok = t < kSt || mbar_wait(&sh.kv_empty[st], ((t / kSt) - 1) & 1, abort);
      if (!__all_sync(kFullMask, free_ok)) break;
      if (elect_one()) {
        mbar_arrive_expect_tx(&sh.kv_full[st], L::kStageBytes);
        uint8_t* kdst = smem + L::kKV + st * L::kStageBytes;
#pragma unroll
        for (int gi = 0; gi < 8; ++gi) {
          const int32_t row = int32_t(kv_row0 + int64_t(sh.grp[si * 8 + gi]) * kGroup);
          tma_load_3d(kdst + gi * 2048, &tm_k, &sh.kv_full[st], 0, row, 0);
          tma_load_3d(kdst + 16384 + gi * 2048, &tm_v, &sh.kv_full[st], 0, row, 0);
        }
      }
      __syncwarp();
      issued = t + 1;
    }
    // drain: wait (bounded, independent of abort) for the copies in flight
    if (lane == 0) {
      int never = 0;
      mbar_wait(&sh.q_full, 0, &never);
      for (int t = issued - 1; t >= 0 && t >= issued - kSt; --t)
        mbar_wait(&sh.kv_full[t % kSt], (t / kSt) & 1, &never);
    }
  } else if (warp == 1 || warp == 3) {
    // ---------------- MMA issuers (whole warp each, one lane issues) ----------
    // Ops s = t * MT + m (tile t, M tile m) alternate between the two TMEM
    // regions (region s & 1).  Warp 1 issues S = Q K^T and dP = dO V^T of op
    // s once the K/V of tile t are in and the region is back from op s - 2
    // (whose dQ has read its dS); warp 3 issues dQ += dS K of op s once its
    // dS is in.  Two issuers, so that a dQ never queues behind the sixteen
    // S/dP MMAs of the other M tile: the tensor core takes both streams.  The
    // stage of tile t is free once the last S/dP and the last dQ of the tile
    // have completed (two commits on kv_empty).
    const int iss = warp == 1 ? 0 : 1;
    if (iss == 1) {
      // the inverted selection for the dK/dV kernel: which groups of each
      // earlier block kb of the active segment this query block attends,
      // inv[b, h][kb][j] = token << 8 | mask (every entry of column j is
      // written, 0 for blocks it does not attend); one lane per block
      uint32_t mk0 = 0u, mk1 = 0u;
      const int64_t act0 = q_begin / kGroup;
      for (int i = 0; i < n_tiles * 8; ++i) {
        const int64_t ga = int64_t(sh.grp[i]) - act0;
        if (ga >= 0 && ga < int64_t(j) * kGroupsPerBlock) {
          const int kb = int(ga / kGroupsPerBlock);
          const uint32_t bit = 1u << int(ga % kGroupsPerBlock);
          if (kb == lane) mk0 |= bit;
          if (kb == lane + 32) mk1 |= bit;
        }
      }
      const uint32_t tk = (token & 0xffffffu) << 8;
      int* inv_bh = inv + (int64_t(b) * n_kv_heads + h) * n_qb * n_qb;
      if (lane < n_qb) inv_bh[lane * n_qb + j] = int(tk | mk0);
      if (lane + 32 < n_qb) inv_bh[(lane + 32) * n_qb + j] = int(tk | mk1);
      if (d_done) {
        __threadfence();
        if (atomicAdd(&sh.d_arrived, 1) == kArrive - 1 && !*abort)
          flag_release(d_done + item, token);
      }
    }
    constexpr uint32_t idesc_s = idesc_bf16_f32(128, 64, 0, 0);
    constexpr uint32_t idesc_dq = idesc_bf16_f32(128, kD, 0, 1);
    bool ok = __all_sync(kFullMask, mbar_wait(&sh.q_full, 0, abort));
    bool issued_any = false;
    const int n_ops = n_tiles * MT;
    for (int op = 0; ok && op < n_ops; ++op) {
      const int t = op / MT, m = op % MT, rg = op & 1;
      const uint32_t kb = sKV + (t % kSt) * L::kStageBytes;
      if (iss == 0) {
        bool ready = m != 0 || mbar_wait(&sh.kv_full[t % kSt], (t / kSt) & 1, abort);
        if (op >= 2) ready = ready && mbar_wait(&sh.ds_done[rg], ((op - 2) >> 1) & 1, abort);
        if (!(ok = __all_sync(kFullMask, ready))) break;
        tc_fence_after();
        if (elect_one()) {
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t ko = (kk >> 2) * 16384 + (kk & 3) * 32;
            const uint32_t bo = (kk >> 2) * 1024 + (kk & 3) * 32;
            mma_bf16(tmem + L::colS(rg), smem_desc_sw128(sQ + m * 32768 + ko, 16, 1024),
                     smem_desc_sw128(kb + bo, 16, 2048), idesc_s, kk > 0);
            mma_bf16(tmem + L::colDP(rg), smem_desc_sw128(sDO + m * 32768 + ko, 16, 1024),
                     smem_desc_sw128(kb + 16384 + bo, 16, 2048), idesc_s, kk > 0);
          }
          mma_commit(&sh.sdp_full[rg]);
          if (m == MT - 1) mma_commit(&sh.kv_empty[t % kSt]);
        }
      } else {
        if (!(ok = __all_sync(kFullMask, mbar_wait(&sh.ds_full[rg], (op >> 1) & 1, abort))))
          break;
        tc_fence_after();
        if (elect_one()) {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_bf16_tmem_a(tmem + L::colDQ(m), tmem + L::colS(rg) + kk * 8,
                            smem_desc_sw128(kb + kk * 4096, 1024, 2048), idesc_dq,
                            (t > 0 || kk > 0) ? 1u : 0u);
          mma_commit(&sh.ds_done[rg]);
          if (m == MT - 1) mma_commit(&sh.kv_empty[t % kSt]);
        }
      }
      __syncwarp();
      issued_any = true;
    }
    if (issued_any) {
      // every MMA this warp issued must finish before TMEM is freed
      if (elect_one()) mma_commit(&sh.mma_done[iss]);
      __syncwarp();
      int never = 0;
      mbar_wait(&sh.mma_done[iss], 0, &never);
    }
  } else if (warp >= 4) {
    const int m = (warp - 4) >> 2, wq = warp & 3;
    const int row = wq * 32 + lane;
    const int grow = m * 128 + row, g = grow >> 6, r = grow & 63;
    const uint32_t lane_addr = uint32_t(wq * 32) << 16;
    const int hq = h * G + g;
    const int64_t rix = (int64_t(b) * n_q_heads + hq) * s_len + int64_t(j) * kQBlock + r;
    // D = rowsum(dO * O), saved for the dK/dV kernel.  A warp takes two rows
    // per step (16 lanes x 16 B each): O by coalesced 256-byte row loads, all
    // issued first, dO from shared memory; lane i keeps the sum of row i.
    float dsum = 0.f;
    if ((!fwd_done || flag_wait(fwd_done + item, token, abort)) &&
        mbar_wait(&sh.q_full, 0, abort)) {
      const int half = lane >> 4, c = lane & 15;   // row of the pair, 16-byte chunk
      const uint8_t* dO_m = smem + L::kDO + m * 32768;
      uint4 ov[16];
#pragma unroll
      for (int p2 = 0; p2 < 16; ++p2) {
        const int rw = wq * 32 + 2 * p2 + half;    // row in the M tile
        const int gw = (m * 128 + rw) >> 6, tw = (m * 128 + rw) & 63;
        const int64_t orow =
            (int64_t(b) * n_q_heads + h * G + gw) * s_len + int64_t(j) * kQBlock + tw;
        ov[p2] = *reinterpret_cast<const uint4*>(o + orow * kD + c * 8);
      }
#pragma unroll
      for (int p2 = 0; p2 < 16; ++p2) {
        const int rw = wq * 32 + 2 * p2 + half;
        float df[8];
        load8(reinterpret_cast<const __nv_bfloat16*>(
                  dO_m + (c >> 3) * 16384 + rw * 128 + (((c & 7) ^ (rw & 7)) << 4)),
              df);
        const uint32_t w4[4] = {ov[p2].x, ov[p2].y, ov[p2].z, ov[p2].w};
        float part = 0.f;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          part = fmaf(__uint_as_float(w4[i] << 16), df[2 * i], part);
          part = fmaf(__uint_as_float(w4[i] & 0xffff0000u), df[2 * i + 1], part);
        }
#pragma unroll
        for (int off = 8; off > 0; off >>= 1) part += __shfl_xor_sync(0xffffffffu, part, off);
        // row 2 p2 + h' is now in every lane of half h': lane 2 p2 + h' takes it
        const float mine = __shfl_sync(0xffffffffu, part, 16 * (lane & 1));
        if ((lane >> 1) == p2) dsum = mine;
      }
    }
    dvec[rix] = dsum;
    if (d_done) {
      // fused: the last of this CTA's rows to write D publishes the item
      __threadfence();
      if (atomicAdd(&sh.d_arrived, 1) == kArrive - 1 && !*abort)
        flag_release(d_done + item, token);
    }
    const float lse2 = lse[rix] * 1.4426950408889634f;
    const float2 c2 = make_float2(scale_log2, scale_log2);
    const float2 nl = make_float2(-lse2, -lse2);
    const float2 nd = make_float2(-dsum, -dsum);
    bool ok = true;
    for (int t = 0; t < n_tiles && ok; ++t) {
      const int op = t * MT + m, rg = op & 1;
      if (!(ok = mbar_wait(&sh.sdp_full[rg], (op >> 1) & 1, abort))) break;
      tc_fence_after();
      float sv[64], dp[64];
      tmem_ld32(tmem + lane_addr + L::colS(rg), sv);
      tmem_ld32(tmem + lane_addr + L::colS(rg) + 32, sv + 32);
      tmem_ld32(tmem + lane_addr + L::colDP(rg), dp);
      tmem_ld32(tmem + lane_addr + L::colDP(rg) + 32, dp + 32);
      tmem_wait_ld();
      const bool own = t == n_tiles - 1;
      const uint32_t mask = sh.tile_mask[sched_tile(t, n_tiles)];
      if (own || mask != 0xffu) {
#pragma unroll
        for (int i = 0; i < 64; ++i) {
          const bool valid = ((mask >> (i >> 3)) & 1u) && (!own || i <= r);
          if (!valid) sv[i] = -INFINITY;
        }
      }
      uint32_t packed[32];
#pragma unroll
      for (int i = 0; i < 64; i += 2) {
        float2 x = __ffma2_rn(make_float2(sv[i], sv[i + 1]), c2, nl);
        x.x = ex2_approx(x.x);
        x.y = ex2_approx(x.y);
        const float2 y = __fmul2_rn(x, __fadd2_rn(make_float2(dp[i], dp[i + 1]), nd));
        packed[i / 2] = pack_bf16x2(y.x, y.y);
      }
      // dS over the S columns of this op's region (A operand of dQ += dS K)
      tmem_st32_u(tmem + lane_addr + L::colS(rg), packed);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&sh.ds_full[rg]);
    }
    if (ok) {
      const int op = (n_tiles - 1) * MT + m;
      ok = mbar_wait(&sh.ds_done[op & 1], (op >> 1) & 1, abort);
    }
    // dQ of this M tile goes out through shared memory, over its own Q tile
    // (every MMA that reads it has completed), in the layout Q came in; one
    // TMA store per head and column half
    uint8_t* stage = smem + L::kQ + m * 32768 + (row >> 6) * 8192 + r * 128;
    if (ok) {
      tc_fence_after();
      for (int c = 0; c < kD; c += 32) {
        float vv[32];
        tmem_ld32(tmem + lane_addr + L::colDQ(m) + c, vv);
        tmem_wait_ld();
#pragma unroll
        for (int q8 = 0; q8 < 4; ++q8) {
          const int ch = c / 8 + q8;
          const float* f = vv + 8 * q8;
          *reinterpret_cast<uint4*>(stage + (ch >> 3) * 16384 + (((ch & 7) ^ (r & 7)) << 4)) =
              make_uint4(pack_bf16x2(f[0] * scale, f[1] * scale),
                         pack_bf16x2(f[2] * scale, f[3] * scale),
                         pack_bf16x2(f[4] * scale, f[5] * scale),
                         pack_bf16x2(f[6] * scale, f[7] * scale));
        }
      }
      fence_proxy_async_smem();
    }
    if (m == 0)
      named_barrier<1, 128>();
    else
      named_barrier<2, 128>();
    if (ok && row == 0) {
      for (int gg = 0; gg < 2; ++gg) {
        const int32_t row0 =
            int32_t((int64_t(b) * n_q_heads + h * G + 2 * m + gg) * s_len + j * kQBlock);
        for (int hf = 0; hf < 2; ++hf)
          tma_store_2d(&tm_dq, smem + L::kQ + m * 32768 + hf * 16384 + gg * 8192, hf * 64, row0);
      }
      bulk_commit_group();
      bulk_wait_read_all();
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, L::kTmemCols);
  }
  // fused: this grid completes only after the forward grid has, so that the
  // kernels after it on the stream see both complete
  if (fwd_done) pdl_wait();
}

// ------------------------------------------------------------------------
// dK / dV kernel
// ------------------------------------------------------------------------
// Work item = (attending query block jj, M tile m): 128 query rows = two heads
// x 64 tokens.  Items run through two buffers (u = item & 1): Q_m / dO_m by
// TMA (64-row boxes), S / dP in TMEM, P / dS in shared memory; warp group u
// does the softmax of the items of buffer u, so one group's softmax overlaps
// the other buffer's MMAs and loads.
struct KvLayout {
  static constexpr uint32_t kK = 0;                    // [2 halves][64][128 B]
  static constexpr uint32_t kV = 16384;
  static constexpr uint32_t kQD = 32768;               // [buf][Q_m 32 KB | dO_m 32 KB]
  static constexpr uint32_t kQDBytes = 65536;
  static constexpr uint32_t kPD = kQD + 2 * kQDBytes;  // [buf][P 16 KB | dS 16 KB]
  static constexpr uint32_t kPDBytes = 32768;
  static constexpr uint32_t kBytes = kPD + 2 * kPDBytes;
  static constexpr uint32_t kDynSmem = kBytes + 1024;
  static constexpr uint32_t kThreads = 384;
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t colS(int u) { return u * 128; }
  static constexpr uint32_t colDP(int u) { return u * 128 + 64; }
  // dV^T and dK^T of a unit in one of two sets (unit n uses set n & 1), so
  // that a unit's epilogue can read its set while the next unit's MMAs
  // accumulate into the other
  static constexpr uint32_t colDV(int set) { return 256 + set * 128; }
  static constexpr uint32_t colDK(int set) { return 320 + set * 128; }
};

struct KvShared {
  uint64_t kv_full;
  uint64_t qd_full[2];
  uint64_t qd_empty[2];
  uint64_t sdp_full[2];
  uint64_t pds_full[2];
  uint64_t mma_done;
  uint64_t issued_all;  // the producer has requested every item of the unit
  uint64_t plan_full;   // the next unit's plan is in (phase n: the plan of unit n)
  uint32_t tmem_base;
  int abort;
  // plans of two units (slot = unit index & 1): the unit, its item count,
  // the attending query blocks in increasing order and their group masks
  int unit[2];
  int n_items[2];
  int masks[2][64];
  int js[2][64];
};

template <int MT>
__global__ void __launch_bounds__(KvLayout::kThreads, 1)
    attn_bwd_dkdv_tc_kernel(const __grid_constant__ CUtensorMap tm_q,
                            const __grid_constant__ CUtensorMap tm_do,
                            const __grid_constant__ CUtensorMap tm_k,
                            const __grid_constant__ CUtensorMap tm_v, int64_t ctx_cap,
                            int64_t q_begin, int s_len, int batch, int n_q_heads, int n_kv_heads,
                            int topk_groups, const int32_t* __restrict__ sel_grp, float scale,
                            float scale_log2, const float* __restrict__ lse,
                            const float* __restrict__ dvec, __nv_bfloat16* __restrict__ dk,
                            __nv_bfloat16* __restrict__ dv, int* __restrict__ unit_counter,
                            const int* __restrict__ d_done, uint32_t token,
                            const int* __restrict__ inv) {
  using L = KvLayout;
  constexpr int G = 2 * MT;
  extern __shared__ uint8_t dsmem_raw[];
  __shared__ KvShared sh;
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(dsmem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sK = smem_u32(smem + L::kK), sV = smem_u32(smem + L::kV);
  const uint32_t sQD = smem_u32(smem + L::kQD), sPD = smem_u32(smem + L::kPD);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int n_qb = s_len / kQBlock;
  const int n_bh = batch * n_kv_heads, n_units = n_qb * n_bh;
  // Q_m and dO_m of query block jj (two heads x 64 rows) into Q/dO buffer u
  auto load_qd = [&](int u, int b, int h, int jj, int m) {
    mbar_arrive_expect_tx(&sh.qd_full[u], 65536);
    uint8_t* dst = smem + L::kQD + u * L::kQDBytes;
    for (int g = 0; g < 2; ++g) {
      const int32_t row =
          int32_t((int64_t(b) * n_q_heads + h * G + 2 * m + g) * s_len + jj * kQBlock);
      for (int hf = 0; hf < 2; ++hf) {
        tma_load_2d(dst + hf * 16384 + g * 8192, &tm_q, &sh.qd_full[u], hf * 64, row);
        tma_load_2d(dst + 32768 + hf * 16384 + g * 8192, &tm_do, &sh.qd_full[u], hf * 64,
                    row);
      }
    }
  };
  // K and V of key block gblk of (b, h)
  auto load_kv = [&](int b, int h, int64_t gblk) {
    const int32_t krow = int32_t((int64_t(b) * n_kv_heads + h) * ctx_cap + gblk * kBlock);
    mbar_arrive_expect_tx(&sh.kv_full, 32768);
    for (int gi = 0; gi < 8; ++gi)
      for (int hf = 0; hf < 2; ++hf) {
        tma_load_2d(smem + L::kK + hf * 8192 + gi * 1024, &tm_k, &sh.kv_full, hf * 64,
                    krow + gi * kGroup);
        tma_load_2d(smem + L::kV + hf * 8192 + gi * 1024, &tm_v, &sh.kv_full, hf * 64,
                    krow + gi * kGroup);
      }
  };
  volatile int* abort = &sh.abort;
  // The plan of the next unit (one warp, all lanes): claim it from the
  // counter, then find the later query blocks of the segment that selected
  // groups of its key block (only query blocks after kb can).  Their dQ CTAs
  // wrote the inverted selection, tagged with the call's token, before
  // releasing their D flags; the entry and (fused) the flag are read in one
  // round, and an entry that is not yet this call's is read again once the
  // flag is in.  The own block is always the first item.
  auto plan = [&](int slot) {
    int w = 0;
    if (lane == 0) w = *abort ? n_units : atomicAdd(unit_counter, 1);
    w = __shfl_sync(kFullMask, w, 0);
    int n = 0;
    if (w < n_units) {
      const int kb = w / n_bh, bh = w % n_bh;
      const int* inv_row = inv + (int64_t(bh) * n_qb + kb) * n_qb;
      const uint32_t tk = token & 0xffffffu;
      for (int c0 = kb; c0 < n_qb; c0 += 32) {
        const int jj = c0 + lane;
        int mask = 0;
        if (jj < n_qb) {
          uint32_t v = jj > kb ? uint32_t(__ldcg(inv_row + jj)) : 0u;
          const bool ready = !d_done || flag_wait(d_done + bh * n_qb + jj, token, abort);
          if (jj == kb) {
            mask = 0xff;
          } else if (ready) {
            if ((v >> 8) != tk) v = uint32_t(__ldcg(inv_row + jj));
            if ((v >> 8) != tk)
              latch_status(HGA_ERR_DEVICE_CHECK);
            else
              mask = int(v & 0xffu);
          }
        }
        const bool on = mask != 0;
        const unsigned ball = __ballot_sync(kFullMask, on);
        if (on) {
          sh.js[slot][n + __popc(ball & ((1u << lane) - 1u))] = jj;
          sh.masks[slot][jj] = mask;
        }
        n += __popc(ball);
      }
    }
    if (lane == 0) {
      sh.unit[slot] = w;
      sh.n_items[slot] = n * MT;
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&sh.plan_full);
    __syncwarp();
  };
  pdl_launch_dependents();

  if (tid == 0) {
    mbar_init(&sh.kv_full, 1);
    for (int u = 0; u < 2; ++u) {
      mbar_init(&sh.qd_full[u], 1);
      mbar_init(&sh.qd_empty[u], 1);
      mbar_init(&sh.sdp_full[u], 1);
      mbar_init(&sh.pds_full[u], 128);
    }
    mbar_init(&sh.mma_done, 2);  // one commit from each issuer per unit
    mbar_init(&sh.issued_all, 1);
    mbar_init(&sh.plan_full, 1);
    sh.abort = 0;
    fence_barrier_init();
  }
  // the previous kernel may still hold this SM's tensor memory or write
  // this kernel's inputs (the dQ kernel zeroes the unit counter): wait for
  // it.  In a fused forward + backward each unit instead waits for the D of
  // the query blocks it visits (d_done); the counter was zeroed before the
  // dQ grid let this one start, and the two kernels' CTAs cannot share an SM.
  if (!d_done) pdl_wait();
  if (tid == 0) {
    prefetch_tmap(&tm_q);
    prefetch_tmap(&tm_do);
    prefetch_tmap(&tm_k);
    prefetch_tmap(&tm_v);
  }
  if (warp == 1) {
    tmem_alloc(&sh.tmem_base, L::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sh.tmem_base;

  // Work units (key block kb, batch x KV head) in order of kb, so the blocks
  // that the most query blocks can select come first; each CTA takes the
  // next unit from the counter until none is left.  Item indices run on
  // across units (it_base), so every barrier's phase sequence continues.
  // Warp 2 plans unit n + 1 while unit n runs (once unit n's last item has
  // been requested, so that a CTA does not hold a unit long before it can
  // start it), and the producer requests the next unit's K/V and first items
  // as soon as unit n's MMAs are done, under unit n's epilogue.
  // dV and dK of unit w from tensor-memory set `set` (warp group 0: TMEM
  // lanes 0..127 are the 128 head dims), once every MMA of that unit has
  // completed (its mma_done phase, parity `par`)
  auto epilogue = [&](int set, int w, int par) {
    if (!mbar_wait(&sh.mma_done, par, abort)) return;
    tc_fence_after();
    const int wq = warp & 3, dcol = wq * 32 + lane;
    const uint32_t lane_addr = uint32_t(wq * 32) << 16;
    const int ekb = w / n_bh, ebh = w % n_bh;
    const int eb = ebh / n_kv_heads, eh = ebh % n_kv_heads;
    const int64_t base = ((int64_t(eb) * n_kv_heads + eh) * s_len + int64_t(ekb) * kBlock) * kD;
    for (int c = 0; c < 64; c += 32) {
      float vv[32], kk[32];
      tmem_ld32(tmem + lane_addr + L::colDV(set) + c, vv);
      tmem_ld32(tmem + lane_addr + L::colDK(set) + c, kk);
      tmem_wait_ld();
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const int64_t at = base + int64_t(c + i) * kD + dcol;
        dv[at] = __float2bfloat16_rn(vv[i]);
        dk[at] = __float2bfloat16_rn(kk[i] * scale);
      }
    }
  };
  if (warp == 2) plan(0);
  __syncthreads();
  int it_base = 0;
  int prev_w = -1;  // the unit whose epilogue is still to run (warp group 0)
  // producer (warp 0): what it has already requested of the next unit
  bool ahead_kv = false;
  int ahead_items = 0;
  int un = 0;
  for (;; ++un) {
    const int slot = un & 1;
    const int w = sh.unit[slot];
    if (w >= n_units) break;
    const int kb = w / n_bh, bh = w % n_bh, b = bh / n_kv_heads, h = bh % n_kv_heads;
    const int64_t gblk = q_begin / kBlock + kb;  // global index of this key block
    const int n_items = sh.n_items[slot];
    const int* js = sh.js[slot];
    const int* masks = sh.masks[slot];

    if (warp == 0) {
      // ---------------- TMA producer (whole warp; one elected lane issues) --
      // this block's keys and values, unless requested during the last unit
      if (!ahead_kv && elect_one()) load_kv(b, h, gblk);
      __syncwarp();
      int issued = ahead_items;
      for (int it = issued; it < n_items; ++it) {
        const int gi = it_base + it, u = gi & 1;
        const bool free_ok =
            gi < 2 || mbar_wait(&sh.qd_empty[u], ((gi >> 1) - 1) & 1, abort);
        if (!__all_sync(kFullMask, free_ok)) break;
        const int jj = js[it / MT], m = it % MT;
        if (elect_one()) load_qd(u, b, h, jj, m);
        __syncwarp();
        issued = it + 1;
      }
      if (elect_one()) mbar_arrive(&sh.issued_all);
      __syncwarp();
      // drain: wait (bounded, independent of abort) for this unit's copies,
      // before the next unit's requests arm the same barriers again
      if (lane == 0) {
        int never = 0;
        mbar_wait(&sh.kv_full, un & 1, &never);
        for (int it = issued - 1; it >= 0 && it >= issued - 2; --it) {
          const int gi = it_base + it;
          mbar_wait(&sh.qd_full[gi & 1], (gi >> 1) & 1, &never);
        }
      }
      __syncwarp();
      // the next unit: once its plan is in and every MMA of this unit has
      // completed (the K/V tiles and both Q/dO buffers are free), its K/V
      // and its first two items (item i of it reuses the buffer of this
      // unit's item n_items - 2 + i, whose copy has landed: the drain)
      ahead_kv = false;
      ahead_items = 0;
      const bool next_ok =
          issued == n_items &&
          __all_sync(kFullMask, mbar_wait(&sh.plan_full, (un + 1) & 1, abort) &&
                                    mbar_wait(&sh.mma_done, un & 1, abort) && !*abort);
      const int w2 = sh.unit[slot ^ 1];
      if (next_ok && w2 < n_units) {
        const int kb2 = w2 / n_bh, bh2 = w2 % n_bh;
        const int b2 = bh2 / n_kv_heads, h2 = bh2 % n_kv_heads;
        const int n2 = min(2, sh.n_items[slot ^ 1]);
        if (elect_one()) {
          load_kv(b2, h2, q_begin / kBlock + kb2);
          for (int it = 0; it < n2; ++it)
            load_qd((it_base + n_items + it) & 1, b2, h2, sh.js[slot ^ 1][it / MT], it % MT);
        }
        __syncwarp();
        ahead_kv = true;
        ahead_items = n2;
      }
    } else if (warp == 2) {
      // ---------------- planner: the next unit, once this one is requested --
      mbar_wait(&sh.issued_all, un & 1, abort);
      plan(slot ^ 1);
    } else if (warp == 1 || warp == 3) {
      // ---------------- MMA issuers (whole warp each, one lane issues) ------
      // Warp 1 issues S/dP(i) into TMEM buffer i & 1 once Q/dO of item i
      // are in and the softmax of item i - 2 has taken that buffer's S and
      // dP (its P/dS are then in shared memory); warp 3 issues dV/dK(i) once
      // P/dS(i) are in.  Two issuers, so that a ready dV/dK never queues
      // behind the sixteen S/dP MMAs of the next item.
      const int iss = warp == 1 ? 0 : 1;
      constexpr uint32_t idesc_s = idesc_bf16_f32(128, 64, 0, 0);
      constexpr uint32_t idesc_t = idesc_bf16_f32(128, 64, 1, 1);
      bool ok = __all_sync(kFullMask, mbar_wait(&sh.kv_full, un & 1, abort));
      for (int it = 0; ok && it < n_items; ++it) {
        const int gi = it_base + it, u = gi & 1;
        const uint32_t qd = sQD + u * L::kQDBytes;
        if (iss == 0) {
          bool ready = mbar_wait(&sh.qd_full[u], (gi >> 1) & 1, abort);
          if (it >= 2) ready = ready && mbar_wait(&sh.pds_full[u], ((gi - 2) >> 1) & 1, abort);
          if (!(ok = __all_sync(kFullMask, ready))) break;
          tc_fence_after();
          if (elect_one()) {
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
              const uint32_t ao = (kk >> 2) * 16384 + (kk & 3) * 32;
              const uint32_t bo = (kk >> 2) * 8192 + (kk & 3) * 32;
              mma_bf16(tmem + L::colS(u), smem_desc_sw128(qd + ao, 16, 1024),
                       smem_desc_sw128(sK + bo, 16, 1024), idesc_s, kk > 0);
              mma_bf16(tmem + L::colDP(u), smem_desc_sw128(qd + 32768 + ao, 16, 1024),
                       smem_desc_sw128(sV + bo, 16, 1024), idesc_s, kk > 0);
            }
            mma_commit(&sh.sdp_full[u]);
          }
        } else {
          // dV^T += dO^T P and dK^T += Q^T dS over this item's 128 query rows
          if (!(ok = __all_sync(kFullMask, mbar_wait(&sh.pds_full[u], (gi >> 1) & 1, abort))))
            break;
          const uint32_t pd = sPD + u * L::kPDBytes;
          tc_fence_after();
          if (elect_one()) {
#pragma unroll
            for (int s8 = 0; s8 < 8; ++s8) {
              const uint32_t ro = s8 * 2048;
              const uint32_t acc = (it > 0 || s8 > 0) ? 1u : 0u;
              mma_bf16(tmem + L::colDV(un & 1), smem_desc_sw128(qd + 32768 + ro, 16384, 1024),
                       smem_desc_sw128(pd + ro, 8192, 1024), idesc_t, acc);
              mma_bf16(tmem + L::colDK(un & 1), smem_desc_sw128(qd + ro, 16384, 1024),
                       smem_desc_sw128(pd + 16384 + ro, 8192, 1024), idesc_t, acc);
            }
            mma_commit(&sh.qd_empty[u]);
          }
        }
        __syncwarp();
      }
      // one mma_done phase per unit (a commit from each issuer): every MMA of
      // this unit has finished before its epilogue reads TMEM and before the
      // next unit overwrites the tiles in shared memory (a commit with none
      // pending arrives at once)
      if (elect_one()) mma_commit(&sh.mma_done);
      __syncwarp();
      int never = 0;
      mbar_wait(&sh.mma_done, un & 1, &never);
    } else if (warp >= 4) {
      // ---------------- softmax (two warp groups, one per buffer) --------------
      const int u = (warp - 4) >> 2, wq = warp & 3;
      const int row = wq * 32 + lane;
      const int g = row >> 6, r = row & 63;
      const uint32_t lane_addr = uint32_t(wq * 32) << 16;
      const float2 c2 = make_float2(scale_log2, scale_log2);
      bool ok = true;
      uint8_t* prow = smem + L::kPD + u * L::kPDBytes + row * 128;
      uint8_t* drow = prow + 16384;
      // warp group 0 first stores the previous unit's dV and dK (its set is
      // not touched by this unit's MMAs)
      if (u == 0 && prev_w >= 0 && !*abort) epilogue((un - 1) & 1, prev_w, (un - 1) & 1);
      // this group's items: those whose running index has parity u
      for (int it = (u - it_base) & 1; it < n_items && ok; it += 2) {
        const int gi = it_base + it;
        const int jj = js[it / MT], m = it % MT;
        const bool own = jj == kb;
        const uint32_t mask = masks[jj];
        const int hq = h * G + 2 * m + g;
        const int64_t rix = (int64_t(b) * n_q_heads + hq) * s_len + int64_t(jj) * kQBlock + r;
        const float lse2 = lse[rix] * 1.4426950408889634f;
        const float dsum = dvec[rix];
        const float2 nl = make_float2(-lse2, -lse2), nd = make_float2(-dsum, -dsum);
        if (!(ok = mbar_wait(&sh.sdp_full[u], (gi >> 1) & 1, abort))) break;
        tc_fence_after();
        const bool full = !own && mask == 0xffu;
#pragma unroll
        for (int hb = 0; hb < 2; ++hb) {
          float sv[32], dp[32];
          tmem_ld32(tmem + lane_addr + L::colS(u) + hb * 32, sv);
          tmem_ld32(tmem + lane_addr + L::colDP(u) + hb * 32, dp);
          tmem_wait_ld();
          if (!full) {
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              const int key = hb * 32 + i;
              const bool valid = ((mask >> (key >> 3)) & 1u) && (!own || key <= r);
              if (!valid) sv[i] = -INFINITY;
            }
          }
          uint32_t pk[16], dk2[16];
#pragma unroll
          for (int i = 0; i < 32; i += 2) {
            float2 p = __ffma2_rn(make_float2(sv[i], sv[i + 1]), c2, nl);
            p.x = ex2_approx(p.x);
            p.y = ex2_approx(p.y);
            const float2 d2 = __fmul2_rn(p, __fadd2_rn(make_float2(dp[i], dp[i + 1]), nd));
            pk[i / 2] = pack_bf16x2(p.x, p.y);
            dk2[i / 2] = pack_bf16x2(d2.x, d2.y);
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
        mbar_arrive(&sh.pds_full[u]);
      }
    }
    it_base += n_items;
    prev_w = w;
    // end of the unit: every role is done with its barriers, tiles and TMEM
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (*abort) break;
  }
  // the last unit's dV and dK (the loop ended at a unit that does not exist)
  if (warp >= 4 && warp < 8 && prev_w >= 0 && !*abort) epilogue((un - 1) & 1, prev_w, (un - 1) & 1);
  // copies the producer requested for a unit that will not run (the loop
  // ended on an abort): wait for them (bounded, independent of abort)
  if (warp == 0 && lane == 0 && ahead_kv) {
    int never = 0;
    mbar_wait(&sh.kv_full, (un + 1) & 1, &never);
    for (int it = 0; it < ahead_items; ++it) {
      const int gi = it_base + it;
      mbar_wait(&sh.qd_full[gi & 1], (gi >> 1) & 1, &never);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, L::kTmemCols);
  }
  // fused: this grid completes only after the dQ grid has
  if (d_done) pdl_wait();
}

}  // namespace bwdtc
}  // namespace hga
