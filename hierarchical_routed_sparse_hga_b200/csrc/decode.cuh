// Decode: one new token per sequence, routed against the resident summaries
// and attending to its selection ("Long-Context Fine-Tuning with Limited
// VRAM", adnankhan.ai notes, section "Raw Abstract / Excerpt": HGA can also
// be used for generation; routing as in "BMW如何通过重新设计注意力机制…",
// section "HGA的不同之处").
//
// The query block of a decode step is the one token: qbar is the mean of its
// query over the G heads of the KV head; the candidates are the complete
// blocks before the token's own block; the token attends to the selected
// groups' tokens and to its own block up to and including itself.
//
// One thread-block cluster of nc CTAs per (sequence, KV head), nc in
// {1, 2, 4, 8} chosen at launch so that the grid fills the GPU about once
// (8 for a single sequence, 1 from about 40 sequences of 8 KV heads up).
// Every phase is latency- or HBM-bound:
//   0. the token's own block is known at once: each CTA starts bulk copies of
//      its share of those K/V rows into shared memory;
//   1. each CTA scores a contiguous share of the J candidate blocks
//      (qbar . bsum), keeps its local top-k_b and stores them into every CTA
//      of the cluster (distributed shared memory) at its rank's slot; one
//      cluster barrier; every CTA selects the top-k_b of the nc x k_b
//      finalists (the global top-k_b is a subset of their union; the slots
//      in rank order are in ascending block order, so ties keep the lower
//      block);
//   2. each CTA scores a share of the 8 k_b groups of the kept blocks and
//      stores the scores into every CTA; one cluster barrier; every CTA
//      selects the top-k_g groups;
//   3. the attended tokens are dealt out in 8-token units (the own block's
//      first, then the selected groups in ascending order): unit u goes to
//      CTA u mod nc, which bulk-copies its K/V rows (2 KiB per tensor at
//      d = 128, bf16) into shared memory and runs an online softmax per
//      query head over them (a warp takes 4 tokens at a time, 8 lanes per
//      token);
//   4. warps merge their (max, sum, output) partials in a fixed order; each
//      CTA stores its partial into rank 0, which merges them in rank order
//      after one cluster barrier and writes O and LSE.
// Every merge runs in a fixed order, so results are deterministic.
#pragma once

#include <cooperative_groups.h>

#include "hga_common.cuh"
#include "route.cuh"
#include "sm100_ptx.cuh"

namespace hga {
namespace dec {

namespace cg = cooperative_groups;

constexpr int kMaxC = 8;               // CTAs per cluster, at most (portable size)
constexpr int kThreads = kRouteThreads;  // score_rows() is written for this count
constexpr int kWarps = kThreads / 32;
constexpr int kMaxKb = 64;
constexpr int kMaxKg = 256;
constexpr int kMaxMerged = kMaxC * kMaxKb;  // level-1 finalists of the whole cluster
constexpr int kMaxN2 = 8 * kMaxKb;          // level-2 candidates
constexpr int kStageBudget = 64 * 1024;     // shared memory for K/V rows per CTA
constexpr int kMinStageUnits = 8;           // the own block's units always fit one round
constexpr int kScoreRows = 8;               // summary rows in flight per warp

template <int D, int G>
struct Shared {
  alignas(16) float qb[D];                  // mean query (score_rows reads it as float4)
  alignas(16) float qh[G][D];               // the G query rows
  alignas(16) uint32_t fin_key[kMaxKb];     // this CTA's level-1 finalists
  int fin_idx[kMaxKb];
  alignas(16) uint32_t mkey[kMaxMerged];    // every CTA's finalists, at its rank's slot
  int midx[kMaxMerged];
  uint8_t msel[kMaxMerged];
  int blocks[kMaxKb];
  alignas(16) uint32_t key2[kMaxN2];        // level-2 scores, filled by every CTA
  uint8_t sel2[kMaxN2];
  int grp[kMaxKg];
  int hist[256];
  int scratch[kWarps + 1];
  float wm[kWarps][G], wl[kWarps][G];
  float pm[kMaxC][G], pl[kMaxC][G];          // the CTAs' partials (rank 0's copy is read)
  alignas(8) uint64_t bar_own, bar_rt;
  int abort;
};

template <int D, int G>
__host__ __device__ constexpr size_t shared_bytes() {
  return (sizeof(Shared<D, G>) + 127) & ~size_t(127);
}

// bytes of one 8-token unit of one tensor
template <typename T, int D>
__host__ __device__ constexpr uint32_t unit_bytes() {
  return uint32_t(kGroup * D * sizeof(T));
}

// dynamic shared memory: Shared | K/V stage [stage_units][2][8][D] (after
// the attention it holds the warps' partial outputs [kWarps][G][D] float) |
// the CTAs' partial outputs [nc][G][D] float (rank 0's copy is read) |
// level-1 keys [share_cap] | level-1 flags [share_cap]
template <typename T, int D, int G>
__host__ __device__ inline size_t stage_bytes(int stage_units) {
  return size_t(stage_units) * 2 * unit_bytes<T, D>();
}
template <typename T, int D, int G>
__host__ __device__ inline size_t smem_bytes(int64_t share_cap, int stage_units, int nc) {
  return shared_bytes<D, G>() + stage_bytes<T, D, G>(stage_units) + size_t(nc) * G * D * 4 +
         ((size_t(share_cap) * 5 + 15) & ~size_t(15));
}
// the stage holds the warps' partial outputs once the attention is done
static_assert(kMinStageUnits * 2 * kGroup * 2 >= kWarps * 8 * 4, "stage too small for wo");

// grid (nc, n_kv_heads, batch) in clusters of (nc, 1, 1)
template <typename T, int D, int G>
__global__ void __launch_bounds__(kThreads, G <= 4 ? 2 : 1)
    decode_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                  int64_t ctx_cap, const int64_t* __restrict__ pos,
                  const float* __restrict__ bsum, const float* __restrict__ gsum,
                  int n_kv_heads, int topk_blocks, int topk_groups, float scale_log2,
                  int64_t share_cap, int stage_units, int32_t* __restrict__ sel_blk,
                  int32_t* __restrict__ sel_grp, T* __restrict__ o, float* __restrict__ lse) {
  pdl_launch_dependents();
  cg::cluster_group cluster = cg::this_cluster();
  const int rank = int(cluster.block_rank());
  const int nc = int(cluster.num_blocks());
  extern __shared__ __align__(128) unsigned char sm_raw[];
  Shared<D, G>& sh = *reinterpret_cast<Shared<D, G>*>(sm_raw);
  T* stage = reinterpret_cast<T*>(sm_raw + shared_bytes<D, G>());
  float* wo = reinterpret_cast<float*>(stage);  // [kWarps][G][D], after the attention
  float* po = reinterpret_cast<float*>(sm_raw + shared_bytes<D, G>() +
                                       stage_bytes<T, D, G>(stage_units));  // [nc][G][D]
  uint32_t* key1 = reinterpret_cast<uint32_t*>(po + size_t(nc) * G * D);
  uint8_t* sel1 = reinterpret_cast<uint8_t*>(key1 + share_cap);
  const int h = blockIdx.y, b = blockIdx.z;
  const int n_q_heads = n_kv_heads * G;
  const int64_t head = int64_t(b) * n_kv_heads + h;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  constexpr uint32_t kUnit = unit_bytes<T, D>();
  constexpr size_t kUnitElems = kUnit / sizeof(T);
  if (tid == 0) {
    sm100::mbar_init(&sh.bar_own, 1);
    sm100::mbar_init(&sh.bar_rt, 1);
    sh.abort = 0;
    sm100::fence_barrier_init();
  }
  pdl_wait();

  // the G query rows (their loads in flight while the position is read)
  const T* qsrc = q + (int64_t(b) * n_q_heads + int64_t(h) * G) * D;
  constexpr int kQPer = (G * D + kThreads - 1) / kThreads;
  float qv[kQPer];
#pragma unroll
  for (int u = 0; u < kQPer; ++u) {
    const int i = tid + u * kThreads;
    qv[u] = i < G * D ? to_float(qsrc[i]) : 0.f;
  }
  const int64_t p = pos[b];
  if (p < 0 || p >= ctx_cap) {
    // every CTA of the cluster reads the same position and leaves here
    if (rank == 0 && tid == 0) latch_status(HGA_ERR_DEVICE_CHECK);
    return;
  }
  const int64_t J = p / kBlock;  // own block; candidates [0, J)
  const int64_t own0 = J * kBlock;
  const int n_own = int((p - own0) / kGroup) + 1;  // own-block units (the last one partial)
  const T* kh = k + head * ctx_cap * D;
  const T* vh = v + head * ctx_cap * D;
  // barriers initialised, and every CTA of the cluster running before any
  // touches a peer's shared memory
  cluster.sync();

  // 0. this CTA's own-block units (u = rank + s*nc < n_own) start loading;
  //    they are the first slots, all inside the first round
  const int own_mine = n_own > rank ? (n_own - rank + nc - 1) / nc : 0;
  if (tid == 0 && own_mine > 0) {
    sm100::mbar_arrive_expect_tx(&sh.bar_own, uint32_t(own_mine) * 2 * kUnit);
    for (int s = 0; s < own_mine; ++s) {
      const int64_t row = own0 + int64_t(rank + s * nc) * kGroup;
      T* dst = stage + size_t(s) * 2 * kUnitElems;
      sm100::bulk_load(dst, kh + row * D, kUnit, &sh.bar_own);
      sm100::bulk_load(dst + kUnitElems, vh + row * D, kUnit, &sh.bar_own);
    }
  }

  // the query rows and their mean (added in head order)
#pragma unroll
  for (int u = 0; u < kQPer; ++u) {
    const int i = tid + u * kThreads;
    if (i < G * D) sh.qh[i / D][i % D] = qv[u];
  }
  __syncthreads();
  for (int e = tid; e < D; e += kThreads) {
    float s = 0.f;
#pragma unroll
    for (int g = 0; g < G; ++g) s += sh.qh[g][e];
    sh.qb[e] = s * (1.f / float(G));
  }
  __syncthreads();

  // 1. level-1 scores of this CTA's share of the candidates, local top-k_b,
  //    stored into every CTA's finalist slots (padding key 0 ranks below
  //    every finite score)
  const int kb = int(J < topk_blocks ? J : topk_blocks);
  const int64_t share = (J + nc - 1) / nc;
  const int64_t lo = J < rank * share ? J : rank * share;
  const int n_loc = int((J < lo + share ? J : lo + share) - lo);
  auto block_row = [](int i) { return int64_t(i); };
  score_rows<D, decltype(block_row), kScoreRows>(bsum + (head * (ctx_cap / kBlock) + lo) * D,
                                                 sh.qb, n_loc, block_row, key1);
  __syncthreads();
  const int k_loc = kb < n_loc ? kb : n_loc;
  block_topk_indices(key1, n_loc, k_loc, sh.fin_idx, sel1, sh.hist, sh.scratch);
  for (int r = tid; r < k_loc; r += kThreads) {
    sh.fin_key[r] = key1[sh.fin_idx[r]];
    sh.fin_idx[r] += int(lo);
  }
  __syncthreads();
  for (int i = tid; i < nc * kb; i += kThreads) {
    const int dst = i / kb, j = i % kb;
    Shared<D, G>* peer = cluster.map_shared_rank(&sh, dst);
    peer->mkey[rank * kb + j] = j < k_loc ? sh.fin_key[j] : 0u;
    peer->midx[rank * kb + j] = j < k_loc ? sh.fin_idx[j] : -1;
  }
  cluster.sync();

  // every CTA: the global top-k_b (ascending block index)
  const int n_m = nc * kb;
  block_topk_indices(sh.mkey, n_m, kb, sh.blocks, sh.msel, sh.hist, sh.scratch);
  for (int r = tid; r < kb; r += kThreads) sh.blocks[r] = sh.midx[sh.blocks[r]];
  __syncthreads();
  if (rank == 0 && sel_blk)
    for (int i = tid; i < topk_blocks; i += kThreads)
      sel_blk[head * topk_blocks + i] = i < kb ? sh.blocks[i] : -1;

  // 2. level 2: this CTA scores its share of the 8 k_b groups (candidate
  //    p -> group blocks[p/8]*8 + p%8, ascending in p) and stores the scores
  //    into every CTA
  const int n2 = 8 * kb;
  const int share2 = (n2 + nc - 1) / nc;
  const int lo2 = n2 < rank * share2 ? n2 : rank * share2;
  const int n2_loc = (n2 < lo2 + share2 ? n2 : lo2 + share2) - lo2;
  auto group_row = [&](int i) {
    const int pp = lo2 + i;
    return int64_t(sh.blocks[pp >> 3]) * kGroupsPerBlock + (pp & 7);
  };
  score_rows<D, decltype(group_row), kScoreRows>(gsum + head * (ctx_cap / kGroup) * D, sh.qb,
                                                 n2_loc, group_row, sh.key2 + lo2);
  __syncthreads();
  if (nc > 1)
    for (int i = tid; i < (nc - 1) * n2_loc; i += kThreads) {
      const int dst = (rank + 1 + i / n2_loc) % nc, j = i % n2_loc;
      cluster.map_shared_rank(sh.key2, dst)[lo2 + j] = sh.key2[lo2 + j];
    }
  cluster.sync();
  const int kg = topk_groups < n2 ? topk_groups : n2;
  block_topk_indices(sh.key2, n2, kg, sh.grp, sh.sel2, sh.hist, sh.scratch);
  for (int r = tid; r < kg; r += kThreads)
    sh.grp[r] = sh.blocks[sh.grp[r] >> 3] * kGroupsPerBlock + (sh.grp[r] & 7);
  __syncthreads();
  if (rank == 0 && sel_grp)
    for (int i = tid; i < topk_groups; i += kThreads)
      sel_grp[head * topk_groups + i] = i < kg ? sh.grp[i] : -1;

  // 3. attention.  Units u = rank + s*nc (slot s of this CTA): own-block
  //    units first (u < n_own), then the selected groups (u - n_own).  A
  //    round holds stage_units slots; a CTA with more units runs more rounds.
  constexpr int kChunks = D / 64;  // 8-element chunks per lane: c*64 + ec*8 ..
  const int ts = lane >> 3, ec = lane & 7;
  const int n_units = n_own + kg;
  const int mine = n_units > rank ? (n_units - rank + nc - 1) / nc : 0;
  float m[G], l[G], acc[G][kChunks][8];
#pragma unroll
  for (int g = 0; g < G; ++g) {
    m[g] = -INFINITY;
    l[g] = 0.f;
#pragma unroll
    for (int c = 0; c < kChunks; ++c)
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[g][c][i] = 0.f;
  }
  uint32_t rt_phase = 0;
  bool ok = true;
  for (int s0 = 0; s0 < mine; s0 += stage_units) {
    const int n_slots = mine - s0 < stage_units ? mine - s0 : stage_units;
    // routed units of this round start after the own-block ones
    const int rt_first = s0 == 0 ? own_mine : 0;
    const int n_rt = n_slots > rt_first ? n_slots - rt_first : 0;
    if (s0 > 0) {
      __syncthreads();  // every warp is done with the previous round's rows
      if (tid == 0) sm100::fence_proxy_async_smem();
    }
    if (tid == 0 && n_rt > 0) {
      sm100::mbar_arrive_expect_tx(&sh.bar_rt, uint32_t(n_rt) * 2 * kUnit);
      for (int s = rt_first; s < n_slots; ++s) {
        const int64_t row = int64_t(sh.grp[rank + (s0 + s) * nc - n_own]) * kGroup;
        T* dst = stage + size_t(s) * 2 * kUnitElems;
        sm100::bulk_load(dst, kh + row * D, kUnit, &sh.bar_rt);
        sm100::bulk_load(dst + kUnitElems, vh + row * D, kUnit, &sh.bar_rt);
      }
    }
    bool fail = false;
    if (s0 == 0 && own_mine > 0) fail = !sm100::mbar_wait(&sh.bar_own, 0, &sh.abort);
    if (n_rt > 0) {
      fail = !sm100::mbar_wait(&sh.bar_rt, rt_phase, &sh.abort) || fail;
      rt_phase ^= 1u;
    }
    // one decision for the whole CTA, so that every thread takes the same
    // barriers afterwards
    if (__syncthreads_or(fail)) {
      ok = false;
      break;
    }
    // 4-token quads of this round's slots, dealt out to the warps
    const float* qp = &sh.qh[0][0];
    for (int qi = warp; qi < 2 * n_slots; qi += kWarps) {
      // the query values are re-read from shared memory in every quad rather
      // than held in registers next to the accumulators
      asm volatile("" : "+l"(qp));
      const int s = qi >> 1, tok = (qi & 1) * 4 + ts;
      const int u = rank + (s0 + s) * nc;
      int n_valid = kGroup;
      if (u < n_own) {
        const int64_t left = p - (own0 + int64_t(u) * kGroup) + 1;
        n_valid = left < kGroup ? int(left) : kGroup;
      }
      const bool valid = tok < n_valid;
      const T* krow = stage + size_t(s) * 2 * kUnitElems + size_t(tok) * D;
      const T* vrow = krow + kUnitElems;
      // scores of the G heads, then (K no longer needed) the V row
      float sl[G];
      {
        float kf[kChunks][8];
#pragma unroll
        for (int c = 0; c < kChunks; ++c) load8(krow + c * 64 + ec * 8, kf[c]);
#pragma unroll
        for (int g = 0; g < G; ++g) {
          float sc = 0.f;
#pragma unroll
          for (int c = 0; c < kChunks; ++c)
#pragma unroll
            for (int i = 0; i < 8; ++i) sc = fmaf(kf[c][i], qp[g * D + c * 64 + ec * 8 + i], sc);
          sc += __shfl_xor_sync(0xffffffffu, sc, 1);
          sc += __shfl_xor_sync(0xffffffffu, sc, 2);
          sc += __shfl_xor_sync(0xffffffffu, sc, 4);
          sl[g] = valid ? sc * scale_log2 : -INFINITY;
        }
      }
      float vf[kChunks][8];
#pragma unroll
      for (int c = 0; c < kChunks; ++c) load8(vrow + c * 64 + ec * 8, vf[c]);
#pragma unroll
      for (int g = 0; g < G; ++g) {
        float tmax = fmaxf(sl[g], __shfl_xor_sync(0xffffffffu, sl[g], 8));
        tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 16));
        const float m_new = fmaxf(m[g], tmax);
        if (m_new == -INFINITY) continue;  // warp-uniform: nothing valid yet
        const float alpha = sm100::ex2_approx(m[g] - m_new);
        const float pe = valid ? sm100::ex2_approx(sl[g] - m_new) : 0.f;
        float ps = pe + __shfl_xor_sync(0xffffffffu, pe, 8);
        ps += __shfl_xor_sync(0xffffffffu, ps, 16);
        l[g] = l[g] * alpha + ps;
#pragma unroll
        for (int c = 0; c < kChunks; ++c)
#pragma unroll
          for (int i = 0; i < 8; ++i) acc[g][c][i] = fmaf(pe, vf[c][i], acc[g][c][i] * alpha);
        m[g] = m_new;
      }
    }
  }
  if (!ok && tid == 0) {
    // a copy did not land in time (HGA_ERR_TIMEOUT is latched): give the
    // copies in flight a bounded time to land before the CTA leaves; this
    // sequence's outputs are not written
    if (own_mine > 0) sm100::mbar_wait(&sh.bar_own, 0, &sh.abort, 200000000LL);
    if (rt_phase == 0 && mine > own_mine)
      sm100::mbar_wait(&sh.bar_rt, 0, &sh.abort, 200000000LL);
  }

  // 4. the four token slots of each element chunk, then the warps, then the CTAs
#pragma unroll
  for (int g = 0; g < G; ++g)
#pragma unroll
    for (int c = 0; c < kChunks; ++c)
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        acc[g][c][i] += __shfl_xor_sync(0xffffffffu, acc[g][c][i], 8);
        acc[g][c][i] += __shfl_xor_sync(0xffffffffu, acc[g][c][i], 16);
      }
  __syncthreads();  // every warp is done reading the stage
  if (ts == 0)
#pragma unroll
    for (int g = 0; g < G; ++g)
#pragma unroll
      for (int c = 0; c < kChunks; ++c)
#pragma unroll
        for (int i = 0; i < 8; ++i) wo[(warp * G + g) * D + c * 64 + ec * 8 + i] = acc[g][c][i];
  if (lane == 0)
#pragma unroll
    for (int g = 0; g < G; ++g) {
      sh.wm[warp][g] = m[g];
      sh.wl[warp][g] = l[g];
    }
  __syncthreads();
  Shared<D, G>* root = cluster.map_shared_rank(&sh, 0);
  float* root_po = cluster.map_shared_rank(po, 0);
  for (int i = tid; i < G * D; i += kThreads) {
    const int g = i / D, e = i % D;
    float M = -INFINITY;
    for (int w = 0; w < kWarps; ++w) M = fmaxf(M, sh.wm[w][g]);
    float L = 0.f, O = 0.f;
    if (M != -INFINITY)
      for (int w = 0; w < kWarps; ++w) {
        const float a = exp2f(sh.wm[w][g] - M);
        L = fmaf(a, sh.wl[w][g], L);
        O = fmaf(a, wo[(w * G + g) * D + e], O);
      }
    root_po[(rank * G + g) * D + e] = O;
    if (e == 0) {
      root->pm[rank][g] = M;
      root->pl[rank][g] = L;
    }
  }
  // also publishes `ok` of every CTA through the abort flags below
  if (!ok && tid == 0) root->abort = 1;
  cluster.sync();

  // rank 0 merges the CTAs' partials in rank order and writes O and LSE
  if (rank == 0 && !sh.abort) {
    for (int i = tid; i < G * D; i += kThreads) {
      const int g = i / D, e = i % D;
      float M = -INFINITY;
      for (int r = 0; r < nc; ++r) M = fmaxf(M, sh.pm[r][g]);
      float L = 0.f, O = 0.f;
      for (int r = 0; r < nc; ++r) {
        const float a = exp2f(sh.pm[r][g] - M);  // the own token makes M finite
        L = fmaf(a, sh.pl[r][g], L);
        O = fmaf(a, po[(r * G + g) * D + e], O);
      }
      const int64_t row = int64_t(b) * n_q_heads + int64_t(h) * G + g;
      o[row * D + e] = from_float<T>(O / L);
      if (e == 0) lse[row] = (M + log2f(L)) * 0.6931471805599453f;
    }
  }
}

}  // namespace dec
}  // namespace hga
