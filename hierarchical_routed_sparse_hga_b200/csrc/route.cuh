// Steps a2 + a3: two-level weight-free routing ("BMW如何通过重新设计注意力机制…",
// section "HGA的不同之处": queries score the block summaries, the top-k blocks
// are opened at 8-token-group level, the router uses no learned weights and
// scores the existing projected keys).
//
// One launch (route_cluster_kernel, below) while the candidate blocks number
// at most kClusterMax * kClusterShareRows (2048: contexts up to 131072
// tokens); beyond that three launches, all HBM/L2-bound:
//   qmean_kernel        per (query block j, query head): that head's share of
//                       qbar[b,h,j], the mean of the 64 x G query rows (reads Q
//                       once, 1024 CTAs for Qwen3 shapes, one load round);
//   block_score_kernel  S[b,h,j,c] = qbar[b,h,j] . bsum[b,h,c] on tiles of 32
//                       candidate blocks x 8 query blocks;
//   select_kernel       per (b,h,j): radix top-k over the J candidate scores,
//                       gather the selected blocks' 8*kb group summaries,
//                       score them, radix top-k again, write both selections in
//                       ascending index order.
// Scores are not multiplied by 1/sqrt(d): a positive factor does not change
// the ranking.
#pragma once

#include <cooperative_groups.h>

#include "hga_common.cuh"
#include "sm100_ptx.cuh"

namespace hga {

constexpr int kRouteThreads = 256;
constexpr int kScoreChunk = 16;  // candidate blocks per block_score CTA

// grid (n_qb * G, Hkv, B), 128 threads: the 64 rows of one query head of one
// query block (16 KB), all loads issued in one round; writes that head's
// share of the mean, qpart[b, h, j, g, :] = sum of its rows / (64 G).  The
// consumers add the G shares in a fixed order (deterministic).
constexpr int kQmeanThreads = 128;

template <typename T, int D>
__global__ void __launch_bounds__(kQmeanThreads)
    qmean_kernel(const T* __restrict__ q, int n_q_heads, int n_kv_heads, int s_len,
                 float* __restrict__ qpart) {
  pdl_launch_dependents();
  pdl_wait();
  constexpr int CH = D / 8;                    // 16-byte chunks per row
  constexpr int RS = kQmeanThreads / CH;       // row slots
  constexpr int PASSES = kQBlock / RS;
  __shared__ float part[RS][D];
  const int G = n_q_heads / n_kv_heads;
  const int j = blockIdx.x / G, g = blockIdx.x % G, h = blockIdx.y, b = blockIdx.z;
  const int hq = h * G + g;
  const int ch = threadIdx.x % CH, rs = threadIdx.x / CH;
  const T* src = q + ((int64_t(b) * n_q_heads + hq) * s_len + int64_t(j) * kQBlock) * D + ch * 8;
  float f[PASSES][8];
#pragma unroll
  for (int u = 0; u < PASSES; ++u) load8(src + int64_t(rs + u * RS) * D, f[u]);
  float acc[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[e] = 0.f;
#pragma unroll
  for (int u = 0; u < PASSES; ++u)
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] += f[u][e];
#pragma unroll
  for (int e = 0; e < 8; ++e) part[rs][ch * 8 + e] = acc[e];
  __syncthreads();
  const int n_qb = s_len / kQBlock;
  const float inv = 1.f / float(G * kQBlock);
  for (int e = threadIdx.x; e < D; e += kQmeanThreads) {
    float sum = 0.f;
#pragma unroll
    for (int r = 0; r < RS; ++r) sum += part[r][e];
    qpart[(((int64_t(b) * n_kv_heads + h) * n_qb + j) * G + g) * D + e] = sum * inv;
  }
}

// qbar of (b, h, j) = sum over the G shares (G <= 8), added in order
// g = 0 .. G-1; all G loads are issued before the adds
__device__ __forceinline__ float qbar_elem(const float* qpart_bhj, int G, int D, int e) {
  float x[8];
#pragma unroll
  for (int g = 0; g < 8; ++g) x[g] = g < G ? qpart_bhj[g * D + e] : 0.f;
  float v = x[0];
#pragma unroll
  for (int g = 1; g < 8; ++g)
    if (g < G) v += x[g];
  return v;
}

// q-bar of query block j (global block J = own0 + j) as the routing uses it:
// the sum of its G shares; or, from the resident block mean queries qsum
// (qsum != nullptr), row J - qshift: the block's own mean (qshift 0) or, for
// causal routing, the block before it (qshift 1; zero for the first block of
// a sequence, which has no candidates).
__device__ __forceinline__ float route_qbar(const float* qpart, const float* qsum, int qshift,
                                            int64_t head, int n_qb, int G, int D, int j, int e,
                                            int64_t own0, int64_t ctx_blocks) {
  if (qsum) {
    const int64_t row = own0 + j - qshift;
    return row >= 0 ? qsum[(head * ctx_blocks + row) * D + e] : 0.f;
  }
  return qbar_elem(qpart + ((head * n_qb + j) * G) * D, G, D, e);
}

// grid (ceil(j_max / 32) * ceil(n_qb / 8), Hkv, B), 256 threads: a tile of
// 32 candidate blocks x 8 query blocks, one score per thread, operands
// staged in shared memory (candidates transposed and padded: conflict-free).
constexpr int kScoreCands = 32;
constexpr int kScoreQbs = 8;

template <int D>
__global__ void __launch_bounds__(kRouteThreads)
    block_score_kernel(const float* __restrict__ qpart, const float* __restrict__ qprev,
                       int qshift, const float* __restrict__ bsum, int64_t ctx_cap, int n_kv_heads, int G,
                       int n_qb, int64_t own0, float* __restrict__ scores, int64_t jstride) {
  pdl_launch_dependents();
  pdl_wait();
  __shared__ float qb[kScoreQbs][D];
  __shared__ float bsT[D][kScoreCands + 1];
  const int h = blockIdx.y, b = blockIdx.z;
  const int n_jc = (n_qb + kScoreQbs - 1) / kScoreQbs;
  const int cc = blockIdx.x / n_jc, jc = blockIdx.x % n_jc;
  const int64_t head = int64_t(b) * n_kv_heads + h;
  const int64_t c0 = int64_t(cc) * kScoreCands;
  const int j0 = jc * kScoreQbs;
  const int64_t j_max = own0 + n_qb - 1;
  constexpr int kQ = kScoreQbs * D / kRouteThreads;     // elements per thread
  constexpr int kB = kScoreCands * D / kRouteThreads;
  const float* bsrc = bsum + head * (ctx_cap / kBlock) * D;
  float qv[kQ], bv[kB];
#pragma unroll
  for (int u = 0; u < kQ; ++u) {
    const int i = threadIdx.x + u * kRouteThreads, jl = i / D, e = i % D, j = j0 + jl;
    qv[u] = j < n_qb ? route_qbar(qpart, qprev, qshift, head, n_qb, G, D, j, e, own0,
                                      ctx_cap / kBlock)
                     : 0.f;
  }
#pragma unroll
  for (int u = 0; u < kB; ++u) {
    const int i = threadIdx.x + u * kRouteThreads, cl = i / D, e = i % D;
    const int64_t c = c0 + cl;
    bv[u] = c < j_max ? bsrc[c * D + e] : 0.f;
  }
#pragma unroll
  for (int u = 0; u < kQ; ++u) {
    const int i = threadIdx.x + u * kRouteThreads;
    qb[i / D][i % D] = qv[u];
  }
#pragma unroll
  for (int u = 0; u < kB; ++u) {
    const int i = threadIdx.x + u * kRouteThreads;
    bsT[i % D][i / D] = bv[u];
  }
  __syncthreads();
  const int cl = threadIdx.x % kScoreCands, jl = threadIdx.x / kScoreCands;
  const int64_t c = c0 + cl;
  const int j = j0 + jl;
  float acc = 0.f;
#pragma unroll 16
  for (int e = 0; e < D; ++e) acc = fmaf(qb[jl][e], bsT[e][cl], acc);
  if (j < n_qb && c < own0 + j) scores[(head * n_qb + j) * jstride + c] = acc;
}

// Shared-memory layout of select_kernel (16-byte aligned sections).
struct SelectLayout {
  size_t qb, key1, key2, blocks, hist, scratch, sel1, sel2, total;
};

__host__ __device__ inline size_t align16(size_t x) { return (x + 15) & ~size_t(15); }

__host__ __device__ inline SelectLayout select_layout(int64_t j_cap, int topk_blocks, int D) {
  SelectLayout L;
  size_t o = 0;
  L.qb = o;      o = align16(o + size_t(D) * 4);
  L.key1 = o;    o = align16(o + size_t(j_cap) * 4);
  L.key2 = o;    o = align16(o + size_t(8) * topk_blocks * 4);
  L.blocks = o;  o = align16(o + size_t(topk_blocks) * 4);
  L.hist = o;    o = align16(o + 256 * 4);
  L.scratch = o; o = align16(o + 16 * 4);
  L.sel1 = o;    o = align16(o + size_t(j_cap));
  L.sel2 = o;    o = align16(o + size_t(8) * topk_blocks);
  L.total = o;
  return L;
}

// Scores n rows of a summary table against q-bar (in shared memory): key[p]
// = ordered_key(qb . rows[row_of(p)]).  A warp takes kU rows per pass, lanes
// across the d dimension, all kU row loads issued before any use.
template <int D, typename RowOf, int kU = 16>
__device__ __forceinline__ void score_rows(const float* __restrict__ table, const float* qb,
                                           int n, RowOf row_of, uint32_t* key) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  constexpr int NW = kRouteThreads / 32;
  constexpr int V4 = D / 4;  // float4 per summary row
  const float4* qb4 = reinterpret_cast<const float4*>(qb);
  static_assert(kU <= 32, "one score per lane");
  constexpr int kE = (V4 + 31) / 32;  // float4 per lane per row
  for (int p0 = warp * kU; p0 < n; p0 += NW * kU) {
    float4 x[kU][kE];
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const int p = p0 + u;
      const int64_t r = p < n ? row_of(p) : 0;
      const float4* row = reinterpret_cast<const float4*>(table + r * D);
#pragma unroll
      for (int i = 0; i < kE; ++i) {
        const int e = lane + 32 * i;
        x[u][i] = (p < n && e < V4) ? row[e] : make_float4(0.f, 0.f, 0.f, 0.f);
      }
    }
    float part[kU];
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      part[u] = 0.f;
#pragma unroll
      for (int i = 0; i < kE; ++i) {
        const int e = lane + 32 * i;
        if (e < V4) {
          const float4 y = qb4[e];
          part[u] = fmaf(x[u][i].x, y.x, part[u]);
          part[u] = fmaf(x[u][i].y, y.y, part[u]);
          part[u] = fmaf(x[u][i].z, y.z, part[u]);
          part[u] = fmaf(x[u][i].w, y.w, part[u]);
        }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) part[u] += __shfl_xor_sync(0xffffffffu, part[u], o);
    }
    if (lane < kU && p0 + lane < n) {
      float v = part[0];
#pragma unroll
      for (int u = 1; u < kU; ++u)
        if (lane == u) v = part[u];
      key[p0 + lane] = ordered_key(v);
    }
  }
}

// The two selections of one (b, h, j) once q-bar is in qb and the J block
// scores are in key1: top-k_b blocks, their 8 groups scored, top-k_g groups,
// both written in ascending index order (-1 padded).
template <int D>
__device__ __forceinline__ void select_levels(const SelectLayout& L, unsigned char* sm_raw,
                                              const float* __restrict__ gsum, int64_t head,
                                              int64_t ctx_cap, int n_qb, int j, int64_t J,
                                              int topk_blocks, int topk_groups,
                                              int32_t* __restrict__ sel_blk,
                                              int32_t* __restrict__ sel_grp) {
  const float* qb = reinterpret_cast<const float*>(sm_raw + L.qb);
  uint32_t* key1 = reinterpret_cast<uint32_t*>(sm_raw + L.key1);
  uint32_t* key2 = reinterpret_cast<uint32_t*>(sm_raw + L.key2);
  int* blocks = reinterpret_cast<int*>(sm_raw + L.blocks);
  int* hist = reinterpret_cast<int*>(sm_raw + L.hist);
  int* scratch = reinterpret_cast<int*>(sm_raw + L.scratch);
  uint8_t* sel1 = sm_raw + L.sel1;
  uint8_t* sel2 = sm_raw + L.sel2;
  const int kb = int(J < topk_blocks ? J : topk_blocks);
  const int n2 = 8 * kb;

  // level 1
  block_topk(key1, int(J), kb, sel1, hist, scratch);
  block_enumerate_any(
      int(J), [&](int i) { return sel1[i] != 0; }, [&](int i, int r) { blocks[r] = i; },
      scratch);
  int32_t* out_blk = sel_blk ? sel_blk + (head * n_qb + j) * topk_blocks : nullptr;
  if (out_blk)
    for (int i = threadIdx.x; i < topk_blocks; i += kRouteThreads)
      out_blk[i] = i < kb ? blocks[i] : -1;

  // level 2: score the 8 groups of every kept block (candidate p -> group
  // blocks[p/8]*8 + p%8, which is ascending in p)
  const float* gbase = gsum + head * (ctx_cap / kGroup) * D;
  score_rows<D>(gbase, qb, n2,
                [&](int p) { return int64_t(blocks[p >> 3]) * kGroupsPerBlock + (p & 7); },
                key2);
  __syncthreads();
  const int kg = n2 < topk_groups ? n2 : topk_groups;
  block_topk(key2, n2, kg, sel2, hist, scratch);
  int32_t* out_grp = sel_grp + (head * n_qb + j) * topk_groups;
  block_enumerate_any(
      n2, [&](int p) { return sel2[p] != 0; },
      [&](int p, int r) { out_grp[r] = blocks[p >> 3] * kGroupsPerBlock + (p & 7); }, scratch);
  for (int i = kg + threadIdx.x; i < topk_groups; i += kRouteThreads) out_grp[i] = -1;
}

// grid (n_qb, Hkv, B); dynamic smem select_layout(...).total
template <int D>
__global__ void __launch_bounds__(kRouteThreads)
    select_kernel(const float* __restrict__ qpart, const float* __restrict__ qprev, int qshift,
                  const float* __restrict__ scores,
                  const float* __restrict__ gsum, int64_t ctx_cap, int n_kv_heads, int G, int n_qb,
                  int64_t own0, int64_t jstride, int topk_blocks, int topk_groups,
                  int32_t* __restrict__ sel_blk, int32_t* __restrict__ sel_grp) {
  pdl_launch_dependents();
  pdl_wait();
  extern __shared__ __align__(16) unsigned char sm_raw[];
  const int j = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int64_t head = int64_t(b) * n_kv_heads + h;
  const int64_t J = own0 + j;                 // candidate blocks [0, J)
  const int64_t j_cap = own0 + n_qb;
  const SelectLayout L = select_layout(j_cap, topk_blocks, D);
  float* qb = reinterpret_cast<float*>(sm_raw + L.qb);
  uint32_t* key1 = reinterpret_cast<uint32_t*>(sm_raw + L.key1);
  const float* srow = scores + (head * n_qb + j) * jstride;
  for (int64_t i = threadIdx.x; i < J; i += kRouteThreads) key1[i] = ordered_key(srow[i]);
  for (int i = threadIdx.x; i < D; i += kRouteThreads)
    qb[i] = route_qbar(qpart, qprev, qshift, head, n_qb, G, D, j, i, own0, ctx_cap / kBlock);
  __syncthreads();
  select_levels<D>(L, sm_raw, gsum, head, ctx_cap, n_qb, j, J, topk_blocks, topk_groups, sel_blk,
                   sel_grp);
}

// rows summed per thread slot in block_query_mean
template <int D>
__host__ __device__ constexpr int query_mean_rows() { return kRouteThreads / (D / 8); }

// Mean of the G x 64 query rows of query block j of KV head h (rows of the
// segment's Q [B, Hq, S, d]): thread (row slot rs, 8-column chunk ch) sums
// rows rs, rs + RS, ... (several rows' loads in flight), the RS partial rows
// are then added in order; out[e] = mean (shared or global memory).  All
// kRouteThreads threads; `part` is RS x D floats of shared memory.
template <typename T, int D>
__device__ __forceinline__ void block_query_mean(const T* __restrict__ q, int b, int h, int j,
                                                 int n_q_heads, int G, int s_len, float* part,
                                                 float* out) {
  constexpr int CH = D / 8, RS = query_mean_rows<D>();
  const int ch = threadIdx.x % CH, rs = threadIdx.x / CH;
  const int rows = G * kQBlock;
  const T* qh =
      q + ((int64_t(b) * n_q_heads + int64_t(h) * G) * s_len + int64_t(j) * kQBlock) * D + ch * 8;
  float acc[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[e] = 0.f;
#pragma unroll 8
  for (int rr = rs; rr < rows; rr += RS) {
    float f[8];
    load8(qh + (int64_t(rr >> 6) * s_len + (rr & 63)) * D, f);
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] += f[e];
  }
#pragma unroll
  for (int e = 0; e < 8; ++e) part[rs * D + ch * 8 + e] = acc[e];
  __syncthreads();
  const float inv = 1.f / float(rows);
  for (int e = threadIdx.x; e < D; e += kRouteThreads) {
    float sum = 0.f;
    for (int r = 0; r < RS; ++r) sum += part[r * D + e];
    out[e] = sum * inv;
  }
}

// Resident mean query of every block of the segment (for causal routing):
// qsum[b, h, q_begin/64 + j, :] = mean of the G x 64 query rows of query
// block j.  grid (n_qb, Hkv, B), kRouteThreads threads.
template <typename T, int D>
__global__ void __launch_bounds__(kRouteThreads)
    qsum_kernel(const T* __restrict__ q, int64_t ctx_cap, int n_q_heads, int n_kv_heads,
                int s_len, int64_t own0, float* __restrict__ qsum) {
  pdl_launch_dependents();
  pdl_wait();
  __shared__ float part[query_mean_rows<D>() * D];
  const int j = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int64_t head = int64_t(b) * n_kv_heads + h;
  block_query_mean<T, D>(q, b, h, j, n_q_heads, n_q_heads / n_kv_heads, s_len, part,
                         qsum + (head * (ctx_cap / kBlock) + own0 + j) * D);
}

// ---------------------------------------------------------------------------
// The whole routing of one (batch, KV head) in one thread-block cluster of C
// CTAs (C in {1, 2, 4, 8, 16}; up to kClusterShareRows candidate blocks per
// CTA).  CTA r holds candidate blocks [r*share, (r+1)*share) and owns query
// blocks j = r, r + C, r + 2C, ...
//   A. bulk copy of its share of the block summaries into shared memory
//      (read once for the whole head); meanwhile q-bar of its own query
//      blocks (from Q, then stored into every CTA) or of all of them (from
//      the resident block mean queries); one cluster barrier;
//   B. the scores of every query block against its share (lane = query
//      block, rows broadcast), a local top-k_b per query block (warp rank
//      counting over the valid candidates), the finalists stored into the
//      owner CTA's slots in rank order (padding key 0); one cluster barrier;
//   C. per owned query block: the top-k_b of the C*k_b finalists (slots in
//      rank order are in ascending block order, so ties keep the lower
//      block), the kept blocks' groups scored and the top-k_g kept; both
//      selections written and, in a chained segment call, the item's flag
//      released.
// ---------------------------------------------------------------------------
constexpr int kClusterMax = 16;
constexpr int kClusterShareRows = 128;

struct ClusterLayout {
  size_t bs, qb, sc, fin_key, fin_idx, mkey, midx, msel, blocks, key2, sel2, grp, hist, scratch,
      part, bar, total;
  int qb_stride, sc_stride;
};

__host__ __device__ inline ClusterLayout cluster_layout(int share, int n_qb, int C,
                                                        int topk_blocks, int D) {
  ClusterLayout L;
  const int own = (n_qb + C - 1) / C;
  L.qb_stride = D + 4;
  L.sc_stride = share + 1;
  size_t o = 0;
  L.bs = o;       o = align16(o + size_t(share) * D * 4);
  L.qb = o;       o = align16(o + size_t(n_qb) * L.qb_stride * 4);
  L.sc = o;       o = align16(o + size_t(n_qb) * L.sc_stride * 4);
  L.fin_key = o;  o = align16(o + size_t(own) * C * topk_blocks * 4);
  L.fin_idx = o;  o = align16(o + size_t(own) * C * topk_blocks * 4);
  L.mkey = o;     o = align16(o + size_t(C) * topk_blocks * 4);
  L.midx = o;     o = align16(o + size_t(C) * topk_blocks * 4);
  L.msel = o;     o = align16(o + size_t(C) * topk_blocks);
  L.blocks = o;   o = align16(o + size_t(topk_blocks) * 4);
  L.key2 = o;     o = align16(o + size_t(8) * topk_blocks * 4);
  L.sel2 = o;     o = align16(o + size_t(8) * topk_blocks);
  L.grp = o;      o = align16(o + size_t(8) * topk_blocks * 4);
  L.hist = o;     o = align16(o + 256 * 4);
  L.scratch = o;  o = align16(o + 16 * 4);
  L.part = o;     o = align16(o + size_t(kRouteThreads / (D / 8)) * D * 4);
  L.bar = o;      o = align16(o + 16);
  L.total = o;
  return L;
}

// grid (C, n_kv_heads, batch) in clusters of (C, 1, 1).  q-bar source: the
// segment's Q (q != nullptr), else qsum row own0 + j - qshift.
template <typename T, int D>
__global__ void __launch_bounds__(kRouteThreads)
    route_cluster_kernel(const T* __restrict__ q, const float* __restrict__ qsum, int qshift,
                         const float* __restrict__ bsum, const float* __restrict__ gsum,
                         int64_t ctx_cap, int n_q_heads, int n_kv_heads, int s_len, int64_t own0,
                         int share, int topk_blocks, int topk_groups,
                         int32_t* __restrict__ sel_blk, int32_t* __restrict__ sel_grp,
                         int* __restrict__ done, uint32_t token) {
  namespace cg = cooperative_groups;
  pdl_launch_dependents();
  cg::cluster_group cluster = cg::this_cluster();
  const int rank = int(cluster.block_rank()), C = int(cluster.num_blocks());
  extern __shared__ __align__(16) unsigned char sm_raw[];
  const int h = blockIdx.y, b = blockIdx.z;
  const int G = n_q_heads / n_kv_heads, n_qb = s_len / kQBlock;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t head = int64_t(b) * n_kv_heads + h;
  const ClusterLayout L = cluster_layout(share, n_qb, C, topk_blocks, D);
  float* bs = reinterpret_cast<float*>(sm_raw + L.bs);
  float* qb = reinterpret_cast<float*>(sm_raw + L.qb);
  uint32_t* sc = reinterpret_cast<uint32_t*>(sm_raw + L.sc);
  uint32_t* fin_key = reinterpret_cast<uint32_t*>(sm_raw + L.fin_key);
  int* fin_idx = reinterpret_cast<int*>(sm_raw + L.fin_idx);
  uint32_t* mkey = reinterpret_cast<uint32_t*>(sm_raw + L.mkey);
  int* midx = reinterpret_cast<int*>(sm_raw + L.midx);
  uint8_t* msel = sm_raw + L.msel;
  int* blocks = reinterpret_cast<int*>(sm_raw + L.blocks);
  uint32_t* key2 = reinterpret_cast<uint32_t*>(sm_raw + L.key2);
  uint8_t* sel2 = sm_raw + L.sel2;
  int* grp = reinterpret_cast<int*>(sm_raw + L.grp);
  int* hist = reinterpret_cast<int*>(sm_raw + L.hist);
  int* scratch = reinterpret_cast<int*>(sm_raw + L.scratch);
  float* part = reinterpret_cast<float*>(sm_raw + L.part);
  uint64_t* bar = reinterpret_cast<uint64_t*>(sm_raw + L.bar);
  __shared__ int s_abort;
  const int64_t j_max = own0 + n_qb - 1;  // candidates of the last query block: [0, j_max)
  const int64_t lo = j_max < int64_t(rank) * share ? j_max : int64_t(rank) * share;
  const int n_loc = int((j_max < lo + share ? j_max : lo + share) - lo);
  if (tid == 0) {
    sm100::mbar_init(bar, 1);
    s_abort = 0;
    sm100::fence_barrier_init();
  }
  // every CTA of the cluster is running before any touches a peer's memory
  cluster.sync();

  // A. q-bar; the block-summary share is copied in after the kernel before
  //    has completed (it may have written the summaries)
  if (q) {
    for (int j = rank; j < n_qb; j += C) {
      block_query_mean<T, D>(q, b, h, j, n_q_heads, G, s_len, part, qb + j * L.qb_stride);
      __syncthreads();
    }
  }
  pdl_wait();
  if (tid == 0 && n_loc > 0) {
    const uint32_t bytes = uint32_t(n_loc) * D * 4;
    sm100::mbar_arrive_expect_tx(bar, bytes);
    const char* src = reinterpret_cast<const char*>(bsum + (head * (ctx_cap / kBlock) + lo) * D);
    for (uint32_t off = 0; off < bytes; off += 32768u)
      sm100::bulk_load(reinterpret_cast<char*>(bs) + off, src + off,
                       bytes - off < 32768u ? bytes - off : 32768u, bar);
  }
  if (q) {
    // own q-bar rows into every peer
    for (int j = rank; j < n_qb; j += C)
      for (int i = tid; i < (C - 1) * D; i += kRouteThreads) {
        const int dst = (rank + 1 + i / D) % C, e = i % D;
        cluster.map_shared_rank(qb, dst)[j * L.qb_stride + e] = qb[j * L.qb_stride + e];
      }
  } else {
    for (int i = tid; i < n_qb * D; i += kRouteThreads) {
      const int j = i / D, e = i % D;
      const int64_t row = own0 + j - qshift;
      qb[j * L.qb_stride + e] = row >= 0 ? qsum[(head * (ctx_cap / kBlock) + row) * D + e] : 0.f;
    }
  }
  bool fail = false;
  if (n_loc > 0) fail = !sm100::mbar_wait(bar, 0, &s_abort);
  const bool ok = !__syncthreads_or(fail);
  cluster.sync();

  // B. scores of every query block against the share: lane = query block
  //    (two rounds past 32), each warp a slice of the rows, 8 rows at a time
  if (ok) {
    const int rows_per_warp = (n_loc + 7) / 8;
    const int r0 = warp * rows_per_warp;
    const int r1 = r0 + rows_per_warp < n_loc ? r0 + rows_per_warp : n_loc;
    for (int jb = 0; jb < n_qb; jb += 32) {
      const int j = jb + lane;
      const float4* qj = reinterpret_cast<const float4*>(qb + (j < n_qb ? j : 0) * L.qb_stride);
      for (int i0 = r0; i0 < r1; i0 += 8) {
        float acc[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) acc[u] = 0.f;
#pragma unroll 4
        for (int e4 = 0; e4 < D / 4; ++e4) {
          const float4 x = qj[e4];
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            const int i = i0 + u < r1 ? i0 + u : i0;
            const float4 y = reinterpret_cast<const float4*>(bs + size_t(i) * D)[e4];
            acc[u] = fmaf(x.x, y.x, fmaf(x.y, y.y, fmaf(x.z, y.z, fmaf(x.w, y.w, acc[u]))));
          }
        }
        if (j < n_qb)
#pragma unroll
          for (int u = 0; u < 8; ++u)
            if (i0 + u < r1) sc[j * L.sc_stride + i0 + u] = ordered_key(acc[u]);
      }
    }
  }
  __syncthreads();
  // local top-k_b of each query block over its valid candidates (c < own0 + j),
  // one warp per query block; finalists in ascending index into the owner
  if (ok) {
    for (int j = warp; j < n_qb; j += kRouteThreads / 32) {
      const int64_t J = own0 + j;
      const int kb = int(J < topk_blocks ? J : topk_blocks);
      int n_val = int(J - lo);
      n_val = n_val < 0 ? 0 : (n_val > n_loc ? n_loc : n_val);
      const int k_loc = kb < n_val ? kb : n_val;
      const uint32_t* row = sc + j * L.sc_stride;
      const int owner = j % C, jl = j / C;
      uint32_t* okey = cluster.map_shared_rank(fin_key, owner) + (jl * C + rank) * topk_blocks;
      int* oidx = cluster.map_shared_rank(fin_idx, owner) + (jl * C + rank) * topk_blocks;
      int written = 0;
      for (int m0 = 0; m0 < n_val; m0 += 32) {
        const int i = m0 + lane;
        bool pick = false;
        if (i < n_val && k_loc > 0) {
          const uint32_t ki = row[i];
          int r = 0;
          for (int i2 = 0; i2 < n_val; ++i2) {
            const uint32_t k2 = row[i2];
            r += (k2 > ki) || (k2 == ki && i2 < i);
          }
          pick = r < k_loc;
        }
        const unsigned ball = __ballot_sync(0xffffffffu, pick);
        if (pick) {
          const int pos = written + __popc(ball & ((1u << lane) - 1u));
          okey[pos] = row[i];
          oidx[pos] = int(lo + i);
        }
        written += __popc(ball);
      }
      for (int p = k_loc + lane; p < kb; p += 32) {
        okey[p] = 0u;
        oidx[p] = -1;
      }
    }
  }
  cluster.sync();

  // C. the owned query blocks: merge, level 2, write
  if (ok) {
    for (int j = rank; j < n_qb; j += C) {
      const int jl = j / C;
      const int64_t J = own0 + j;
      const int kb = int(J < topk_blocks ? J : topk_blocks);
      const int n_m = C * kb;
      for (int i = tid; i < n_m; i += kRouteThreads) {
        const int r = i / kb, p = i % kb;
        mkey[i] = fin_key[(jl * C + r) * topk_blocks + p];
        midx[i] = fin_idx[(jl * C + r) * topk_blocks + p];
      }
      __syncthreads();
      block_topk_indices(mkey, n_m, kb, blocks, msel, hist, scratch);
      for (int r = tid; r < kb; r += kRouteThreads) blocks[r] = midx[blocks[r]];
      __syncthreads();
      if (sel_blk)
        for (int i = tid; i < topk_blocks; i += kRouteThreads)
          sel_blk[(head * n_qb + j) * topk_blocks + i] = i < kb ? blocks[i] : -1;
      const int n2 = 8 * kb;
      score_rows<D>(gsum + head * (ctx_cap / kGroup) * D, qb + j * L.qb_stride, n2,
                    [&](int p) {
                      // a block index below 0 only comes from a non-finite summary;
                      // it is kept in bounds (the attention rejects the result)
                      const int blk = blocks[p >> 3];
                      return int64_t(blk < 0 ? 0 : blk) * kGroupsPerBlock + (p & 7);
                    },
                    key2);
      __syncthreads();
      const int kg = n2 < topk_groups ? n2 : topk_groups;
      block_topk_indices(key2, n2, kg, grp, sel2, hist, scratch);
      int32_t* out = sel_grp + (head * n_qb + j) * topk_groups;
      for (int i = tid; i < topk_groups; i += kRouteThreads)
        out[i] = i < kg ? blocks[grp[i] >> 3] * kGroupsPerBlock + (grp[i] & 7) : -1;
      if (done) {
        // chained segment call: this item's selections are written
        __threadfence();
        __syncthreads();
        if (tid == 0) flag_release(done + j + n_qb * (h + n_kv_heads * b), token);
      }
      __syncthreads();
    }
  } else if (tid == 0) {
    // a copy did not land in time (HGA_ERR_TIMEOUT is latched): give it a
    // bounded time more before the CTA leaves; no selection is written
    sm100::mbar_wait(bar, 0, &s_abort, 200000000LL);
  }
}

}  // namespace hga
