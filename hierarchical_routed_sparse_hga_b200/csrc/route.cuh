// Steps a2 + a3: two-level weight-free routing ("BMW如何通过重新设计注意力机制…",
// section "HGA的不同之处": queries score the block summaries, the top-k blocks
// are opened at 8-token-group level, the router uses no learned weights and
// scores the existing projected keys).
//
// One launch (route_fused_kernel) while the candidate blocks number at most
// kFusedRouteMaxBlocks; beyond that three launches, all HBM/L2-bound:
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

#include "hga_common.cuh"

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

// The whole routing of one (b, h, j) in one CTA, used while every CTA can
// afford to read all J block summaries (J <= kFusedRouteMaxBlocks; they stay
// in L2): q-bar from the G heads' 64 query rows (the loads of several rows in
// flight per thread), the J block scores, then select_levels.  One launch
// instead of qmean + block_score + select.  Dynamic shared memory:
// fused_route_smem(), the select layout followed by the q-bar partial sums.
constexpr int kFusedRouteMaxBlocks = 512;

template <int D>
__host__ __device__ constexpr int fused_route_rows() { return kRouteThreads / (D / 8); }

template <int D>
__host__ __device__ inline size_t fused_route_smem(int64_t j_cap, int topk_blocks) {
  return select_layout(j_cap, topk_blocks, D).total + size_t(fused_route_rows<D>()) * D * 4;
}

// Mean of the G x 64 query rows of query block j of KV head h (rows of the
// segment's Q [B, Hq, S, d]): thread (row slot rs, 8-column chunk ch) sums
// rows rs, rs + RS, ... (several rows' loads in flight), the RS partial rows
// are then added in order; out[e] = mean (shared or global memory).  All
// kRouteThreads threads; `part` is RS x D floats of shared memory.
template <typename T, int D>
__device__ __forceinline__ void block_query_mean(const T* __restrict__ q, int b, int h, int j,
                                                 int n_q_heads, int G, int s_len, float* part,
                                                 float* out) {
  constexpr int CH = D / 8, RS = fused_route_rows<D>();
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
  __shared__ float part[fused_route_rows<D>() * D];
  const int j = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int64_t head = int64_t(b) * n_kv_heads + h;
  block_query_mean<T, D>(q, b, h, j, n_q_heads, n_q_heads / n_kv_heads, s_len, part,
                         qsum + (head * (ctx_cap / kBlock) + own0 + j) * D);
}

// grid (n_qb, Hkv, B)
template <typename T, int D>
__global__ void __launch_bounds__(kRouteThreads)
    route_fused_kernel(const T* __restrict__ q, const float* __restrict__ bsum,
                       const float* __restrict__ gsum, int64_t ctx_cap, int n_q_heads,
                       int n_kv_heads, int s_len, int64_t own0, int topk_blocks, int topk_groups,
                       int32_t* __restrict__ sel_blk, int32_t* __restrict__ sel_grp,
                       int* __restrict__ done, uint32_t token, const float* __restrict__ qprev,
                       int qshift) {
  // q-bar needs only the queries, which the kernels before this one do not
  // write: it is formed while the kernel before still runs; the summaries
  // are read only after it has completed (the wait below).  A chained
  // forward waits for each item's flag, so it may be scheduled at once.
  pdl_launch_dependents();
  extern __shared__ __align__(16) unsigned char sm_raw[];
  const int j = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int G = n_q_heads / n_kv_heads, n_qb = s_len / kQBlock;
  const int64_t head = int64_t(b) * n_kv_heads + h;
  const int64_t J = own0 + j;                 // candidate blocks [0, J)
  const SelectLayout L = select_layout(own0 + n_qb, topk_blocks, D);
  float* qb = reinterpret_cast<float*>(sm_raw + L.qb);
  uint32_t* key1 = reinterpret_cast<uint32_t*>(sm_raw + L.key1);
  float* part = reinterpret_cast<float*>(sm_raw + L.total);

  if (!qprev) block_query_mean<T, D>(q, b, h, j, n_q_heads, G, s_len, part, qb);
  // from here on everything before this kernel has completed
  pdl_wait();
  if (qprev)
    for (int e = threadIdx.x; e < D; e += kRouteThreads)
      qb[e] = J - qshift >= 0 ? qprev[(head * (ctx_cap / kBlock) + J - qshift) * D + e] : 0.f;
  __syncthreads();
  // level-1 scores of the J candidate blocks
  score_rows<D>(bsum + head * (ctx_cap / kBlock) * D, qb, int(J),
                [](int p) { return int64_t(p); }, key1);
  __syncthreads();
  select_levels<D>(L, sm_raw, gsum, head, ctx_cap, n_qb, j, J, topk_blocks, topk_groups, sel_blk,
                   sel_grp);
  if (done) {
    // chained segment call: this item's selections are written
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0)
      flag_release(done + blockIdx.x + gridDim.x * (blockIdx.y + gridDim.y * blockIdx.z), token);
  }
}

}  // namespace hga
