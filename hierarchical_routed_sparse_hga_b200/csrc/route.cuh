// Steps a2 + a3: two-level weight-free routing ("BMW如何通过重新设计注意力机制…",
// section "HGA的不同之处": queries score the block summaries, the top-k blocks
// are opened at 8-token-group level, the router uses no learned weights and
// scores the existing projected keys).
//
// One launch (route_fused_kernel) while the candidate blocks number at most
// kFusedRouteMaxBlocks; beyond that three launches, all HBM/L2-bound:
//   qbar_kernel         per (query block j, KV head): qbar[b,h,j], the mean of
//                       the 64 x G query rows (the block's rows of Q in one
//                       pass by one CTA);
//   block_topk_kernel   per (chunk of kChunkCands candidate blocks, KV head):
//                       the chunk's block summaries and every query block's
//                       q-bar in shared memory, the scores of all query blocks
//                       against the chunk, and per query block the local
//                       top-k_b of its valid candidates (the finalists);
//   select_kernel       per (b,h,j): the top-k_b of the chunks' finalists
//                       (the global top-k_b is a subset of their union),
//                       gather the selected blocks' 8*kb group summaries,
//                       score them, top-k again, write both selections in
//                       ascending index order.
// Scores are not multiplied by 1/sqrt(d): a positive factor does not change
// the ranking.
#pragma once

#include "hga_common.cuh"

namespace hga {

constexpr int kRouteThreads = 256;

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
                                              int32_t* __restrict__ sel_grp, float scale,
                                              float* __restrict__ scores_out) {
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

  float* so = scores_out ? scores_out + (head * n_qb + j) * 4 : nullptr;
  // level 1
  block_topk(key1, int(J), kb, sel1, hist, scratch);
  if (so) kth_scores(key1, sel1, int(J), scale, so);
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
  if (so) kth_scores(key2, sel2, n2, scale, so + 2);
  int32_t* out_grp = sel_grp + (head * n_qb + j) * topk_groups;
  block_enumerate_any(
      n2, [&](int p) { return sel2[p] != 0; },
      [&](int p, int r) { out_grp[r] = blocks[p >> 3] * kGroupsPerBlock + (p & 7); }, scratch);
  for (int i = kg + threadIdx.x; i < topk_groups; i += kRouteThreads) out_grp[i] = -1;
}

// The whole routing of one (b, h, j) in one CTA, used while every CTA can
// afford to read all J block summaries (J <= kFusedRouteMaxBlocks; they stay
// in L2): q-bar from the G heads' 64 query rows (the loads of several rows in
// flight per thread), the J block scores, then select_levels.  One launch
// instead of qbar + block_topk + select.  Dynamic shared memory:
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
// With kWaitBeforeWrite, the grid-dependency wait comes between reading Q
// and writing `out`: Q is read while the kernel before still runs (none of
// the library's kernels that trigger their dependents early writes Q), and
// `out` is written only once that kernel has completed.
template <typename T, int D, bool kWaitBeforeWrite = false>
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
  // rows whose loads are in flight together (raw, 4 or 8 registers each):
  // at d = 128 and G <= 4 every row of the thread in one round
  constexpr int kRound = sizeof(T) == 2 ? 16 : 8;
  for (int rr0 = rs; rr0 < rows; rr0 += kRound * RS) {
    Raw8<T> x[kRound];
#pragma unroll
    for (int u = 0; u < kRound; ++u) {
      const int rr = rr0 + u * RS;
      if (rr < rows) x[u].load(qh + (int64_t(rr >> 6) * s_len + (rr & 63)) * D);
    }
#pragma unroll
    for (int u = 0; u < kRound; ++u)
      if (rr0 + u * RS < rows) x[u].add_to(acc);
  }
#pragma unroll
  for (int e = 0; e < 8; ++e) part[rs * D + ch * 8 + e] = acc[e];
  if constexpr (kWaitBeforeWrite) pdl_wait();
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
                       int qshift, float scale, float* __restrict__ scores_out) {
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
                   sel_grp, scale, scores_out);
  if (done) {
    // chained segment call: this item's selections are written
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0)
      flag_release(done + blockIdx.x + gridDim.x * (blockIdx.y + gridDim.y * blockIdx.z), token);
  }
}

// ---------------------------------------------------------------------------
// routing past kFusedRouteMaxBlocks candidate blocks (three launches)
// ---------------------------------------------------------------------------
constexpr int kChunkCands = 128;  // candidate blocks per block_topk CTA

// grid (n_qb, Hkv, B), kRouteThreads threads: q-bar of (b, h, j) into
// qbar[(b*Hkv + h)*n_qb + j, :]
template <typename T, int D>
__global__ void __launch_bounds__(kRouteThreads)
    qbar_kernel(const T* __restrict__ q, int n_q_heads, int n_kv_heads, int s_len,
                float* __restrict__ qbar) {
  pdl_launch_dependents();
  __shared__ float part[fused_route_rows<D>() * D];
  const int j = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int n_qb = s_len / kQBlock;
  block_query_mean<T, D, true>(q, b, h, j, n_q_heads, n_q_heads / n_kv_heads, s_len, part,
                               qbar + ((int64_t(b) * n_kv_heads + h) * n_qb + j) * D);
}

// threads of a block_topk_kernel CTA: 16 warps, each scoring 8 of the
// chunk's rows and ranking 2 of the 32 query blocks
constexpr int kChunkThreads = 512;

struct ChunkLayout {
  size_t bs, qb, sc, cand, total;
  int qb_stride, sc_stride;
};

__host__ __device__ inline ChunkLayout chunk_layout(int n_qb, int D) {
  ChunkLayout L;
  L.qb_stride = D + 4;             // lanes read rows 4 floats apart: no bank conflicts
  L.sc_stride = kChunkCands + 4;   // rows 16-byte aligned (read 4 keys at a time)
  size_t o = 0;
  L.bs = o;  o = align16(o + size_t(kChunkCands) * D * 4);
  L.qb = o;  o = align16(o + size_t(n_qb) * L.qb_stride * 4);
  L.sc = o;  o = align16(o + size_t(n_qb) * L.sc_stride * 4);
  L.total = o;
  // each warp's candidate list (keys and indices) over the block summaries,
  // which are dead once the scores are in
  L.cand = L.bs;
  static_assert(size_t(kChunkThreads / 32) * kChunkCands * 8 <= size_t(kChunkCands) * 64 * 4,
                "candidate lists fit in the block-summary tile");
  return L;
}

// grid (n_chunks, Hkv, B * n_split), kChunkThreads threads, dynamic shared
// memory chunk_layout(nq_max, D).total; split z % n_split takes query blocks
// [split * nq_max, min(n_qb, (split + 1) * nq_max)).  Chunk c holds candidate blocks
// [c*kChunkCands, ...) of the segment's largest candidate set [0, j_max).
// Finalists of query block j: fin_key/fin_idx[((b*Hkv + h)*n_qb + j)*n_chunks
// + c][0 .. kb_j] (topk_blocks + 1 slots per chunk) with kb_j = min(topk_blocks,
// J_j): the chunk's local top kb_j + 1 among j's valid candidates (block <
// J_j) in ascending block order, then padding (key 0, which ranks below every
// finite score; index -1).  The extra one makes the global (k+1)-th score
// available to the merge.
template <int D>
__global__ void __launch_bounds__(kChunkThreads)
    block_topk_kernel(const float* __restrict__ qpart, const float* __restrict__ qprev,
                      int qshift, const float* __restrict__ bsum, int64_t ctx_cap,
                      int n_kv_heads, int n_qb, int64_t own0, int topk_blocks, int n_split,
                      int nq_max, uint32_t* __restrict__ fin_key,
                      int32_t* __restrict__ fin_idx) {
  pdl_launch_dependents();
  pdl_wait();
  extern __shared__ __align__(16) unsigned char sm_raw[];
  const int q0 = int(blockIdx.z % n_split) * nq_max;      // this CTA's first query block
  const int nq = n_qb - q0 < nq_max ? n_qb - q0 : nq_max;  // and their number
  const ChunkLayout L = chunk_layout(nq_max, D);
  float* bs = reinterpret_cast<float*>(sm_raw + L.bs);
  float* qb = reinterpret_cast<float*>(sm_raw + L.qb);
  uint32_t* sc = reinterpret_cast<uint32_t*>(sm_raw + L.sc);
  const int c = blockIdx.x, h = blockIdx.y, b = blockIdx.z / n_split, n_chunks = gridDim.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t head = int64_t(b) * n_kv_heads + h;
  const int64_t ctx_blocks = ctx_cap / kBlock;
  const int64_t j_max = own0 + n_qb - 1;
  const int64_t lo = int64_t(c) * kChunkCands;
  const int n_loc = int(j_max - lo < kChunkCands ? j_max - lo : kChunkCands);

  // the chunk's block summaries (16-byte loads, 16 per thread in flight)
  {
    constexpr int kV = kChunkCands * D / 4 / kChunkThreads;
    const float4* src = reinterpret_cast<const float4*>(bsum + (head * ctx_blocks + lo) * D);
    float4* dst = reinterpret_cast<float4*>(bs);
    const int n4 = n_loc * D / 4;
    float4 x[kV];
#pragma unroll
    for (int u = 0; u < kV; ++u) {
      const int i = tid + u * kChunkThreads;
      x[u] = i < n4 ? src[i] : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int u = 0; u < kV; ++u) dst[tid + u * kChunkThreads] = x[u];
  }
  // every query block's q-bar row (the segment's rows of qpart, or rows
  // own0 + j - qshift of the resident block means), all loads in flight
  {
    constexpr int kQV = 32 * D / 4 / kChunkThreads;  // up to 32 query blocks per CTA
    float4 x[kQV];
#pragma unroll
    for (int u = 0; u < kQV; ++u) {
      const int i = tid + u * kChunkThreads, jj = i / (D / 4), e4 = i % (D / 4);
      const float* src = nullptr;
      if (jj < nq) {
        if (qprev) {
          const int64_t r = own0 + q0 + jj - qshift;
          if (r >= 0) src = qprev + (head * ctx_blocks + r) * D;
        } else {
          src = qpart + (head * n_qb + q0 + jj) * D;
        }
      }
      x[u] = src ? reinterpret_cast<const float4*>(src)[e4] : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int u = 0; u < kQV; ++u) {
      const int i = tid + u * kChunkThreads, jj = i / (D / 4), e4 = i % (D / 4);
      if (jj < nq) reinterpret_cast<float4*>(qb + jj * L.qb_stride)[e4] = x[u];
    }
  }
  __syncthreads();

  // scores: lane = query block (a second round past 32), each warp a slice
  // of the chunk's rows (8 of 128), 8 rows at a time, the rows read as
  // broadcasts
  {
    constexpr int kWarps = kChunkThreads / 32;
    const int rows_per_warp = (n_loc + kWarps - 1) / kWarps;
    const int r0 = warp * rows_per_warp;
    const int r1 = r0 + rows_per_warp < n_loc ? r0 + rows_per_warp : n_loc;
    for (int jb = 0; jb < nq; jb += 32) {
      const int jj = jb + lane;
      const float4* qj = reinterpret_cast<const float4*>(qb + (jj < nq ? jj : 0) * L.qb_stride);
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
        if (jj < nq)
#pragma unroll
          for (int u = 0; u < 8; ++u)
            if (i0 + u < r1) sc[jj * L.sc_stride + i0 + u] = ordered_key(acc[u]);
      }
    }
  }
  __syncthreads();

  // local top-k_b of each query block over its valid candidates, one warp
  // per query block (rank counting; ties to the lower index), compacted in
  // ascending index by ballots
  for (int jl = warp; jl < nq; jl += kChunkThreads / 32) {
    const int jj = q0 + jl;   // query block within the segment
    const int64_t J = own0 + jj;
    const int kb = int(J < topk_blocks ? J : topk_blocks) + 1;   // + the (k+1)-th
    int n_val = int(J - lo);
    n_val = n_val < 0 ? 0 : (n_val > n_loc ? n_loc : n_val);
    const int k_loc = kb < n_val ? kb : n_val;
    const uint32_t* row = sc + jl * L.sc_stride;
    const int64_t slot = ((head * n_qb + jj) * n_chunks + c) * (topk_blocks + 1);
    // keys lane, lane + 32, ... (at most 4) per lane.  Threshold: the
    // k_loc-th largest of the 32 lane maxima; at least k_loc keys reach it,
    // so only keys >= it can be selected, and they are ranked among
    // themselves (the others rank below all of them)
    constexpr int kPer = kChunkCands / 32;
    uint32_t ki[kPer];
    uint32_t lmax = 0u;
#pragma unroll
    for (int m = 0; m < kPer; ++m) {
      const int i = m * 32 + lane;
      ki[m] = i < n_val ? row[i] : 0u;
      lmax = ki[m] > lmax ? ki[m] : lmax;
    }
    uint32_t* ck = reinterpret_cast<uint32_t*>(sm_raw + L.cand) + warp * 2 * kChunkCands;
    int* ci = reinterpret_cast<int*>(ck + kChunkCands);
    int n_c = 0;
    if (k_loc > 0) {
      int rl = 0;
#pragma unroll 8
      for (int o = 0; o < 32; ++o) {
        const uint32_t other = __shfl_sync(0xffffffffu, lmax, o);
        rl += (other > lmax) || (other == lmax && o < lane);
      }
      // with k_loc above 32 there is no such lane: every valid key competes
      const unsigned who = __ballot_sync(0xffffffffu, rl == k_loc - 1);
      const uint32_t tl = __shfl_sync(0xffffffffu, lmax, who ? __ffs(who) - 1 : 0);
      const uint32_t t = who ? tl : 0u;
#pragma unroll
      for (int m = 0; m < kPer; ++m) {
        const int i = m * 32 + lane;
        const bool c = i < n_val && ki[m] >= t;
        const unsigned ball = __ballot_sync(0xffffffffu, c);
        if (c) {
          const int pos = n_c + __popc(ball & ((1u << lane) - 1u));
          ck[pos] = ki[m];
          ci[pos] = i;
        }
        n_c += __popc(ball);
      }
    }
    __syncwarp();
    // rank the candidates (in ascending index) among themselves; picks in
    // list order are in ascending index
    int written = 0;
    for (int c0 = 0; c0 < n_c; c0 += 32) {
      const int cc = c0 + lane;
      bool pick = false;
      uint32_t kc = 0u;
      if (cc < n_c) {
        kc = ck[cc];
        int r = 0;
#pragma unroll 4
        for (int c2 = 0; c2 < n_c; ++c2) {
          const uint32_t k2 = ck[c2];
          r += (k2 > kc) || (k2 == kc && c2 < cc);
        }
        pick = r < k_loc;
      }
      const unsigned ball = __ballot_sync(0xffffffffu, pick);
      if (pick) {
        const int pos = written + __popc(ball & ((1u << lane) - 1u));
        fin_key[slot + pos] = kc;
        fin_idx[slot + pos] = int(lo + ci[cc]);
      }
      written += __popc(ball);
    }
    __syncwarp();
    for (int p = k_loc + lane; p < kb; p += 32) {
      fin_key[slot + p] = 0u;
      fin_idx[slot + p] = -1;
    }
  }
}

// Shared-memory layout of select_kernel (16-byte aligned sections).
struct MergeLayout {
  size_t qb, mkey, midx, msel, blocks, key2, sel2, grp, hist, scratch, total;
};

__host__ __device__ inline MergeLayout merge_layout(int n_chunks, int topk_blocks, int D) {
  MergeLayout L;
  const size_t n_m = size_t(n_chunks) * (topk_blocks + 1);
  size_t o = 0;
  L.qb = o;      o = align16(o + size_t(D) * 4);
  L.mkey = o;    o = align16(o + n_m * 4);
  L.midx = o;    o = align16(o + n_m * 4);
  L.msel = o;    o = align16(o + n_m);
  L.blocks = o;  o = align16(o + size_t(topk_blocks) * 4);
  L.key2 = o;    o = align16(o + size_t(8) * topk_blocks * 4);
  L.sel2 = o;    o = align16(o + size_t(8) * topk_blocks);
  L.grp = o;     o = align16(o + size_t(8) * topk_blocks * 4);
  L.hist = o;    o = align16(o + 256 * 4);
  L.scratch = o; o = align16(o + 16 * 4);
  L.total = o;
  return L;
}

// grid (n_qb, Hkv, B), kRouteThreads threads, dynamic shared memory
// merge_layout(n_chunks, topk_blocks, D).total
template <int D>
__global__ void __launch_bounds__(kRouteThreads)
    select_kernel(const float* __restrict__ qpart, const float* __restrict__ qprev, int qshift,
                  const uint32_t* __restrict__ fin_key, const int32_t* __restrict__ fin_idx,
                  int n_chunks, const float* __restrict__ gsum, int64_t ctx_cap, int n_kv_heads,
                  int n_qb, int64_t own0, int topk_blocks, int topk_groups,
                  int32_t* __restrict__ sel_blk, int32_t* __restrict__ sel_grp, float scale,
                  float* __restrict__ scores_out) {
  pdl_launch_dependents();
  pdl_wait();
  extern __shared__ __align__(16) unsigned char sm_raw[];
  const MergeLayout L = merge_layout(n_chunks, topk_blocks, D);
  float* qb = reinterpret_cast<float*>(sm_raw + L.qb);
  uint32_t* mkey = reinterpret_cast<uint32_t*>(sm_raw + L.mkey);
  int* midx = reinterpret_cast<int*>(sm_raw + L.midx);
  uint8_t* msel = sm_raw + L.msel;
  int* blocks = reinterpret_cast<int*>(sm_raw + L.blocks);
  uint32_t* key2 = reinterpret_cast<uint32_t*>(sm_raw + L.key2);
  uint8_t* sel2 = sm_raw + L.sel2;
  int* grp = reinterpret_cast<int*>(sm_raw + L.grp);
  int* hist = reinterpret_cast<int*>(sm_raw + L.hist);
  int* scratch = reinterpret_cast<int*>(sm_raw + L.scratch);
  const int j = blockIdx.x, h = blockIdx.y, b = blockIdx.z, tid = threadIdx.x;
  const int64_t head = int64_t(b) * n_kv_heads + h;
  const int64_t J = own0 + j;
  const int kb = int(J < topk_blocks ? J : topk_blocks);
  const int kf = kb + 1;             // finalists per chunk
  const int n_m = n_chunks * kf;
  const int64_t base = (head * n_qb + j) * n_chunks * (topk_blocks + 1);
  for (int i = tid; i < n_m; i += kRouteThreads) {
    const int c = i / kf, p = i % kf;
    mkey[i] = fin_key[base + int64_t(c) * (topk_blocks + 1) + p];
    midx[i] = fin_idx[base + int64_t(c) * (topk_blocks + 1) + p];
  }
  float* so = scores_out ? scores_out + (head * n_qb + j) * 4 : nullptr;
  for (int e = tid; e < D; e += kRouteThreads)
    qb[e] = route_qbar(qpart, qprev, qshift, head, n_qb, 1, D, j, e, own0, ctx_cap / kBlock);
  __syncthreads();
  // level 1: the chunks' finalists in chunk order are in ascending block
  // order, so ties keep the lower block
  block_topk_indices(mkey, n_m, kb, blocks, msel, hist, scratch, scale, so);
  for (int r = tid; r < kb; r += kRouteThreads) blocks[r] = midx[blocks[r]];
  __syncthreads();
  if (sel_blk)
    for (int i = tid; i < topk_blocks; i += kRouteThreads)
      sel_blk[(head * n_qb + j) * topk_blocks + i] = i < kb ? blocks[i] : -1;
  // level 2
  const int n2 = 8 * kb;
  score_rows<D>(gsum + head * (ctx_cap / kGroup) * D, qb, n2,
                [&](int p) {
                  // a block index below 0 only comes from a non-finite summary;
                  // it is kept in bounds (the attention rejects the result)
                  const int blk = blocks[p >> 3];
                  return int64_t(blk < 0 ? 0 : blk) * kGroupsPerBlock + (p & 7);
                },
                key2);
  __syncthreads();
  const int kg = n2 < topk_groups ? n2 : topk_groups;
  block_topk_indices(key2, n2, kg, grp, sel2, hist, scratch, scale, so ? so + 2 : nullptr);
  int32_t* out = sel_grp + (head * n_qb + j) * topk_groups;
  for (int i = tid; i < topk_groups; i += kRouteThreads)
    out[i] = i < kg ? blocks[grp[i] >> 3] * kGroupsPerBlock + (grp[i] & 7) : -1;
}

}  // namespace hga
