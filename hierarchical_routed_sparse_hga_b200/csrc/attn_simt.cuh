// Steps a4 + a5 on CUDA cores (float32 FMA): exact-token attention over the
// selected 8-token groups plus the query block's causal own block, forward
// and backward under segment-wise backprop ("BMW如何通过重新设计注意力机制…",
// section "HGA的不同之处": only the selected groups' exact K/V enter the
// attention; same section, last paragraph: history is detached, later
// segments still attend to earlier exact tokens).
//
// These kernels serve float32 inputs (where tensor-core TF32 would miss a
// 1e-4 absolute tolerance) and are the fallback-free reference layout for the
// tensor-core kernels: same inputs, same key enumeration, same masks.
//
// Key enumeration of query block j (KV head h): tiles of 64 keys; routed
// tiles take 8 consecutive entries of sel_grp[b,h,j] (group g -> tokens
// 8g..8g+7), the last tile is the own block (tokens 64*J .. 64*J+63, query r
// sees own token i iff i <= r).  A group entry g is valid iff
// 0 <= g < 8*J; -1 is padding; anything else latches HGA_ERR_DEVICE_CHECK and
// is skipped.
#pragma once

#include <math.h>

#include "hga_common.cuh"

namespace hga {

constexpr int kSimtFwdThreads = 128;   // 2 threads per query row
constexpr int kSimtKvThreads = 256;    // 4 threads per key

// [part][64 rows][PW] float tile with a 4-float skew between parts, so the
// parts of one row fall in different shared-memory banks.
template <int PW>
struct SplitTile {
  static constexpr int kPartStride = 64 * PW + 4;
  __device__ static int at(int part, int row, int e) { return part * kPartStride + row * PW + e; }
};

__device__ __forceinline__ bool group_ok(int g, int64_t own_blk) {
  if (g == -1) return false;
  if (g < 0 || int64_t(g) >= own_blk * kGroupsPerBlock) {
    latch_status(HGA_ERR_DEVICE_CHECK);
    return false;
  }
  return true;
}

// Loads 64 keys (rows of K and V) of one tile into float shared memory split
// into NP parts.  pos[i] < 0 marks an invalid key (zero-filled).
template <typename T, int D, int NP>
__device__ void load_kv_tile(const T* kh, const T* vh, const int64_t* pos, float* Ks, float* Vs) {
  constexpr int PW = D / NP;
  constexpr int CH = D / 8;
  for (int c = threadIdx.x; c < 64 * CH; c += blockDim.x) {
    const int i = c / CH, col = (c % CH) * 8;
    const int part = col / PW, e = col % PW;
    float kf[8], vf[8];
    if (pos[i] >= 0) {
      load8(kh + pos[i] * D + col, kf);
      load8(vh + pos[i] * D + col, vf);
    } else {
#pragma unroll
      for (int u = 0; u < 8; ++u) kf[u] = vf[u] = 0.f;
    }
    float* kd = Ks + SplitTile<PW>::at(part, i, e);
    float* vd = Vs + SplitTile<PW>::at(part, i, e);
#pragma unroll
    for (int u = 0; u < 8; ++u) { kd[u] = kf[u]; vd[u] = vf[u]; }
  }
}

// Fills pos[64] for tile `tile` (tile == n_routed_tiles -> own block).
__device__ __forceinline__ void tile_positions(int tile, int n_routed_tiles, const int* sel,
                                               int topk_groups, int64_t own_blk, int64_t* pos) {
  for (int i = threadIdx.x; i < 64; i += blockDim.x) {
    if (tile == n_routed_tiles) {
      pos[i] = own_blk * kBlock + i;
    } else {
      const int gi = tile * kGroupsPerBlock + i / kGroup;
      const int g = gi < topk_groups ? sel[gi] : -1;
      pos[i] = (g >= 0 && int64_t(g) < own_blk * kGroupsPerBlock) ? int64_t(g) * kGroup + i % kGroup
                                                                  : -1;
    }
  }
}

template <int D>
__host__ __device__ constexpr int simt_fwd_smem_floats() {
  return 2 * 2 * SplitTile<D / 2>::kPartStride;  // Ks, Vs (2 parts each)
}

// grid (n_qb, Hq, B), 128 threads: thread = (row, half of d)
template <typename T, int D>
__global__ void __launch_bounds__(kSimtFwdThreads)
    attn_fwd_simt_kernel(const T* __restrict__ q, const T* __restrict__ k,
                         const T* __restrict__ v, int64_t ctx_cap, int64_t q_begin, int s_len,
                         int n_q_heads, int n_kv_heads, int topk_groups,
                         const int32_t* __restrict__ sel_grp, float scale, T* __restrict__ o,
                         float* __restrict__ lse) {
  constexpr int HD = D / 2;
  extern __shared__ __align__(16) float fsm[];
  float* Ks = fsm;
  float* Vs = fsm + 2 * SplitTile<HD>::kPartStride;
  __shared__ int sel[256];
  __shared__ int64_t pos[64];

  const int j = blockIdx.x, hq = blockIdx.y, b = blockIdx.z;
  const int G = n_q_heads / n_kv_heads, h = hq / G;
  const int n_qb = s_len / kQBlock;
  const int row = threadIdx.x >> 1, half = threadIdx.x & 1;
  const int64_t own_blk = (q_begin + int64_t(j) * kQBlock) / kBlock;
  const int64_t kvh = (int64_t(b) * n_kv_heads + h) * ctx_cap * D;
  const int32_t* srow = sel_grp + ((int64_t(b) * n_kv_heads + h) * n_qb + j) * topk_groups;
  for (int i = threadIdx.x; i < topk_groups; i += blockDim.x) {
    const int g = srow[i];
    sel[i] = group_ok(g, own_blk) ? g : -1;
  }

  float qr[HD], acc[HD];
  const T* qrow = q + ((int64_t(b) * n_q_heads + hq) * s_len + int64_t(j) * kQBlock + row) * D + half * HD;
#pragma unroll
  for (int e = 0; e < HD; e += 8) load8(qrow + e, qr + e);
#pragma unroll
  for (int e = 0; e < HD; ++e) acc[e] = 0.f;
  float m = -INFINITY, l = 0.f;

  const int n_routed_tiles = (topk_groups + kGroupsPerBlock - 1) / kGroupsPerBlock;
  __syncthreads();
  for (int tile = 0; tile <= n_routed_tiles; ++tile) {
    tile_positions(tile, n_routed_tiles, sel, topk_groups, own_blk, pos);
    __syncthreads();
    load_kv_tile<T, D, 2>(k + kvh, v + kvh, pos, Ks, Vs);
    __syncthreads();
    const bool own = tile == n_routed_tiles;
    for (int i = 0; i < 64; ++i) {
      const float* kr = Ks + SplitTile<HD>::at(half, i, 0);
      float part = 0.f;
#pragma unroll
      for (int e = 0; e < HD; e += 4) {
        const float4 kv4 = *reinterpret_cast<const float4*>(kr + e);
        part = fmaf(qr[e], kv4.x, part);
        part = fmaf(qr[e + 1], kv4.y, part);
        part = fmaf(qr[e + 2], kv4.z, part);
        part = fmaf(qr[e + 3], kv4.w, part);
      }
      part += __shfl_xor_sync(0xffffffffu, part, 1);
      const bool ok = pos[i] >= 0 && (!own || i <= row);
      if (ok) {
        const float s = part * scale;
        if (s > m) {
          const float c = expf(m - s);
          l *= c;
#pragma unroll
          for (int e = 0; e < HD; ++e) acc[e] *= c;
          m = s;
        }
        const float p = expf(s - m);
        l += p;
        const float* vr = Vs + SplitTile<HD>::at(half, i, 0);
#pragma unroll
        for (int e = 0; e < HD; e += 4) {
          const float4 vv = *reinterpret_cast<const float4*>(vr + e);
          acc[e] = fmaf(p, vv.x, acc[e]);
          acc[e + 1] = fmaf(p, vv.y, acc[e + 1]);
          acc[e + 2] = fmaf(p, vv.z, acc[e + 2]);
          acc[e + 3] = fmaf(p, vv.w, acc[e + 3]);
        }
      }
    }
    __syncthreads();
  }
  const float inv = 1.f / l;
#pragma unroll
  for (int e = 0; e < HD; ++e) acc[e] *= inv;
  T* orow = o + ((int64_t(b) * n_q_heads + hq) * s_len + int64_t(j) * kQBlock + row) * D + half * HD;
#pragma unroll
  for (int e = 0; e < HD; e += 8) store8(orow + e, acc + e);
  if (half == 0) lse[(int64_t(b) * n_q_heads + hq) * s_len + int64_t(j) * kQBlock + row] = m + logf(l);
}

// grid (n_qb, Hq, B), 128 threads.  dQ for every attended key; also writes
// D = rowsum(dO * O) to dvec for the dK/dV kernel.
template <typename T, int D>
__global__ void __launch_bounds__(kSimtFwdThreads)
    attn_bwd_dq_simt_kernel(const T* __restrict__ q, const T* __restrict__ k,
                            const T* __restrict__ v, int64_t ctx_cap, int64_t q_begin, int s_len,
                            int n_q_heads, int n_kv_heads, int topk_groups,
                            const int32_t* __restrict__ sel_grp, float scale,
                            const T* __restrict__ o, const float* __restrict__ lse,
                            const T* __restrict__ d_o, T* __restrict__ dq,
                            float* __restrict__ dvec) {
  constexpr int HD = D / 2;
  extern __shared__ __align__(16) float fsm[];
  float* Ks = fsm;
  float* Vs = fsm + 2 * SplitTile<HD>::kPartStride;
  __shared__ int sel[256];
  __shared__ int64_t pos[64];

  const int j = blockIdx.x, hq = blockIdx.y, b = blockIdx.z;
  const int G = n_q_heads / n_kv_heads, h = hq / G;
  const int n_qb = s_len / kQBlock;
  const int row = threadIdx.x >> 1, half = threadIdx.x & 1;
  const int64_t own_blk = (q_begin + int64_t(j) * kQBlock) / kBlock;
  const int64_t kvh = (int64_t(b) * n_kv_heads + h) * ctx_cap * D;
  const int32_t* srow = sel_grp + ((int64_t(b) * n_kv_heads + h) * n_qb + j) * topk_groups;
  for (int i = threadIdx.x; i < topk_groups; i += blockDim.x) {
    const int g = srow[i];
    sel[i] = group_ok(g, own_blk) ? g : -1;
  }

  const int64_t rix = (int64_t(b) * n_q_heads + hq) * s_len + int64_t(j) * kQBlock + row;
  float qr[HD], dor[HD], acc[HD];
  float drow;
  {
    float orr[HD];
#pragma unroll
    for (int e = 0; e < HD; e += 8) {
      load8(q + rix * D + half * HD + e, qr + e);
      load8(d_o + rix * D + half * HD + e, dor + e);
      load8(o + rix * D + half * HD + e, orr + e);
    }
    float part = 0.f;
#pragma unroll
    for (int e = 0; e < HD; ++e) part = fmaf(dor[e], orr[e], part);
    drow = part + __shfl_xor_sync(0xffffffffu, part, 1);
  }
  if (half == 0) dvec[rix] = drow;
  const float lrow = lse[rix];
#pragma unroll
  for (int e = 0; e < HD; ++e) acc[e] = 0.f;

  const int n_routed_tiles = (topk_groups + kGroupsPerBlock - 1) / kGroupsPerBlock;
  __syncthreads();
  for (int tile = 0; tile <= n_routed_tiles; ++tile) {
    tile_positions(tile, n_routed_tiles, sel, topk_groups, own_blk, pos);
    __syncthreads();
    load_kv_tile<T, D, 2>(k + kvh, v + kvh, pos, Ks, Vs);
    __syncthreads();
    const bool own = tile == n_routed_tiles;
    for (int i = 0; i < 64; ++i) {
      const float* kr = Ks + SplitTile<HD>::at(half, i, 0);
      const float* vr = Vs + SplitTile<HD>::at(half, i, 0);
      float sp = 0.f, dpp = 0.f;
#pragma unroll
      for (int e = 0; e < HD; e += 4) {
        const float4 kv4 = *reinterpret_cast<const float4*>(kr + e);
        const float4 vv4 = *reinterpret_cast<const float4*>(vr + e);
        sp = fmaf(qr[e], kv4.x, sp);
        sp = fmaf(qr[e + 1], kv4.y, sp);
        sp = fmaf(qr[e + 2], kv4.z, sp);
        sp = fmaf(qr[e + 3], kv4.w, sp);
        dpp = fmaf(dor[e], vv4.x, dpp);
        dpp = fmaf(dor[e + 1], vv4.y, dpp);
        dpp = fmaf(dor[e + 2], vv4.z, dpp);
        dpp = fmaf(dor[e + 3], vv4.w, dpp);
      }
      sp += __shfl_xor_sync(0xffffffffu, sp, 1);
      dpp += __shfl_xor_sync(0xffffffffu, dpp, 1);
      const bool ok = pos[i] >= 0 && (!own || i <= row);
      if (ok) {
        const float p = expf(sp * scale - lrow);
        const float ds = p * (dpp - drow);
#pragma unroll
        for (int e = 0; e < HD; e += 4) {
          const float4 kv4 = *reinterpret_cast<const float4*>(kr + e);
          acc[e] = fmaf(ds, kv4.x, acc[e]);
          acc[e + 1] = fmaf(ds, kv4.y, acc[e + 1]);
          acc[e + 2] = fmaf(ds, kv4.z, acc[e + 2]);
          acc[e + 3] = fmaf(ds, kv4.w, acc[e + 3]);
        }
      }
    }
    __syncthreads();
  }
#pragma unroll
  for (int e = 0; e < HD; ++e) acc[e] *= scale;
#pragma unroll
  for (int e = 0; e < HD; e += 8) store8(dq + rix * D + half * HD + e, acc + e);
}

template <int D>
__host__ __device__ constexpr int simt_kv_smem_floats() {
  return 2 * 4 * SplitTile<D / 4>::kPartStride;  // Qs, dOs (4 parts each)
}

// grid (n_qb, Hkv, B), 256 threads: thread = (key of the active key block
// kb = blockIdx.x, quarter of d).  Visits every query block j >= kb of the
// segment that attends to block kb (its own query block causally, later ones
// through the groups of kb they selected), in increasing j and head order, so
// the sums are deterministic.
template <typename T, int D>
__global__ void __launch_bounds__(kSimtKvThreads)
    attn_bwd_dkdv_simt_kernel(const T* __restrict__ q, const T* __restrict__ k,
                              const T* __restrict__ v, int64_t ctx_cap, int64_t q_begin,
                              int s_len, int n_q_heads, int n_kv_heads, int topk_groups,
                              const int32_t* __restrict__ sel_grp, float scale,
                              const float* __restrict__ lse, const T* __restrict__ d_o,
                              const float* __restrict__ dvec, T* __restrict__ dk,
                              T* __restrict__ dv) {
  constexpr int QD = D / 4;
  extern __shared__ __align__(16) float fsm[];
  float* Qs = fsm;
  float* dOs = fsm + 4 * SplitTile<QD>::kPartStride;
  __shared__ float lse_s[64], d_s[64];
  __shared__ int masks[64];  // per query block of the segment (s_len <= 4096)

  const int kb = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int G = n_q_heads / n_kv_heads;
  const int n_qb = s_len / kQBlock;
  const int key = threadIdx.x >> 2, quarter = threadIdx.x & 3;
  const int64_t gblk = q_begin / kBlock + kb;  // global index of this key block
  const int64_t kpos = gblk * kBlock + key;
  const int64_t kvh = (int64_t(b) * n_kv_heads + h) * ctx_cap * D;

  for (int jj = threadIdx.x; jj < n_qb; jj += blockDim.x) masks[jj] = jj == kb ? 0xff : 0;
  __syncthreads();
  const int32_t* sel_bh = sel_grp + (int64_t(b) * n_kv_heads + h) * n_qb * topk_groups;
  for (int idx = threadIdx.x; idx < n_qb * topk_groups; idx += blockDim.x) {
    const int jj = idx / topk_groups;
    if (jj <= kb) continue;
    const int g = sel_bh[idx];
    const int64_t own_jj = q_begin / kBlock + jj;
    if (g >= 0 && int64_t(g) < own_jj * kGroupsPerBlock && int64_t(g) / kGroupsPerBlock == gblk)
      atomicOr(&masks[jj], 1 << (g % kGroupsPerBlock));
  }

  float kr[QD], vr[QD], dka[QD], dva[QD];
#pragma unroll
  for (int e = 0; e < QD; e += 8) {
    load8(k + kvh + kpos * D + quarter * QD + e, kr + e);
    load8(v + kvh + kpos * D + quarter * QD + e, vr + e);
  }
#pragma unroll
  for (int e = 0; e < QD; ++e) dka[e] = dva[e] = 0.f;
  __syncthreads();

  constexpr int CH = D / 8;
  for (int jj = kb; jj < n_qb; ++jj) {
    const int mask = masks[jj];
    if (mask == 0) continue;
    const bool own = jj == kb;
    const bool key_on = (mask >> (key / kGroup)) & 1;
    for (int hq = h * G; hq < (h + 1) * G; ++hq) {
      const int64_t r0 = (int64_t(b) * n_q_heads + hq) * s_len + int64_t(jj) * kQBlock;
      for (int c = threadIdx.x; c < 64 * CH; c += blockDim.x) {
        const int r = c / CH, col = (c % CH) * 8;
        float qf[8], df[8];
        load8(q + (r0 + r) * D + col, qf);
        load8(d_o + (r0 + r) * D + col, df);
        float* qd = Qs + SplitTile<QD>::at(col / QD, r, col % QD);
        float* dd = dOs + SplitTile<QD>::at(col / QD, r, col % QD);
#pragma unroll
        for (int u = 0; u < 8; ++u) { qd[u] = qf[u]; dd[u] = df[u]; }
      }
      for (int r = threadIdx.x; r < 64; r += blockDim.x) {
        lse_s[r] = lse[r0 + r];
        d_s[r] = dvec[r0 + r];
      }
      __syncthreads();
      for (int r = 0; r < 64; ++r) {
        const float* qrow = Qs + SplitTile<QD>::at(quarter, r, 0);
        const float* drow = dOs + SplitTile<QD>::at(quarter, r, 0);
        float sp = 0.f, dpp = 0.f;
#pragma unroll
        for (int e = 0; e < QD; e += 4) {
          const float4 q4 = *reinterpret_cast<const float4*>(qrow + e);
          const float4 d4 = *reinterpret_cast<const float4*>(drow + e);
          sp = fmaf(kr[e], q4.x, sp);
          sp = fmaf(kr[e + 1], q4.y, sp);
          sp = fmaf(kr[e + 2], q4.z, sp);
          sp = fmaf(kr[e + 3], q4.w, sp);
          dpp = fmaf(vr[e], d4.x, dpp);
          dpp = fmaf(vr[e + 1], d4.y, dpp);
          dpp = fmaf(vr[e + 2], d4.z, dpp);
          dpp = fmaf(vr[e + 3], d4.w, dpp);
        }
        sp += __shfl_xor_sync(0xffffffffu, sp, 1);
        sp += __shfl_xor_sync(0xffffffffu, sp, 2);
        dpp += __shfl_xor_sync(0xffffffffu, dpp, 1);
        dpp += __shfl_xor_sync(0xffffffffu, dpp, 2);
        const bool ok = key_on && (!own || key <= r);
        if (ok) {
          const float p = expf(sp * scale - lse_s[r]);
          const float ds = p * (dpp - d_s[r]);
#pragma unroll
          for (int e = 0; e < QD; e += 4) {
            const float4 q4 = *reinterpret_cast<const float4*>(qrow + e);
            const float4 d4 = *reinterpret_cast<const float4*>(drow + e);
            dva[e] = fmaf(p, d4.x, dva[e]);
            dva[e + 1] = fmaf(p, d4.y, dva[e + 1]);
            dva[e + 2] = fmaf(p, d4.z, dva[e + 2]);
            dva[e + 3] = fmaf(p, d4.w, dva[e + 3]);
            dka[e] = fmaf(ds, q4.x, dka[e]);
            dka[e + 1] = fmaf(ds, q4.y, dka[e + 1]);
            dka[e + 2] = fmaf(ds, q4.z, dka[e + 2]);
            dka[e + 3] = fmaf(ds, q4.w, dka[e + 3]);
          }
        }
      }
      __syncthreads();
    }
  }
#pragma unroll
  for (int e = 0; e < QD; ++e) dka[e] *= scale;
  const int64_t orow = ((int64_t(b) * n_kv_heads + h) * s_len + int64_t(kb) * kBlock + key) * D +
                       quarter * QD;
#pragma unroll
  for (int e = 0; e < QD; e += 8) {
    store8(dk + orow + e, dka + e);
    store8(dv + orow + e, dva + e);
  }
}

}  // namespace hga
