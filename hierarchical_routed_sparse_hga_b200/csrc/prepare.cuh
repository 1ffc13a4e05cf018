// The upstream pass of a segment: from the Q/K/V projection outputs to what
// the path reads, in one read of the projections ("BMW如何通过重新设计注意力
// 机制…", section "HGA的不同之处": the router scores the existing projected
// keys; the workloads apply RoPE, base 1e6, before the summaries).
//
// One CTA per (64-token block, KV head, batch).  It rotates the block's
// G query rows and its key rows (rotate-half RoPE at the global position,
// theta_i = base^(-2i/d)), stores Q head-major and K/V into the whole-context
// buffers, and from the stored (rounded) values forms the block's 8 group
// summaries, its block summary and its mean query (over the 64 tokens and
// the G heads).  The routing can then work from the resident summaries
// alone, without reading Q or K again.
//
// Angles p * theta_i are reduced modulo 2 pi in double precision before the
// single-precision sine and cosine: at p = 131071 a float product alone
// would be off by ~1e-2 rad.
#pragma once

#include "hga_common.cuh"

namespace hga {

constexpr int kPrepThreads = 256;

// (cos, sin) of token t, frequency i = 8c + k (lane c of a row holds
// frequencies 8c .. 8c+7) at cs[t][k * LANES + c]: the lanes of a warp (rows
// t .. t+R-1, all c) read one k at a time; the row stride (LANES*8 + pad
// entries) puts the rows on different bank halves, so a read takes the two
// wavefronts its 256 bytes need.  The key tile and the query partials have
// one float of padding per row for the same reason.
template <int D>
struct PrepShared {
  static constexpr int kLanes = D / 16;
  static constexpr int kCsStride = kLanes * 8 + (kLanes == 8 ? 8 : 4);
  float2 cs[kQBlock][kCsStride];
  double theta[D / 2];          // base^(-2i/d)
  float kt[kQBlock][D + 1];     // the block's stored keys, as float
  float qp[kPrepThreads / kLanes][D + 1];  // per row slot: partial sums of the stored queries
};

// grid (s_len/64, n_kv_heads, batch), kPrepThreads threads, dynamic shared
// memory sizeof(PrepShared<D>).  Lanes per row: D/16, each holding 8
// rotation pairs (elements 8c .. 8c+7 and D/2 + 8c .. D/2 + 8c+7).
template <typename T, int D>
__global__ void __launch_bounds__(kPrepThreads)
    prepare_kernel(const T* __restrict__ q_proj, const T* __restrict__ k_proj,
                   const T* __restrict__ v_proj, int64_t q_row_stride, int64_t kv_row_stride,
                   int64_t q_begin, int s_len,
                   int64_t ctx_cap, int n_q_heads, int n_kv_heads, double log2_base,
                   T* __restrict__ q_out, T* __restrict__ k, T* __restrict__ v,
                   float* __restrict__ gsum, float* __restrict__ bsum, float* __restrict__ qsum) {
  extern __shared__ __align__(16) unsigned char sm_raw[];
  PrepShared<D>& sh = *reinterpret_cast<PrepShared<D>*>(sm_raw);
  constexpr int HALF = D / 2, LANES = D / 16, SLOTS = kPrepThreads / LANES;
  const int j = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int G = n_q_heads / n_kv_heads;
  const int tid = threadIdx.x, c = tid % LANES, slot = tid / LANES;
  const bool rotate = log2_base > 0.0;

  // rows: G x 64 query rows, then 64 key rows, then 64 value rows; a round
  // takes kBatch rows per row slot, their loads in flight together (raw
  // 8-element words until used)
  const int n_rows = (G + 2) * kQBlock;
  constexpr int kBatch = sizeof(T) == 2 ? 6 : 3;
  auto row_src = [&](int r) {
    const int kind = r / kQBlock;  // 0..G-1: query head; G: key; G+1: value
    const int64_t tok = int64_t(b) * s_len + int64_t(j) * kQBlock + r % kQBlock;
    return kind < G ? q_proj + tok * q_row_stride + int64_t(h * G + kind) * D
                    : (kind == G ? k_proj : v_proj) + tok * kv_row_stride + int64_t(h) * D;
  };
  Raw8<T> x1[kBatch], x2[kBatch];
  auto load_round = [&](int r0) {
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      const int r = r0 + u * SLOTS;
      if (r < n_rows) {
        const T* src = row_src(r);
        x1[u].load(src + 8 * c);
        x2[u].load(src + HALF + 8 * c);
      }
    }
  };
  // the projections are inputs no kernel of the library writes: the first
  // round's loads go out before the table is built and before the wait for
  // the previous kernel (which only this kernel's stores must follow)
  load_round(slot);

  // (cos, sin) of the 64 tokens' angles, reduced modulo 2 pi in double
  if (rotate) {
    for (int i = tid; i < HALF; i += kPrepThreads) sh.theta[i] = exp2(-(2.0 * i / D) * log2_base);
    __syncthreads();
    constexpr double kTwoPi = 6.283185307179586476925286766559;
    for (int idx = tid; idx < kQBlock * HALF; idx += kPrepThreads) {
      const int t = idx / HALF, i = idx % HALF;
      const double ang = double(q_begin + int64_t(j) * kQBlock + t) * sh.theta[i];
      const double red = fma(-rint(ang * (1.0 / kTwoPi)), kTwoPi, ang);
      float s, co;
      sincosf(float(red), &s, &co);
      sh.cs[t][(i % 8) * LANES + i / 8] = make_float2(co, s);
    }
  }
  pdl_wait();
  __syncthreads();

  float qacc[16];
#pragma unroll
  for (int e = 0; e < 16; ++e) qacc[e] = 0.f;
  for (int r0 = slot; r0 < n_rows; r0 += kBatch * SLOTS) {
    if (r0 != slot) load_round(r0);
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      const int r = r0 + u * SLOTS;
      if (r >= n_rows) continue;
      const int kind = r / kQBlock;
      const int t = r % kQBlock;
      float y1[8], y2[8];
      x1[u].get(y1);
      x2[u].get(y2);
      if (kind <= G && rotate) {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const float2 cs = sh.cs[t][i * LANES + c];
          const float a = y1[i], bb = y2[i];
          y1[i] = a * cs.x - bb * cs.y;
          y2[i] = bb * cs.x + a * cs.y;
        }
      }
      // the stored values (rounded to T) are what the summaries see
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        y1[i] = to_float(from_float<T>(y1[i]));
        y2[i] = to_float(from_float<T>(y2[i]));
      }
      const int64_t ts = int64_t(j) * kQBlock + t;
      T* dst;
      if (kind < G) {
        dst = q_out + ((int64_t(b) * n_q_heads + h * G + kind) * s_len + ts) * D;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          qacc[i] += y1[i];
          qacc[8 + i] += y2[i];
        }
      } else {
        dst = (kind == G ? k : v) + ((int64_t(b) * n_kv_heads + h) * ctx_cap + q_begin + ts) * D;
        if (kind == G)
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            sh.kt[t][8 * c + i] = y1[i];
            sh.kt[t][HALF + 8 * c + i] = y2[i];
          }
      }
      store8(dst + 8 * c, y1);
      store8(dst + HALF + 8 * c, y2);
    }
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    sh.qp[slot][8 * c + i] = qacc[i];
    sh.qp[slot][HALF + 8 * c + i] = qacc[8 + i];
  }
  __syncthreads();

  // the block's 8 group summaries, its block summary and its mean query
  const int64_t head = int64_t(b) * n_kv_heads + h;
  const int64_t g0 = q_begin / kGroup + int64_t(j) * kGroupsPerBlock;
  const int64_t blk = q_begin / kBlock + j;
  for (int idx = tid; idx < kGroupsPerBlock * D; idx += kPrepThreads) {
    const int g = idx / D, e = idx % D;
    float s = 0.f;
#pragma unroll
    for (int t = 0; t < kGroup; ++t) s += sh.kt[g * kGroup + t][e];
    gsum[(head * (ctx_cap / kGroup) + g0 + g) * D + e] = s * (1.f / kGroup);
  }
  for (int e = tid; e < D; e += kPrepThreads) {
    float s = 0.f;
    for (int t = 0; t < kQBlock; ++t) s += sh.kt[t][e];
    bsum[(head * (ctx_cap / kBlock) + blk) * D + e] = s * (1.f / kBlock);
    float qs = 0.f;
    for (int r = 0; r < SLOTS; ++r) qs += sh.qp[r][e];
    qsum[(head * (ctx_cap / kBlock) + blk) * D + e] = qs / float(G * kQBlock);
  }
  // The next kernel may start only once every CTA's stores are visible:
  // the routing and summary kernels read Q and K before their own wait for
  // this grid, so the trigger comes after the CTA's last store (the barrier)
  // and a device-scope fence.
  __syncthreads();
  __threadfence();
  pdl_launch_dependents();
}

}  // namespace hga
