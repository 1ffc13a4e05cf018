// libhga: C ABI of the HGA hot path (declarations and contracts in hga.h).
// Host side: argument checks, workspace carving, kernel selection and launch.
// Nothing here allocates, frees or synchronises (except hga_get_device_status).
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>
#include <cmath>
#include <atomic>
#include <initializer_list>
#include <map>
#include <mutex>
#include <utility>

#include "hga.h"
#include "hga_common.cuh"
#include "summaries.cuh"
#include "route.cuh"
#include "attn_simt.cuh"
#include "attn_fwd_sm100.cuh"
#include "attn_bwd_sm100.cuh"
#include "tier.cuh"
#include "decode.cuh"
#include "prepare.cuh"
#include "file_tier.h"
#include "trace.cuh"

using namespace hga;

namespace {

constexpr int64_t kMaxSegment = 4096;  // s_len limit (64 query blocks)

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

hga_status_t check_cfg(const hga_config_t* c) {
  if (!c) return HGA_ERR_INVALID_ARG;
  if (c->batch < 1 || c->n_kv_heads < 1 || c->n_q_heads < 1) return HGA_ERR_INVALID_ARG;
  if (c->n_q_heads % c->n_kv_heads != 0) return HGA_ERR_INVALID_ARG;
  if (c->n_q_heads / c->n_kv_heads > 8) return HGA_ERR_UNSUPPORTED;
  if (c->head_dim != 64 && c->head_dim != 128) return HGA_ERR_UNSUPPORTED;
  if (c->dtype != HGA_F32 && c->dtype != HGA_BF16) return HGA_ERR_UNSUPPORTED;
  if (c->topk_blocks < 1 || c->topk_blocks > 64) return HGA_ERR_UNSUPPORTED;
  if (c->topk_groups < 1 || c->topk_groups > 256) return HGA_ERR_UNSUPPORTED;
  if (!(c->scale > 0.f) || c->scale != c->scale) return HGA_ERR_INVALID_ARG;
  if (c->batch > 65535 || c->n_q_heads > 65535) return HGA_ERR_UNSUPPORTED;
  return HGA_OK;
}

hga_status_t check_segment(int64_t ctx_cap, int64_t q_begin, int32_t s_len) {
  if (ctx_cap <= 0 || ctx_cap % kBlock) return HGA_ERR_INVALID_ARG;
  if (q_begin < 0 || q_begin % kBlock) return HGA_ERR_INVALID_ARG;
  if (s_len <= 0 || s_len % kQBlock) return HGA_ERR_INVALID_ARG;
  if (s_len > kMaxSegment) return HGA_ERR_UNSUPPORTED;
  if (q_begin + s_len > ctx_cap) return HGA_ERR_INVALID_ARG;
  return HGA_OK;
}

// Raise a kernel's dynamic shared-memory limit once per (kernel, device).
hga_status_t ensure_smem(const void* fn, size_t bytes) {
  if (bytes <= 48 * 1024) return HGA_OK;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return HGA_ERR_CUDA;
  static std::mutex mu;
  static std::map<std::pair<const void*, int>, size_t> done;
  std::lock_guard<std::mutex> lock(mu);
  auto key = std::make_pair(fn, dev);
  auto it = done.find(key);
  if (it != done.end() && it->second >= bytes) return HGA_OK;
  int optin = 0;
  if (cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess)
    return HGA_ERR_CUDA;
  if (bytes > size_t(optin)) return HGA_ERR_UNSUPPORTED;
  if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, int(bytes)) !=
      cudaSuccess)
    return HGA_ERR_CUDA;
  done[key] = bytes;
  return HGA_OK;
}

// Calls body.template operator()<T, D>() for the configured element type and d.
template <typename Body>
hga_status_t dispatch(const hga_config_t* c, Body&& body) {
  if (c->dtype == HGA_BF16) {
    if (c->head_dim == 128) return body.template operator()<__nv_bfloat16, 128>();
    return body.template operator()<__nv_bfloat16, 64>();
  }
  if (c->head_dim == 128) return body.template operator()<float, 128>();
  return body.template operator()<float, 64>();
}

// ---- TMA tensor maps (driver entry point reached through the runtime) ----
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_tiled() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// Row-major [rows, 128] bf16 matrix, boxes of 64 columns (128 B, swizzled) x box_rows.
bool make_map_bf16_d128(CUtensorMap* map, const void* base, uint64_t rows, uint32_t box_rows) {
  EncodeTiledFn fn = encode_tiled();
  if (!fn) return false;
  cuuint64_t dims[2] = {128, rows};
  cuuint64_t strides[1] = {128 * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The same matrix seen as [halves = 2][rows][64 columns] (global strides
// 128 B for a half, 256 B for a row), boxes of 64 x box_rows x 2 land in
// shared memory as [half][row][128 B]: a group of 8 rows in one copy.
bool make_map_bf16_d128_groups(CUtensorMap* map, const void* base, uint64_t rows,
                               uint32_t box_rows) {
  EncodeTiledFn fn = encode_tiled();
  if (!fn) return false;
  cuuint64_t dims[3] = {64, rows, 2};
  cuuint64_t strides[2] = {256, 128};
  cuuint32_t box[3] = {64, box_rows, 2};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// SM count of the current device (cached per device)
int sm_count() {
  static int cache[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (cache[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      n = 148;
    cache[dev] = n;
  }
  return cache[dev];
}

bool use_tensor_cores(const hga_config_t* c, int64_t ctx_cap, int32_t s_len) {
  const int G = c->n_q_heads / c->n_kv_heads;
  if (c->flags & HGA_FLAG_SIMT) return false;
  if (c->dtype != HGA_BF16 || c->head_dim != 128 || (G != 2 && G != 4)) return false;
  // TMA row coordinates are 32-bit
  if (int64_t(c->batch) * c->n_kv_heads * ctx_cap >= (int64_t(1) << 31)) return false;
  if (int64_t(c->batch) * c->n_q_heads * s_len >= (int64_t(1) << 31)) return false;
  return true;
}

template <int MT>
hga_status_t launch_fwd_tc(const hga_config_t* cfg, const void* q, const void* k, const void* v,
                           int64_t ctx_cap, int64_t q_begin, int32_t s_len,
                           const int32_t* sel_grp, void* o, float* lse, const int* route_done,
                           int* done, uint32_t token, cudaStream_t s) {
  using L = fwdtc::Layout<MT>;
  CUtensorMap tq, tk, tv, to;
  const uint64_t q_rows = uint64_t(cfg->batch) * cfg->n_q_heads * s_len;
  const uint64_t kv_rows = uint64_t(cfg->batch) * cfg->n_kv_heads * ctx_cap;
  if (!make_map_bf16_d128(&tq, q, q_rows, 64) || !make_map_bf16_d128(&to, o, q_rows, 64) ||
      !make_map_bf16_d128_groups(&tk, k, kv_rows, 8) ||
      !make_map_bf16_d128_groups(&tv, v, kv_rows, 8))
    return HGA_ERR_CUDA;
  hga_status_t e = ensure_smem(
      reinterpret_cast<const void*>(&fwdtc::attn_fwd_tc_kernel<MT>), L::kDynSmem);
  if (e != HGA_OK) return e;
  const int sets = cfg->n_q_heads / cfg->n_kv_heads / (2 * MT);
  dim3 grid((s_len / kQBlock) * sets, cfg->n_kv_heads, cfg->batch);
  const float scale_log2 = cfg->scale * 1.4426950408889634f;
  return traced_launch(HGA_K_FWD_TC, s, [&] {
    return launch_pdl(fwdtc::attn_fwd_tc_kernel<MT>, grid, dim3(L::kThreads), L::kDynSmem, s, tq,
        tk, tv, to, ctx_cap, q_begin, s_len, cfg->n_q_heads, cfg->n_kv_heads, cfg->topk_groups,
        sel_grp, scale_log2, lse, cfg->flags, route_done, done, token);
  });
}

template <int MT>
hga_status_t launch_bwd_tc(const hga_config_t* cfg, const void* q, const void* k, const void* v,
                           int64_t ctx_cap, int64_t q_begin, int32_t s_len,
                           const int32_t* sel_grp, const void* o, const float* lse,
                           const void* d_o, void* dq, void* dk, void* dv, float* dvec,
                           int* unit_counter, const int* fwd_done, int* d_done, uint32_t token,
                           int* inv, cudaStream_t s) {
  using LQ = bwdtc::DqLayout<MT>;
  using LK = bwdtc::KvLayout;
  CUtensorMap tq, tdo, tk, tv, tdq, tkg, tvg;
  const uint64_t q_rows = uint64_t(cfg->batch) * cfg->n_q_heads * s_len;
  const uint64_t kv_rows = uint64_t(cfg->batch) * cfg->n_kv_heads * ctx_cap;
  if (!make_map_bf16_d128(&tq, q, q_rows, 64) || !make_map_bf16_d128(&tdo, d_o, q_rows, 64) ||
      !make_map_bf16_d128(&tdq, dq, q_rows, 64) ||
      !make_map_bf16_d128_groups(&tkg, k, kv_rows, 8) ||
      !make_map_bf16_d128_groups(&tvg, v, kv_rows, 8) ||
      !make_map_bf16_d128(&tk, k, kv_rows, 8) || !make_map_bf16_d128(&tv, v, kv_rows, 8))
    return HGA_ERR_CUDA;
  hga_status_t e = ensure_smem(
      reinterpret_cast<const void*>(&bwdtc::attn_bwd_dq_tc_kernel<MT>), LQ::kDynSmem);
  if (e != HGA_OK) return e;
  e = ensure_smem(reinterpret_cast<const void*>(&bwdtc::attn_bwd_dkdv_tc_kernel<MT>),
                  LK::kDynSmem);
  if (e != HGA_OK) return e;
  dim3 grid(s_len / kQBlock, cfg->n_kv_heads, cfg->batch);
  const float scale_log2 = cfg->scale * 1.4426950408889634f;
  e = traced_launch(HGA_K_BWD_DQ_TC, s, [&] {
    return launch_pdl(bwdtc::attn_bwd_dq_tc_kernel<MT>, grid, dim3(LQ::kThreads), LQ::kDynSmem, s,
        tq, tdo, tkg, tvg, ctx_cap, q_begin, s_len, cfg->n_q_heads, cfg->n_kv_heads, cfg->topk_groups, sel_grp,
        cfg->scale, scale_log2, static_cast<const __nv_bfloat16*>(o),
        static_cast<const __nv_bfloat16*>(d_o), lse, tdq, dvec,
        unit_counter, fwd_done, d_done, token, inv);
  });
  if (e != HGA_OK) return e;
  // persistent: at most one CTA per SM over the (key block, head) units
  const int n_units = (s_len / kBlock) * cfg->batch * cfg->n_kv_heads;
  dim3 grid_kv(unsigned(std::min(n_units, sm_count())));
  return traced_launch(HGA_K_BWD_DKDV_TC, s, [&] {
    return launch_pdl(bwdtc::attn_bwd_dkdv_tc_kernel<MT>, grid_kv, dim3(LK::kThreads),
        LK::kDynSmem, s, tq, tdo, tk, tv, ctx_cap, q_begin, s_len, cfg->batch, cfg->n_q_heads,
        cfg->n_kv_heads, cfg->topk_groups, sel_grp, cfg->scale, scale_log2, lse, dvec,
        static_cast<__nv_bfloat16*>(dk), static_cast<__nv_bfloat16*>(dv), unit_counter,
        fwd_done ? d_done : nullptr, token, inv);
  });
}

struct RouteCarve {
  float* qbar;          // [B, Hkv, S/64, d]
  uint32_t* fin_key;    // [B, Hkv, S/64, n_chunks, topk_blocks + 1]
  int32_t* fin_idx;     // same
  int n_chunks;
  size_t bytes;
};

// The routing workspace of the three-launch path: the query blocks' q-bar,
// then the candidate chunks' finalists (keys, then block indices), each
// section 256-byte aligned.
RouteCarve route_carve(const hga_config_t* c, int32_t s_len, int64_t q_begin, void* base) {
  const int64_t n_qb = s_len / kQBlock;
  const int64_t heads = int64_t(c->batch) * c->n_kv_heads;
  const int64_t j_max = q_begin / kBlock + n_qb - 1;
  RouteCarve r;
  r.n_chunks = int(j_max > 0 ? (j_max + kChunkCands - 1) / kChunkCands : 1);
  const size_t qbar_bytes = align256(size_t(heads * n_qb * c->head_dim) * 4);
  const size_t fin_bytes =
      align256(size_t(heads * n_qb) * r.n_chunks * (c->topk_blocks + 1) * 4);
  char* p = static_cast<char*>(base);
  r.qbar = static_cast<float*>(base);
  r.fin_key = base ? reinterpret_cast<uint32_t*>(p + qbar_bytes) : nullptr;
  r.fin_idx = base ? reinterpret_cast<int32_t*>(p + qbar_bytes + fin_bytes) : nullptr;
  r.bytes = qbar_bytes + 2 * fin_bytes;
  return r;
}

}  // namespace

// Scratch of hga_route_noalloc: a fixed device array, so that entry point
// never allocates.  Host code must not pass `g_noalloc_scratch` itself to a
// kernel (on the host it names a host-side stand-in); it passes the device
// address that cudaGetSymbolAddress returns for the current device.
static __device__ __align__(256) unsigned char g_noalloc_scratch[HGA_NOALLOC_SCRATCH_BYTES];

namespace {

constexpr int kMaxDevices = 64;

// Device address of g_noalloc_scratch on the current device, looked up once
// per device (with that device current) and cached; nullptr on failure.
void* noalloc_scratch() {
  static std::mutex mu;
  static void* addr[kMaxDevices] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (!addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess) return nullptr;
    addr[dev] = p;
  }
  return addr[dev];
}

}  // namespace

extern "C" {

const char* hga_version(void) { return "libhga 0.1 (sm_100a)"; }

const char* hga_last_cuda_error(void) { return cudaGetErrorName(last_launch_error()); }

const char* hga_status_string(hga_status_t s) {
  switch (s) {
    case HGA_OK: return "ok";
    case HGA_ERR_INVALID_ARG: return "invalid argument";
    case HGA_ERR_UNSUPPORTED: return "unsupported configuration";
    case HGA_ERR_CUDA: return "CUDA error";
    case HGA_ERR_TIMEOUT: return "device wait timed out";
    case HGA_ERR_DEVICE_CHECK: return "device-side index check failed";
    case HGA_ERR_WORKSPACE: return "workspace too small";
    case HGA_ERR_IO: return "tier file read or write failed";
  }
  return "unknown status";
}

hga_status_t hga_build_summaries(const hga_config_t* cfg, const void* k, int64_t ctx_cap,
                                 int64_t t_begin, int64_t t_end, float* gsum, float* bsum,
                                 void* stream) {
  hga_status_t st = check_cfg(cfg);
  if (st != HGA_OK) return st;
  if (!k || !gsum || !bsum || !aligned16(k) || !aligned16(gsum) || !aligned16(bsum))
    return HGA_ERR_INVALID_ARG;
  if (ctx_cap <= 0 || ctx_cap % kBlock || t_begin < 0 || t_begin % kBlock || t_end % kBlock ||
      t_end < t_begin || t_end > ctx_cap)
    return HGA_ERR_INVALID_ARG;
  if (t_end == t_begin) return HGA_OK;
  const int64_t n_blk = (t_end - t_begin) / kBlock;
  if (n_blk > 0x7fffffff) return HGA_ERR_UNSUPPORTED;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  return dispatch(cfg, [&]<typename T, int D>() -> hga_status_t {
    dim3 grid(unsigned(n_blk), cfg->n_kv_heads, cfg->batch);
    return traced_launch(HGA_K_SUMMARIES, s, [&] {
      return launch_pdl(summaries_kernel<T, D>, grid, dim3(D), 0, s, static_cast<const T*>(k),
          ctx_cap, t_begin, ctx_cap, t_begin / kBlock, cfg->n_kv_heads, gsum, bsum);
    });
  });
}

hga_status_t hga_build_summaries_seg(const hga_config_t* cfg, const void* k_seg, int64_t seg_cap,
                                     int64_t t_begin, int64_t t_end, int64_t ctx_cap,
                                     float* gsum, float* bsum, void* stream) {
  hga_status_t st = check_cfg(cfg);
  if (st != HGA_OK) return st;
  if (!k_seg || !gsum || !bsum || !aligned16(k_seg) || !aligned16(gsum) || !aligned16(bsum))
    return HGA_ERR_INVALID_ARG;
  if (ctx_cap <= 0 || ctx_cap % kBlock || t_begin < 0 || t_begin % kBlock || t_end % kBlock ||
      t_end < t_begin || t_end > ctx_cap || seg_cap < t_end - t_begin)
    return HGA_ERR_INVALID_ARG;
  if (t_end == t_begin) return HGA_OK;
  const int64_t n_blk = (t_end - t_begin) / kBlock;
  if (n_blk > 0x7fffffff) return HGA_ERR_UNSUPPORTED;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  return dispatch(cfg, [&]<typename T, int D>() -> hga_status_t {
    dim3 grid(unsigned(n_blk), cfg->n_kv_heads, cfg->batch);
    return traced_launch(HGA_K_SUMMARIES, s, [&] {
      return launch_pdl(summaries_kernel<T, D>, grid, dim3(D), 0, s, static_cast<const T*>(k_seg),
          seg_cap, 0, ctx_cap, t_begin / kBlock, cfg->n_kv_heads, gsum, bsum);
    });
  });
}

size_t hga_route_workspace_size(const hga_config_t* cfg, int32_t s_len, int64_t q_begin) {
  if (check_cfg(cfg) != HGA_OK || s_len <= 0 || q_begin < 0) return 0;
  return route_carve(cfg, s_len, q_begin, nullptr).bytes;
}

// The routing of hga_route.  With `done`, a fused routing launch also stores
// `token` into done[item] once item's selections are written (chained
// segment call); the three-launch path ignores it.
static hga_status_t route_impl(const hga_config_t* cfg, const void* q, int64_t q_begin,
                               int32_t s_len, int64_t ctx_cap, const float* bsum,
                               const float* gsum, int32_t* sel_blk, int32_t* sel_grp,
                               void* workspace, size_t ws_bytes, int* done, uint32_t token,
                               cudaStream_t s, const float* qprev = nullptr,
                               int qshift = 1, float* scores_out = nullptr) {
  hga_status_t st = check_cfg(cfg);
  if (st != HGA_OK) return st;
  if ((st = check_segment(ctx_cap, q_begin, s_len)) != HGA_OK) return st;
  if ((!q && !qprev) || !bsum || !gsum || !sel_grp || !workspace) return HGA_ERR_INVALID_ARG;
  if ((q && !aligned16(q)) || !aligned16(bsum) || !aligned16(gsum) || !aligned16(sel_grp) ||
      !aligned16(workspace) || (sel_blk && !aligned16(sel_blk)) ||
      (scores_out && !aligned16(scores_out)))
    return HGA_ERR_INVALID_ARG;
  RouteCarve ws = route_carve(cfg, s_len, q_begin, workspace);
  if (ws_bytes < ws.bytes) return HGA_ERR_WORKSPACE;
  const int n_qb = s_len / kQBlock;
  const int64_t own0 = q_begin / kBlock;
  const int64_t j_max = own0 + n_qb - 1;
  return dispatch(cfg, [&]<typename T, int D>() -> hga_status_t {
    if (j_max <= kFusedRouteMaxBlocks) {
      // the whole routing in one launch (every CTA reads all J block summaries)
      dim3 g1(n_qb, cfg->n_kv_heads, cfg->batch);
      const size_t smf = fused_route_smem<D>(own0 + n_qb, cfg->topk_blocks);
      hga_status_t e = ensure_smem(reinterpret_cast<const void*>(&route_fused_kernel<T, D>), smf);
      if (e != HGA_OK) return e;
      return traced_launch(HGA_K_ROUTE_FUSED, s, [&] {
        return launch_pdl(route_fused_kernel<T, D>, g1, dim3(kRouteThreads), smf, s,
                          static_cast<const T*>(q), bsum, gsum, ctx_cap, cfg->n_q_heads,
                          cfg->n_kv_heads, s_len, own0, cfg->topk_blocks, cfg->topk_groups,
                          sel_blk, sel_grp, done, token, qprev, qshift, cfg->scale,
                          scores_out);
      });
    }
    // three launches: q-bar (unless it comes from the resident block means),
    // the chunks' scores and finalists, the merge and level 2
    hga_status_t e = HGA_OK;
    if (!qprev) {
      dim3 g0(n_qb, cfg->n_kv_heads, cfg->batch);
      e = traced_launch(HGA_K_QBAR, s, [&] {
        return launch_pdl(qbar_kernel<T, D>, g0, dim3(kRouteThreads), 0, s,
            static_cast<const T*>(q), cfg->n_q_heads, cfg->n_kv_heads, s_len, ws.qbar);
      });
      if (e != HGA_OK) return e;
    }
    const float* qsrc = qprev ? qprev : ws.qbar;
    const int shift = qprev ? qshift : 0;
    const float* qpart = qprev ? nullptr : ws.qbar;
    if (j_max > 0) {
      // the query blocks split over CTAs of at most 32 each (splitting
      // further measured slower: the CTAs are not short of SMs)
      const int n_split = (n_qb + 31) / 32;
      const int nq_max = (n_qb + n_split - 1) / n_split;
      const size_t sm2 = chunk_layout(nq_max, D).total;
      e = ensure_smem(reinterpret_cast<const void*>(&block_topk_kernel<D>), sm2);
      if (e != HGA_OK) return e;
      dim3 g2(unsigned(ws.n_chunks), cfg->n_kv_heads, cfg->batch * n_split);
      e = traced_launch(HGA_K_BLOCK_TOPK, s, [&] {
        return launch_pdl(block_topk_kernel<D>, g2, dim3(kChunkThreads), sm2, s, qpart,
            qprev ? qsrc : nullptr, shift, bsum, ctx_cap, cfg->n_kv_heads, n_qb, own0,
            cfg->topk_blocks, n_split, nq_max, ws.fin_key, ws.fin_idx);
      });
      if (e != HGA_OK) return e;
    }
    dim3 g1(n_qb, cfg->n_kv_heads, cfg->batch);
    const size_t sm3 = merge_layout(ws.n_chunks, cfg->topk_blocks, D).total;
    e = ensure_smem(reinterpret_cast<const void*>(&select_kernel<D>), sm3);
    if (e != HGA_OK) return e;
    return traced_launch(HGA_K_SELECT, s, [&] {
      return launch_pdl(select_kernel<D>, g1, dim3(kRouteThreads), sm3, s, qpart,
          qprev ? qsrc : nullptr, shift, ws.fin_key, ws.fin_idx, ws.n_chunks, gsum, ctx_cap,
          cfg->n_kv_heads, n_qb, own0, cfg->topk_blocks, cfg->topk_groups, sel_blk, sel_grp,
          cfg->scale, scores_out);
    });
  });
}

// whether route_impl takes the one-launch path
static bool route_fused(int64_t q_begin, int32_t s_len) {
  return q_begin / kBlock + s_len / kQBlock - 1 <= kFusedRouteMaxBlocks;
}

hga_status_t hga_route(const hga_config_t* cfg, const void* q, int64_t q_begin, int32_t s_len,
                       int64_t ctx_cap, const float* bsum, const float* gsum, int32_t* sel_blk,
                       int32_t* sel_grp, float* scores_out, void* workspace, size_t ws_bytes,
                       void* stream) {
  return route_impl(cfg, q, q_begin, s_len, ctx_cap, bsum, gsum, sel_blk, sel_grp, workspace,
                    ws_bytes, nullptr, 0, static_cast<cudaStream_t>(stream), nullptr, 1,
                    scores_out);
}

hga_status_t hga_attn_fwd(const hga_config_t* cfg, const void* q, const void* k, const void* v,
                          int64_t ctx_cap, int64_t q_begin, int32_t s_len,
                          const int32_t* sel_grp, void* o, float* lse, void* stream) {
  hga_status_t st = check_cfg(cfg);
  if (st != HGA_OK) return st;
  if ((st = check_segment(ctx_cap, q_begin, s_len)) != HGA_OK) return st;
  if (!q || !k || !v || !sel_grp || !o || !lse) return HGA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(sel_grp) || !aligned16(o) ||
      !aligned16(lse))
    return HGA_ERR_INVALID_ARG;
  const int n_qb = s_len / kQBlock;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (use_tensor_cores(cfg, ctx_cap, s_len)) {
    if ((cfg->n_q_heads / cfg->n_kv_heads) % 4 == 0)
      return launch_fwd_tc<2>(cfg, q, k, v, ctx_cap, q_begin, s_len, sel_grp, o, lse, nullptr,
                              nullptr, 0, s);
    return launch_fwd_tc<1>(cfg, q, k, v, ctx_cap, q_begin, s_len, sel_grp, o, lse, nullptr,
                            nullptr, 0, s);
  }
  return dispatch(cfg, [&]<typename T, int D>() -> hga_status_t {
    const size_t sm = size_t(simt_fwd_smem_floats<D>()) * 4;
    hga_status_t e =
        ensure_smem(reinterpret_cast<const void*>(&attn_fwd_simt_kernel<T, D>), sm);
    if (e != HGA_OK) return e;
    dim3 grid(n_qb, cfg->n_q_heads, cfg->batch);
    return traced_launch(HGA_K_FWD_SIMT, s, [&] {
      attn_fwd_simt_kernel<T, D><<<grid, kSimtFwdThreads, sm, s>>>(
          static_cast<const T*>(q), static_cast<const T*>(k), static_cast<const T*>(v), ctx_cap,
          q_begin, s_len, cfg->n_q_heads, cfg->n_kv_heads, cfg->topk_groups, sel_grp,
          cfg->scale, static_cast<T*>(o), lse);
    });
  });
}

hga_status_t hga_route_noalloc(const hga_config_t* cfg, const void* q, int64_t q_begin,
                               int32_t s_len, int64_t ctx_cap, const float* bsum,
                               const float* gsum, int32_t* sel_blk, int32_t* sel_grp,
                               void* stream) {
  hga_status_t st = check_cfg(cfg);
  if (st != HGA_OK) return st;
  if ((st = check_segment(ctx_cap, q_begin, s_len)) != HGA_OK) return st;
  if (hga_route_workspace_size(cfg, s_len, q_begin) > HGA_NOALLOC_SCRATCH_BYTES)
    return HGA_ERR_WORKSPACE;
  void* scratch = noalloc_scratch();
  if (!scratch) return HGA_ERR_CUDA;
  return hga_route(cfg, q, q_begin, s_len, ctx_cap, bsum, gsum, sel_blk, sel_grp, nullptr,
                   scratch, HGA_NOALLOC_SCRATCH_BYTES, stream);
}

// backward workspace, 256-byte aligned sections: D = rowsum(dO * O)
// [B, Hq, S] fp32; the work-unit counter of the persistent dK/dV kernel;
// the per-item completion flags of a fused forward + backward, forward
// items then dQ items, [B, Hkv, S/64] int32 each
static size_t bwd_dvec_bytes(const hga_config_t* cfg, int32_t s_len) {
  return align256(size_t(cfg->batch) * cfg->n_q_heads * size_t(s_len) * 4);
}
static size_t bwd_flag_bytes(const hga_config_t* cfg, int32_t s_len) {
  return align256(size_t(cfg->batch) * cfg->n_kv_heads * size_t(s_len / kQBlock) * 4);
}
// the inverted selection the dQ kernel writes for the dK/dV kernel,
// [B, Hkv, S/64 key blocks, S/64 query blocks] int32
static size_t bwd_inv_bytes(const hga_config_t* cfg, int32_t s_len) {
  const size_t n = size_t(s_len / kQBlock);
  return align256(size_t(cfg->batch) * cfg->n_kv_heads * n * n * 4);
}

// [D][work counter (256 B)][forward flags][dQ flags][inverted selection]
struct BwdCarve {
  float* dvec;
  int* unit_counter;
  int* fwd_done;
  int* d_done;
  int* inv;
};

static BwdCarve bwd_carve(const hga_config_t* cfg, int32_t s_len, void* workspace) {
  char* ws = static_cast<char*>(workspace);
  BwdCarve c;
  c.dvec = reinterpret_cast<float*>(ws);
  ws += bwd_dvec_bytes(cfg, s_len);
  c.unit_counter = reinterpret_cast<int*>(ws);
  ws += 256;
  c.fwd_done = reinterpret_cast<int*>(ws);
  ws += bwd_flag_bytes(cfg, s_len);
  c.d_done = reinterpret_cast<int*>(ws);
  ws += bwd_flag_bytes(cfg, s_len);
  c.inv = reinterpret_cast<int*>(ws);
  return c;
}

size_t hga_attn_bwd_workspace_size(const hga_config_t* cfg, int32_t s_len) {
  if (check_cfg(cfg) != HGA_OK || s_len <= 0) return 0;
  return bwd_dvec_bytes(cfg, s_len) + 256 + 2 * bwd_flag_bytes(cfg, s_len) +
         bwd_inv_bytes(cfg, s_len);
}

hga_status_t hga_attn_bwd(const hga_config_t* cfg, const void* q, const void* k, const void* v,
                          int64_t ctx_cap, int64_t q_begin, int32_t s_len,
                          const int32_t* sel_grp, const void* o, const float* lse,
                          const void* d_o, void* dq, void* dk, void* dv, void* workspace,
                          size_t ws_bytes, void* stream) {
  hga_status_t st = check_cfg(cfg);
  if (st != HGA_OK) return st;
  if ((st = check_segment(ctx_cap, q_begin, s_len)) != HGA_OK) return st;
  const void* ptrs[] = {q, k, v, sel_grp, o, lse, d_o, dq, dk, dv, workspace};
  for (const void* p : ptrs)
    if (!p || !aligned16(p)) return HGA_ERR_INVALID_ARG;
  if (ws_bytes < hga_attn_bwd_workspace_size(cfg, s_len)) return HGA_ERR_WORKSPACE;
  const int n_qb = s_len / kQBlock;
  const BwdCarve wc = bwd_carve(cfg, s_len, workspace);
  float* dvec = wc.dvec;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (use_tensor_cores(cfg, ctx_cap, s_len)) {
    if (cfg->n_q_heads / cfg->n_kv_heads == 4)
      return launch_bwd_tc<2>(cfg, q, k, v, ctx_cap, q_begin, s_len, sel_grp, o, lse, d_o, dq,
                              dk, dv, dvec, wc.unit_counter, nullptr, nullptr, 0, wc.inv, s);
    return launch_bwd_tc<1>(cfg, q, k, v, ctx_cap, q_begin, s_len, sel_grp, o, lse, d_o, dq, dk,
                            dv, dvec, wc.unit_counter, nullptr, nullptr, 0, wc.inv, s);
  }
  return dispatch(cfg, [&]<typename T, int D>() -> hga_status_t {
    const size_t sm1 = size_t(simt_fwd_smem_floats<D>()) * 4;
    hga_status_t e =
        ensure_smem(reinterpret_cast<const void*>(&attn_bwd_dq_simt_kernel<T, D>), sm1);
    if (e != HGA_OK) return e;
    dim3 g1(n_qb, cfg->n_q_heads, cfg->batch);
    e = traced_launch(HGA_K_BWD_DQ_SIMT, s, [&] {
      attn_bwd_dq_simt_kernel<T, D><<<g1, kSimtFwdThreads, sm1, s>>>(
          static_cast<const T*>(q), static_cast<const T*>(k), static_cast<const T*>(v), ctx_cap,
          q_begin, s_len, cfg->n_q_heads, cfg->n_kv_heads, cfg->topk_groups, sel_grp,
          cfg->scale, static_cast<const T*>(o), lse, static_cast<const T*>(d_o),
          static_cast<T*>(dq), dvec);
    });
    if (e != HGA_OK) return e;
    const size_t sm2 = size_t(simt_kv_smem_floats<D>()) * 4;
    e = ensure_smem(reinterpret_cast<const void*>(&attn_bwd_dkdv_simt_kernel<T, D>), sm2);
    if (e != HGA_OK) return e;
    dim3 g2(n_qb, cfg->n_kv_heads, cfg->batch);
    return traced_launch(HGA_K_BWD_DKDV_SIMT, s, [&] {
      attn_bwd_dkdv_simt_kernel<T, D><<<g2, kSimtKvThreads, sm2, s>>>(
          static_cast<const T*>(q), static_cast<const T*>(k), static_cast<const T*>(v), ctx_cap,
          q_begin, s_len, cfg->n_q_heads, cfg->n_kv_heads, cfg->topk_groups, sel_grp,
          cfg->scale, lse, static_cast<const T*>(d_o), dvec, static_cast<T*>(dk),
          static_cast<T*>(dv));
    });
  });
}

static uint32_t next_call_token() {
  // a fresh token per chained call: flags left by earlier calls never match
  static std::atomic<uint32_t> next{0};
  uint32_t token = ++next;
  if (token == 0) token = ++next;
  return token;
}

// hga_attn_fwd_bwd on a checked configuration; with route_done, the forward
// waits for each item's routing flag instead of the whole routing grid
static hga_status_t fwd_bwd_impl(const hga_config_t* cfg, const void* q, const void* k,
                                 const void* v, int64_t ctx_cap, int64_t q_begin, int32_t s_len,
                                 const int32_t* sel_grp, void* o, float* lse, const void* d_o,
                                 void* dq, void* dk, void* dv, void* workspace, size_t ws_bytes,
                                 const int* route_done, uint32_t token, cudaStream_t s) {
  if (!use_tensor_cores(cfg, ctx_cap, s_len)) {
    hga_status_t st = hga_attn_fwd(cfg, q, k, v, ctx_cap, q_begin, s_len, sel_grp, o, lse, s);
    if (st != HGA_OK) return st;
    return hga_attn_bwd(cfg, q, k, v, ctx_cap, q_begin, s_len, sel_grp, o, lse, d_o, dq, dk, dv,
                        workspace, ws_bytes, s);
  }
  const BwdCarve wc = bwd_carve(cfg, s_len, workspace);
  float* dvec = wc.dvec;
  int* unit_counter = wc.unit_counter;
  int* fwd_done = wc.fwd_done;
  int* d_done = wc.d_done;
  hga_status_t st;
  if (cfg->n_q_heads / cfg->n_kv_heads == 4) {
    st = launch_fwd_tc<2>(cfg, q, k, v, ctx_cap, q_begin, s_len, sel_grp, o, lse, route_done,
                          fwd_done, token, s);
    if (st != HGA_OK) return st;
    return launch_bwd_tc<2>(cfg, q, k, v, ctx_cap, q_begin, s_len, sel_grp, o, lse, d_o, dq, dk,
                            dv, dvec, unit_counter, fwd_done, d_done, token, wc.inv, s);
  }
  st = launch_fwd_tc<1>(cfg, q, k, v, ctx_cap, q_begin, s_len, sel_grp, o, lse, route_done,
                        fwd_done, token, s);
  if (st != HGA_OK) return st;
  return launch_bwd_tc<1>(cfg, q, k, v, ctx_cap, q_begin, s_len, sel_grp, o, lse, d_o, dq, dk,
                          dv, dvec, unit_counter, fwd_done, d_done, token, wc.inv, s);
}

static hga_status_t check_fwd_bwd_args(const hga_config_t* cfg, int64_t ctx_cap, int64_t q_begin,
                                       int32_t s_len, std::initializer_list<const void*> ptrs) {
  hga_status_t st = check_cfg(cfg);
  if (st != HGA_OK) return st;
  if ((st = check_segment(ctx_cap, q_begin, s_len)) != HGA_OK) return st;
  for (const void* p : ptrs)
    if (!p || !aligned16(p)) return HGA_ERR_INVALID_ARG;
  return HGA_OK;
}

hga_status_t hga_attn_fwd_bwd(const hga_config_t* cfg, const void* q, const void* k,
                              const void* v, int64_t ctx_cap, int64_t q_begin, int32_t s_len,
                              const int32_t* sel_grp, void* o, float* lse, const void* d_o,
                              void* dq, void* dk, void* dv, void* workspace, size_t ws_bytes,
                              void* stream) {
  hga_status_t st = check_fwd_bwd_args(cfg, ctx_cap, q_begin, s_len,
                                       {q, k, v, sel_grp, o, lse, d_o, dq, dk, dv, workspace});
  if (st != HGA_OK) return st;
  if (ws_bytes < hga_attn_bwd_workspace_size(cfg, s_len)) return HGA_ERR_WORKSPACE;
  return fwd_bwd_impl(cfg, q, k, v, ctx_cap, q_begin, s_len, sel_grp, o, lse, d_o, dq, dk, dv,
                      workspace, ws_bytes, nullptr, next_call_token(),
                      static_cast<cudaStream_t>(stream));
}

size_t hga_segment_workspace_size(const hga_config_t* cfg, int32_t s_len, int64_t q_begin) {
  if (check_cfg(cfg) != HGA_OK || s_len <= 0 || q_begin < 0) return 0;
  return hga_attn_bwd_workspace_size(cfg, s_len) + bwd_flag_bytes(cfg, s_len) +
         align256(hga_route_workspace_size(cfg, s_len, q_begin));
}

hga_status_t hga_segment_fwd_bwd(const hga_config_t* cfg, const void* q, const void* k,
                                 const void* v, int64_t ctx_cap, int64_t q_begin, int32_t s_len,
                                 const float* bsum, const float* gsum, int32_t* sel_blk,
                                 int32_t* sel_grp, void* o, float* lse, const void* d_o, void* dq,
                                 void* dk, void* dv, void* workspace, size_t ws_bytes,
                                 void* stream) {
  hga_status_t st = check_fwd_bwd_args(
      cfg, ctx_cap, q_begin, s_len,
      {q, k, v, bsum, gsum, sel_grp, o, lse, d_o, dq, dk, dv, workspace});
  if (st != HGA_OK) return st;
  if (sel_blk && !aligned16(sel_blk)) return HGA_ERR_INVALID_ARG;
  if (ws_bytes < hga_segment_workspace_size(cfg, s_len, q_begin)) return HGA_ERR_WORKSPACE;
  // workspace: [backward workspace][routing flags][routing workspace]
  const size_t bwd_bytes = hga_attn_bwd_workspace_size(cfg, s_len);
  char* ws = static_cast<char*>(workspace);
  int* route_done = reinterpret_cast<int*>(ws + bwd_bytes);
  char* route_ws = ws + bwd_bytes + bwd_flag_bytes(cfg, s_len);
  const size_t route_bytes = ws_bytes - bwd_bytes - bwd_flag_bytes(cfg, s_len);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const uint32_t token = next_call_token();
  const bool chain = use_tensor_cores(cfg, ctx_cap, s_len) && route_fused(q_begin, s_len);
  st = route_impl(cfg, q, q_begin, s_len, ctx_cap, bsum, gsum, sel_blk, sel_grp, route_ws,
                  route_bytes, chain ? route_done : nullptr, token, s);
  if (st != HGA_OK) return st;
  return fwd_bwd_impl(cfg, q, k, v, ctx_cap, q_begin, s_len, sel_grp, o, lse, d_o, dq, dk, dv,
                      workspace, bwd_bytes, chain ? route_done : nullptr, token, s);
}

namespace {

int64_t tier_slot_cap(const hga_config_t* cfg, int64_t q_begin, int32_t s_len) {
  const int64_t by_sel = int64_t(s_len / kQBlock) * cfg->topk_groups;
  const int64_t by_hist = q_begin / kGroup;
  return by_sel < by_hist ? by_sel : by_hist;
}

// Device address of pinned, device-mapped host memory (nullptr otherwise).
const void* mapped_host(const void* p) {
  cudaPointerAttributes a;
  if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
    cudaGetLastError();
    return nullptr;
  }
  if (a.type != cudaMemoryTypeHost || a.devicePointer == nullptr) return nullptr;
  return a.devicePointer;
}

}  // namespace

size_t hga_tier_workspace_size(const hga_config_t* cfg, int32_t s_len, int64_t q_begin) {
  if (check_cfg(cfg) != HGA_OK || s_len <= 0 || q_begin < 0) return 0;
  const int64_t heads = int64_t(cfg->batch) * cfg->n_kv_heads;
  const int64_t cap = tier_slot_cap(cfg, q_begin, s_len);
  return align256(size_t(heads) * 4) + align256(size_t(heads * (cap > 0 ? cap : 1)) * 4);
}

int64_t hga_tier_stage_rows(const hga_config_t* cfg, int64_t q_begin, int32_t s_len) {
  if (check_cfg(cfg) != HGA_OK || s_len <= 0 || q_begin < 0) return 0;
  const int64_t hist_rows = tier_slot_cap(cfg, q_begin, s_len) * kGroup;
  return ((hist_rows + kBlock - 1) / kBlock) * kBlock + s_len;
}

hga_status_t hga_tier_gather(const hga_config_t* cfg, const void* k_host, const void* v_host,
                             int64_t ctx_cap, int64_t q_begin, int32_t s_len,
                             const int32_t* sel_grp, void* k_stage, void* v_stage,
                             int64_t stage_cap, int32_t* sel_stage, int32_t* n_unique,
                             void* workspace, size_t ws_bytes, void* stream) {
  hga_status_t st = check_cfg(cfg);
  if (st != HGA_OK) return st;
  if ((st = check_segment(ctx_cap, q_begin, s_len)) != HGA_OK) return st;
  const void* ptrs[] = {k_host, v_host, sel_grp, k_stage, v_stage, sel_stage, workspace};
  for (const void* p : ptrs)
    if (!p || !aligned16(p)) return HGA_ERR_INVALID_ARG;
  if (stage_cap % kBlock || stage_cap < hga_tier_stage_rows(cfg, q_begin, s_len))
    return HGA_ERR_INVALID_ARG;
  if (ws_bytes < hga_tier_workspace_size(cfg, s_len, q_begin)) return HGA_ERR_WORKSPACE;
  const void* kd = mapped_host(k_host);
  const void* vd = mapped_host(v_host);
  if (!kd || !vd) return HGA_ERR_INVALID_ARG;  // not pinned, device-mapped host memory
  const int64_t heads = int64_t(cfg->batch) * cfg->n_kv_heads;
  int32_t* counts = static_cast<int32_t*>(workspace);
  int32_t* slots = reinterpret_cast<int32_t*>(static_cast<char*>(workspace) +
                                              align256(size_t(heads) * 4));
  if (n_unique == nullptr) n_unique = counts;
  const int64_t slot_cap = tier_slot_cap(cfg, q_begin, s_len) > 0
                               ? tier_slot_cap(cfg, q_begin, s_len) : 1;
  const int n_qb = s_len / kQBlock;
  const int64_t n_words = (q_begin / kGroup + 31) / 32;
  const size_t sm = size_t(n_words > 0 ? n_words : 1) * 8;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  return dispatch(cfg, [&]<typename T, int D>() -> hga_status_t {
    hga_status_t e = ensure_smem(reinterpret_cast<const void*>(&tier_dedup_kernel<D>), sm);
    if (e != HGA_OK) return e;
    dim3 g1(cfg->n_kv_heads, cfg->batch);
    e = traced_launch(HGA_K_TIER_DEDUP, s, [&] {
      tier_dedup_kernel<D><<<g1, kTierThreads, sm, s>>>(sel_grp, cfg->n_kv_heads, n_qb,
                                                        cfg->topk_groups, q_begin, stage_cap,
                                                        s_len, sel_stage, slots, n_unique,
                                                        slot_cap);
    });
    if (e != HGA_OK || q_begin == 0) return e;
    const int per_cta = 8 * kTierCopyWarps;
    dim3 g2(unsigned((slot_cap + per_cta - 1) / per_cta), cfg->n_kv_heads, cfg->batch);
    return traced_launch(HGA_K_TIER_COPY, s, [&] {
      tier_copy_kernel<T, D><<<g2, kTierCopyWarps * 32, 0, s>>>(
          static_cast<const T*>(kd), static_cast<const T*>(vd), ctx_cap, cfg->n_kv_heads, slots,
          n_unique, slot_cap, static_cast<T*>(k_stage), static_cast<T*>(v_stage), stage_cap);
    });
  });
}

hga_status_t hga_tier_append(const hga_config_t* cfg, const void* k_stage, const void* v_stage,
                             int64_t stage_cap, void* k_host, void* v_host, int64_t ctx_cap,
                             int64_t q_begin, int32_t s_len, void* stream) {
  hga_status_t st = check_cfg(cfg);
  if (st != HGA_OK) return st;
  if ((st = check_segment(ctx_cap, q_begin, s_len)) != HGA_OK) return st;
  if (!k_stage || !v_stage || !k_host || !v_host || stage_cap < s_len || stage_cap % kBlock)
    return HGA_ERR_INVALID_ARG;
  if (!mapped_host(k_host) || !mapped_host(v_host)) return HGA_ERR_INVALID_ARG;
  const size_t elt = cfg->dtype == HGA_BF16 ? 2 : 4;
  const size_t row = size_t(cfg->head_dim) * elt;
  const size_t heads = size_t(cfg->batch) * cfg->n_kv_heads;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const void* srcs[2] = {k_stage, v_stage};
  void* dsts[2] = {k_host, v_host};
  for (int i = 0; i < 2; ++i) {
    const char* src = static_cast<const char*>(srcs[i]) + size_t(stage_cap - s_len) * row;
    char* dst = static_cast<char*>(dsts[i]) + size_t(q_begin) * row;
    if (cudaMemcpy2DAsync(dst, size_t(ctx_cap) * row, src, size_t(stage_cap) * row,
                          size_t(s_len) * row, heads, cudaMemcpyDeviceToHost, s) != cudaSuccess)
      return HGA_ERR_CUDA;
  }
  return HGA_OK;
}

hga_status_t hga_get_device_status(void* stream) {
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) return HGA_ERR_CUDA;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_device_status, sizeof(int)) != cudaSuccess) return HGA_ERR_CUDA;
  const int zero = 0;
  if (cudaMemcpyToSymbol(g_device_status, &zero, sizeof(int)) != cudaSuccess) return HGA_ERR_CUDA;
  return static_cast<hga_status_t>(v);
}

const char* hga_kernel_name(int kind) {
  static const char* names[HGA_K_COUNT] = {
      "summaries",      "route_qbar",        "route_block_topk",    "route_select",
      "attn_fwd_simt",  "attn_bwd_dq_simt",  "attn_bwd_dkdv_simt",  "attn_fwd_tc",
      "attn_bwd_dq_tc", "attn_bwd_dkdv_tc",  "tier_dedup",          "tier_copy",
      "route_fused",    "decode",            "query_summaries",     "prepare"};
  return (kind >= 0 && kind < HGA_K_COUNT) ? names[kind] : "unknown";
}

uint64_t hga_launch_count(void) { return tracer().launches.load(); }

hga_status_t hga_timing_enable(int32_t slots) {
  Tracer& t = tracer();
  std::lock_guard<std::mutex> lock(t.mu);
  if (slots < 0) return HGA_ERR_INVALID_ARG;
  while (t.slots.size() < size_t(slots)) {
    TimingSlot ts;
    if (cudaEventCreate(&ts.begin) != cudaSuccess || cudaEventCreate(&ts.end) != cudaSuccess)
      return HGA_ERR_CUDA;
    t.slots.push_back(ts);
  }
  t.on = slots > 0;
  t.next = 0;
  return HGA_OK;
}

void hga_timing_kinds(uint32_t mask) {
  Tracer& t = tracer();
  std::lock_guard<std::mutex> lock(t.mu);
  t.kinds = mask;
}

hga_status_t hga_timing_collect(void) {
  Tracer& t = tracer();
  std::lock_guard<std::mutex> lock(t.mu);
  for (size_t i = 0; i < t.next; ++i) {
    TimingSlot& ts = t.slots[i];
    if (cudaEventSynchronize(ts.end) != cudaSuccess) return HGA_ERR_CUDA;
    float ms = 0.f;
    if (cudaEventElapsedTime(&ms, ts.begin, ts.end) != cudaSuccess) return HGA_ERR_CUDA;
    t.ms[ts.kind] += ms;
    t.count[ts.kind] += 1;
  }
  return HGA_OK;
}

hga_status_t hga_timing_get(int kind, double* ms, uint64_t* launches) {
  if (kind < 0 || kind >= HGA_K_COUNT || !ms || !launches) return HGA_ERR_INVALID_ARG;
  Tracer& t = tracer();
  std::lock_guard<std::mutex> lock(t.mu);
  *ms = t.ms[kind];
  *launches = t.count[kind];
  return HGA_OK;
}

void hga_timing_reset(void) {
  Tracer& t = tracer();
  std::lock_guard<std::mutex> lock(t.mu);
  for (int i = 0; i < HGA_K_COUNT; ++i) { t.ms[i] = 0.0; t.count[i] = 0; }
}

}  // extern "C"

namespace {

template <typename T, int D, int G>
hga_status_t launch_decode(const hga_config_t* cfg, const void* q, const void* k, const void* v,
                           int64_t ctx_cap, const int64_t* pos, const float* bsum,
                           const float* gsum, int32_t* sel_blk, int32_t* sel_grp, void* o,
                           float* lse, cudaStream_t s) {
  int dev = 0, optin = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess)
    return HGA_ERR_CUDA;
  // cluster size: enough CTAs to fill the GPU about once (two per SM), more
  // where one CTA's share of the candidate scores would not fit
  const int64_t heads = int64_t(cfg->batch) * cfg->n_kv_heads;
  int nc = dec::kMaxC;
  while (nc > 1 && heads * nc > 2 * int64_t(sm_count())) nc /= 2;
  auto plan = [&](int c, int64_t* share_cap, int* stage_units) {
    *share_cap = (ctx_cap / kBlock + c - 1) / c;
    const int per_cta = (kGroupsPerBlock + cfg->topk_groups + c - 1) / c;
    const int fit = int(dec::kStageBudget / (2 * dec::unit_bytes<T, D>()));
    *stage_units = std::max(dec::kMinStageUnits, std::min(per_cta, fit));
    return dec::smem_bytes<T, D, G>(*share_cap, *stage_units, c);
  };
  int64_t share_cap = 0;
  int stage_units = 0;
  size_t smem = plan(nc, &share_cap, &stage_units);
  while (smem > size_t(optin) && nc < dec::kMaxC) smem = plan(nc *= 2, &share_cap, &stage_units);
  if (smem > size_t(optin)) return HGA_ERR_UNSUPPORTED;
  hga_status_t e = ensure_smem(reinterpret_cast<const void*>(&dec::decode_kernel<T, D, G>), smem);
  if (e != HGA_OK) return e;
  const float scale_log2 = cfg->scale * 1.4426950408889634f;
  return traced_launch(HGA_K_DECODE, s, [&] {
    cudaLaunchConfig_t lc = {};
    lc.gridDim = dim3(unsigned(nc), cfg->n_kv_heads, cfg->batch);
    lc.blockDim = dim3(dec::kThreads);
    lc.dynamicSmemBytes = smem;
    lc.stream = s;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = unsigned(nc);
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    lc.attrs = attr;
    lc.numAttrs = 2;
    return cudaLaunchKernelEx(&lc, dec::decode_kernel<T, D, G>, static_cast<const T*>(q),
        static_cast<const T*>(k), static_cast<const T*>(v), ctx_cap, pos, bsum, gsum,
        int(cfg->n_kv_heads), int(cfg->topk_blocks), int(cfg->topk_groups), scale_log2,
        share_cap, stage_units, sel_blk, sel_grp, static_cast<T*>(o), lse);
  });
}

}  // namespace

extern "C" hga_status_t hga_decode(const hga_config_t* cfg, const void* q, const void* k,
                                   const void* v, int64_t ctx_cap, const int64_t* pos,
                                   const float* bsum, const float* gsum, int32_t* sel_blk,
                                   int32_t* sel_grp, void* o, float* lse, void* stream) {
  hga_status_t st = check_cfg(cfg);
  if (st != HGA_OK) return st;
  if (!q || !k || !v || !pos || !bsum || !gsum || !o || !lse) return HGA_ERR_INVALID_ARG;
  for (const void* p : {q, k, v, static_cast<const void*>(pos), static_cast<const void*>(bsum),
                        static_cast<const void*>(gsum), static_cast<const void*>(sel_blk),
                        static_cast<const void*>(sel_grp), static_cast<const void*>(o),
                        static_cast<const void*>(lse)})
    if (p && !aligned16(p)) return HGA_ERR_INVALID_ARG;
  if (ctx_cap <= 0 || ctx_cap % kBlock) return HGA_ERR_INVALID_ARG;
  const int G = cfg->n_q_heads / cfg->n_kv_heads;
  if (G != 1 && G != 2 && G != 4 && G != 8) return HGA_ERR_UNSUPPORTED;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  return dispatch(cfg, [&]<typename T, int D>() -> hga_status_t {
    switch (G) {
      case 1: return launch_decode<T, D, 1>(cfg, q, k, v, ctx_cap, pos, bsum, gsum, sel_blk,
                                            sel_grp, o, lse, s);
      case 2: return launch_decode<T, D, 2>(cfg, q, k, v, ctx_cap, pos, bsum, gsum, sel_blk,
                                            sel_grp, o, lse, s);
      case 4: return launch_decode<T, D, 4>(cfg, q, k, v, ctx_cap, pos, bsum, gsum, sel_blk,
                                            sel_grp, o, lse, s);
      default: return launch_decode<T, D, 8>(cfg, q, k, v, ctx_cap, pos, bsum, gsum, sel_blk,
                                             sel_grp, o, lse, s);
    }
  });
}

static hga_status_t launch_qsum(const hga_config_t* cfg, const void* q, int64_t q_begin,
                                int32_t s_len, int64_t ctx_cap, float* qsum, cudaStream_t s) {
  return dispatch(cfg, [&]<typename T, int D>() -> hga_status_t {
    dim3 grid(s_len / kQBlock, cfg->n_kv_heads, cfg->batch);
    return traced_launch(HGA_K_QSUM, s, [&] {
      return launch_pdl(qsum_kernel<T, D>, grid, dim3(kRouteThreads), 0, s,
                        static_cast<const T*>(q), ctx_cap, cfg->n_q_heads, cfg->n_kv_heads, s_len,
                        q_begin / kBlock, qsum);
    });
  });
}

extern "C" hga_status_t hga_build_query_summaries(const hga_config_t* cfg, const void* q,
                                                  int64_t q_begin, int32_t s_len, int64_t ctx_cap,
                                                  float* qsum, void* stream) {
  hga_status_t st = check_cfg(cfg);
  if (st != HGA_OK) return st;
  if ((st = check_segment(ctx_cap, q_begin, s_len)) != HGA_OK) return st;
  if (!q || !qsum || !aligned16(q) || !aligned16(qsum)) return HGA_ERR_INVALID_ARG;
  return launch_qsum(cfg, q, q_begin, s_len, ctx_cap, qsum, static_cast<cudaStream_t>(stream));
}

extern "C" hga_status_t hga_route_causal(const hga_config_t* cfg, const void* q, int64_t q_begin,
                                         int32_t s_len, int64_t ctx_cap, const float* bsum,
                                         const float* gsum, float* qsum, int32_t* sel_blk,
                                         int32_t* sel_grp, void* workspace, size_t ws_bytes,
                                         void* stream) {
  hga_status_t st = check_cfg(cfg);
  if (st != HGA_OK) return st;
  if ((st = check_segment(ctx_cap, q_begin, s_len)) != HGA_OK) return st;
  if (!qsum || !aligned16(qsum)) return HGA_ERR_INVALID_ARG;
  if (!q || !bsum || !gsum || !sel_grp || !workspace) return HGA_ERR_INVALID_ARG;
  if (ws_bytes < route_carve(cfg, s_len, q_begin, nullptr).bytes) return HGA_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if ((st = launch_qsum(cfg, q, q_begin, s_len, ctx_cap, qsum, s)) != HGA_OK) return st;
  return route_impl(cfg, q, q_begin, s_len, ctx_cap, bsum, gsum, sel_blk, sel_grp, workspace,
                    ws_bytes, nullptr, 0, s, qsum);
}

extern "C" hga_status_t hga_prepare_segment(const hga_config_t* cfg, const void* q_proj,
                                            const void* k_proj, const void* v_proj,
                                            int64_t q_row_stride, int64_t kv_row_stride,
                                            int64_t q_begin, int32_t s_len,
                                            int64_t ctx_cap, float rope_base, void* q_out,
                                            void* k, void* v, float* gsum, float* bsum,
                                            float* qsum, void* stream) {
  hga_status_t st = check_cfg(cfg);
  if (st != HGA_OK) return st;
  if ((st = check_segment(ctx_cap, q_begin, s_len)) != HGA_OK) return st;
  for (const void* p : {q_proj, k_proj, v_proj, static_cast<const void*>(q_out),
                        static_cast<const void*>(k), static_cast<const void*>(v),
                        static_cast<const void*>(gsum), static_cast<const void*>(bsum),
                        static_cast<const void*>(qsum)})
    if (!p || !aligned16(p)) return HGA_ERR_INVALID_ARG;
  const size_t elt = cfg->dtype == HGA_BF16 ? 2 : 4;
  if (q_row_stride < int64_t(cfg->n_q_heads) * cfg->head_dim ||
      kv_row_stride < int64_t(cfg->n_kv_heads) * cfg->head_dim ||
      (size_t(q_row_stride) * elt) % 16 != 0 || (size_t(kv_row_stride) * elt) % 16 != 0)
    return HGA_ERR_INVALID_ARG;
  if (!(rope_base >= 0.f)) return HGA_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const double log2_base = rope_base > 1.f ? std::log2(double(rope_base)) : 0.0;
  return dispatch(cfg, [&]<typename T, int D>() -> hga_status_t {
    const size_t smem = sizeof(PrepShared<D>);
    hga_status_t e = ensure_smem(reinterpret_cast<const void*>(&prepare_kernel<T, D>), smem);
    if (e != HGA_OK) return e;
    dim3 grid(s_len / kQBlock, cfg->n_kv_heads, cfg->batch);
    return traced_launch(HGA_K_PREPARE, s, [&] {
      return launch_pdl(prepare_kernel<T, D>, grid, dim3(kPrepThreads), smem, s,
          static_cast<const T*>(q_proj), static_cast<const T*>(k_proj),
          static_cast<const T*>(v_proj), q_row_stride, kv_row_stride, q_begin, s_len, ctx_cap,
          cfg->n_q_heads,
          cfg->n_kv_heads, log2_base, static_cast<T*>(q_out), static_cast<T*>(k),
          static_cast<T*>(v), gsum, bsum, qsum);
    });
  });
}

extern "C" hga_status_t hga_route_summarized(const hga_config_t* cfg, int64_t q_begin,
                                             int32_t s_len, int64_t ctx_cap, const float* bsum,
                                             const float* gsum, const float* qsum, int32_t causal,
                                             int32_t* sel_blk, int32_t* sel_grp, void* workspace,
                                             size_t ws_bytes, void* stream) {
  if (!qsum || !aligned16(qsum) || (causal != 0 && causal != 1)) return HGA_ERR_INVALID_ARG;
  return route_impl(cfg, nullptr, q_begin, s_len, ctx_cap, bsum, gsum, sel_blk, sel_grp,
                    workspace, ws_bytes, nullptr, 0, static_cast<cudaStream_t>(stream), qsum,
                    causal);
}

extern "C" hga_status_t hga_tier_plan(const hga_config_t* cfg, int64_t q_begin, int32_t s_len,
                                      const int32_t* sel_grp, int64_t stage_cap,
                                      int32_t* sel_stage, int32_t* slot_group,
                                      int32_t* n_unique, int64_t slot_cap, void* stream) {
  hga_status_t st = check_cfg(cfg);
  if (st != HGA_OK) return st;
  if (q_begin < 0 || q_begin % kBlock || s_len <= 0 || s_len % kQBlock || s_len > kMaxSegment)
    return HGA_ERR_INVALID_ARG;
  if (!sel_grp || !sel_stage || !slot_group || !n_unique || !aligned16(sel_grp) ||
      !aligned16(sel_stage) || !aligned16(slot_group) || !aligned16(n_unique))
    return HGA_ERR_INVALID_ARG;
  if (stage_cap % kBlock || stage_cap < hga_tier_stage_rows(cfg, q_begin, s_len) ||
      slot_cap < std::max<int64_t>(tier_slot_cap(cfg, q_begin, s_len), 1))
    return HGA_ERR_INVALID_ARG;
  const int n_qb = s_len / kQBlock;
  const int64_t n_words = (q_begin / kGroup + 31) / 32;
  const size_t sm = size_t(n_words > 0 ? n_words : 1) * 8;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  return dispatch(cfg, [&]<typename T, int D>() -> hga_status_t {
    hga_status_t e = ensure_smem(reinterpret_cast<const void*>(&tier_dedup_kernel<D>), sm);
    if (e != HGA_OK) return e;
    dim3 g1(cfg->n_kv_heads, cfg->batch);
    return traced_launch(HGA_K_TIER_DEDUP, s, [&] {
      tier_dedup_kernel<D><<<g1, kTierThreads, sm, s>>>(sel_grp, cfg->n_kv_heads, n_qb,
                                                        cfg->topk_groups, q_begin, stage_cap,
                                                        s_len, sel_stage, slot_group, n_unique,
                                                        slot_cap);
    });
  });
}

extern "C" hga_status_t hga_tier_read_groups(const hga_config_t* cfg, int fd_k, int fd_v,
                                             int64_t ctx_cap, const int32_t* slot_group,
                                             const int32_t* n_unique, int64_t slot_cap,
                                             void* k_stage_host, void* v_stage_host,
                                             int64_t stage_cap, int32_t n_threads) {
  hga_status_t st = check_cfg(cfg);
  if (st != HGA_OK) return st;
  if (fd_k < 0 || fd_v < 0 || !slot_group || !n_unique || !k_stage_host || !v_stage_host ||
      ctx_cap <= 0 || ctx_cap % kBlock || slot_cap < 1 || stage_cap < 0 || n_threads < 1)
    return HGA_ERR_INVALID_ARG;
  const int64_t row = int64_t(cfg->head_dim) * (cfg->dtype == HGA_BF16 ? 2 : 4);
  const int64_t heads = int64_t(cfg->batch) * cfg->n_kv_heads;
  std::vector<file_tier::Run> runs;
  for (int64_t hd = 0; hd < heads; ++hd) {
    const int32_t U = n_unique[hd];
    if (U < 0 || U > slot_cap || int64_t(U) * kGroup > stage_cap) return HGA_ERR_INVALID_ARG;
    const int32_t* sg = slot_group + hd * slot_cap;
    for (int32_t u = 0; u < U;) {
      const int32_t g0 = sg[u];
      if (g0 < 0 || int64_t(g0 + 1) * kGroup > ctx_cap) return HGA_ERR_INVALID_ARG;
      int32_t n = 1;  // groups g0, g0+1, ... in slots u, u+1, ...: one transfer
      while (u + n < U && sg[u + n] == g0 + n) ++n;
      runs.push_back({(hd * ctx_cap + int64_t(g0) * kGroup) * row,
                      (hd * stage_cap + int64_t(u) * kGroup) * row, int64_t(n) * kGroup * row});
      u += n;
    }
  }
  return file_tier::transfer<false>(runs, fd_k, fd_v, static_cast<char*>(k_stage_host),
                                    static_cast<char*>(v_stage_host), n_threads)
             ? HGA_OK
             : HGA_ERR_IO;
}

extern "C" hga_status_t hga_tier_write_segment(const hga_config_t* cfg, int fd_k, int fd_v,
                                               int64_t ctx_cap, int64_t q_begin, int32_t s_len,
                                               const void* k_seg_host, const void* v_seg_host,
                                               int64_t seg_rows, int32_t n_threads) {
  hga_status_t st = check_cfg(cfg);
  if (st != HGA_OK) return st;
  if ((st = check_segment(ctx_cap, q_begin, s_len)) != HGA_OK) return st;
  if (fd_k < 0 || fd_v < 0 || !k_seg_host || !v_seg_host || seg_rows < s_len || n_threads < 1)
    return HGA_ERR_INVALID_ARG;
  const int64_t row = int64_t(cfg->head_dim) * (cfg->dtype == HGA_BF16 ? 2 : 4);
  const int64_t heads = int64_t(cfg->batch) * cfg->n_kv_heads;
  std::vector<file_tier::Run> runs;
  for (int64_t hd = 0; hd < heads; ++hd)
    runs.push_back({(hd * ctx_cap + q_begin) * row, hd * seg_rows * row, int64_t(s_len) * row});
  return file_tier::transfer<true>(runs, fd_k, fd_v,
                                   const_cast<char*>(static_cast<const char*>(k_seg_host)),
                                   const_cast<char*>(static_cast<const char*>(v_seg_host)),
                                   n_threads)
             ? HGA_OK
             : HGA_ERR_IO;
}
