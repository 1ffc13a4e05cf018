/*
 * libhga -- the data-parallel hot path of Hierarchical Global Attention (HGA)
 * on NVIDIA B200 (sm_100a).  C ABI: plain pointers, sizes and a CUDA stream
 * handle passed as void*.  No call allocates, frees or synchronises unless its
 * comment says so; every call is asynchronous on the given stream.
 *
 * Method sources (the HGA pages, all on "Long-Context Fine-Tuning with Limited
 * VRAM"):
 *   [A] adnankhan.ai notes "Long-Context Fine-Tuning with Limited VRAM",
 *       section "Raw Abstract / Excerpt": a bounded set of exact historical
 *       tokens per query block; only the active segment stays differentiable,
 *       older KV is detached.
 *   [B] seventnews "BMW如何通过重新设计注意力机制，在16 GB GPU上实现16K上下文",
 *       section "HGA的不同之处" (what HGA does differently): 64-token blocks
 *       with one compact summary each kept on the GPU; queries score the
 *       summaries and pick the top-k blocks; the blocks are opened at the level
 *       of 8-token groups; only the selected groups' exact-token K/V enter the
 *       attention; the router has no learned weights; summaries are never
 *       attention values; 2048-token segments with forward and backward per
 *       segment and no gradient across segment boundaries.
 *   [C] gist.science retelling, section "解决方案" (the solution): block
 *       summary cards and an 8-token group summary cache.
 *
 * Readings fixed here (the pages leave them open): a summary is the mean of
 * the post-RoPE keys of its block/group per KV head; a query block is 64
 * tokens; the routing score of a candidate is the mean over the query block's
 * 64 queries and the G = n_q_heads/n_kv_heads heads sharing the KV head of
 * q.s/sqrt(d); candidates of query block j are the complete blocks strictly
 * before its own block; level 2 ranks only the groups of the selected blocks;
 * ties go to the lower index; each query attends to the selected groups plus
 * the causal part of its own block.
 *
 * Layouts (row-major, innermost last; element type = cfg->dtype unless noted):
 *   K, V            [batch, n_kv_heads, ctx_cap, head_dim]   whole context;
 *                   the active segment occupies tokens [q_begin, q_begin+s_len)
 *   Q, O, dO, dQ    [batch, n_q_heads, s_len, head_dim]      active segment
 *   dK, dV          [batch, n_kv_heads, s_len, head_dim]     active segment only
 *   LSE             [batch, n_q_heads, s_len]                float32, natural log
 *   gsum            [batch, n_kv_heads, ctx_cap/8,  head_dim] float32
 *   bsum            [batch, n_kv_heads, ctx_cap/64, head_dim] float32
 *   sel_blk         [batch, n_kv_heads, s_len/64, topk_blocks] int32
 *   sel_grp         [batch, n_kv_heads, s_len/64, topk_groups] int32
 *                   global group indices (token = 8*g + i), ascending, -1 padded
 *
 * Ownership: the caller allocates and owns every buffer (device memory for all
 * arrays; the stream).  Pointers must be 16-byte aligned.  ctx_cap, q_begin,
 * t_begin, t_end and s_len must be multiples of 64.
 *
 * Errors: host-side argument checks run before any launch and return
 * HGA_ERR_INVALID_ARG / HGA_ERR_UNSUPPORTED / HGA_ERR_WORKSPACE with nothing
 * launched.  A failed launch returns HGA_ERR_CUDA.  Kernels that detect a bad
 * selection entry (a group outside [0, 8*own_block)) skip it and latch
 * HGA_ERR_DEVICE_CHECK in a per-device status word; a bounded wait that gives
 * up latches HGA_ERR_TIMEOUT.  hga_get_device_status() reads and clears it.
 */
#ifndef HGA_H
#define HGA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define HGA_API __attribute__((visibility("default")))
#else
#define HGA_API
#endif

#define HGA_BLOCK 64   /* tokens per block  [B], [C] */
#define HGA_GROUP 8    /* tokens per group  [B], [C] */
#define HGA_QBLOCK 64  /* queries per query block */

typedef enum {
  HGA_OK = 0,
  HGA_ERR_INVALID_ARG = 1,
  HGA_ERR_UNSUPPORTED = 2,
  HGA_ERR_CUDA = 3,
  HGA_ERR_TIMEOUT = 4,
  HGA_ERR_DEVICE_CHECK = 5,
  HGA_ERR_WORKSPACE = 6,
  HGA_ERR_IO = 7
} hga_status_t;

typedef enum { HGA_F32 = 0, HGA_BF16 = 1 } hga_dtype_t;

/* flags */
#define HGA_FLAG_SIMT 1u  /* force the CUDA-core attention kernels (fp32 always uses them) */
/* Test only: the tensor-core forward kernel skips loading its first key tile,
 * so its bounded wait runs out; the kernel latches HGA_ERR_TIMEOUT, drains
 * what it started, frees its tensor memory and returns (outputs undefined). */
#define HGA_FLAG_TEST_DROP_FIRST_TILE 0x80000000u

/* Which attention kernels a call uses: the tensor-core (tcgen05) kernels for
 * bf16, head_dim 128 and G in {2, 4} unless HGA_FLAG_SIMT is set; the
 * CUDA-core kernels otherwise. */

typedef struct {
  int32_t batch;
  int32_t n_q_heads;     /* multiple of n_kv_heads; G = n_q_heads / n_kv_heads <= 8 */
  int32_t n_kv_heads;
  int32_t head_dim;      /* 64 or 128 */
  int32_t topk_blocks;   /* level-1 k, 1..64 */
  int32_t topk_groups;   /* level-2 k, 1..256 */
  int32_t dtype;         /* hga_dtype_t: HGA_F32 or HGA_BF16 */
  uint32_t flags;        /* HGA_FLAG_* */
  float scale;           /* softmax scale, normally 1/sqrt(head_dim) */
} hga_config_t;

/* Library version string. */
HGA_API const char* hga_version(void);

/* Human-readable name of a status code. */
HGA_API const char* hga_status_string(hga_status_t status);

/* Name of the CUDA error behind the last HGA_ERR_CUDA a kernel launch of this
 * library returned on the calling thread ("cudaSuccess" if none). */
HGA_API const char* hga_last_cuda_error(void);

/*
 * Step a1 -- summaries [B], [C].  For tokens [t_begin, t_end) of K:
 *   gsum[b,h,g] = mean of keys 8g .. 8g+7      (g = t_begin/8 .. t_end/8-1)
 *   bsum[b,h,c] = mean of keys 64c .. 64c+63   (c = t_begin/64 .. t_end/64-1)
 * accumulated in float32.  Rows outside the range are not touched, so calling
 * it once per segment appends that segment's summaries.
 */
HGA_API hga_status_t hga_build_summaries(const hga_config_t* cfg, const void* k, int64_t ctx_cap,
                                 int64_t t_begin, int64_t t_end, float* gsum, float* bsum,
                                 void* stream);

/*
 * Step a1 for a segment held in its own buffer (used with the host tier,
 * where the whole-context K is not on the device).  k_seg is
 * [batch, n_kv_heads, seg_cap, head_dim] with token t_begin + i at row i;
 * gsum/bsum are the whole-context summaries ([.., ctx_cap/8, ..] and
 * [.., ctx_cap/64, ..]) and receive the rows of groups t_begin/8 .. t_end/8-1
 * and blocks t_begin/64 .. t_end/64-1, exactly as hga_build_summaries would.
 */
HGA_API hga_status_t hga_build_summaries_seg(const hga_config_t* cfg, const void* k_seg,
                                             int64_t seg_cap, int64_t t_begin, int64_t t_end,
                                             int64_t ctx_cap, float* gsum, float* bsum,
                                             void* stream);

/* Bytes of device workspace hga_route needs for this segment. */
HGA_API size_t hga_route_workspace_size(const hga_config_t* cfg, int32_t s_len, int64_t q_begin);

/*
 * Steps a2 + a3 -- two-level weight-free routing [B].  For every (b, KV head h,
 * query block j) of the segment starting at global token q_begin:
 *   qbar = mean of Q over the 64 tokens of block j and the G heads of h;
 *   level 1: score_c = qbar . bsum[b,h,c] for c in [0, J), J = q_begin/64 + j,
 *            keep the top min(topk_blocks, J) (ties: lower c);
 *   level 2: score_g = qbar . gsum[b,h,g] for the 8 groups of each kept block,
 *            keep the top min(topk_groups, 8*kept) (ties: lower g).
 * Scores are ranked without the positive factor 1/sqrt(d) (order unchanged).
 * Writes sel_grp and, if sel_blk is not NULL, sel_blk (ascending, -1 padded).
 * If scores_out ([batch, n_kv_heads, s_len/64, 4] float32) is not NULL it
 * receives, per (b, h, j), the k-th and (k+1)-th largest scores of level 1
 * and of level 2, scaled by cfg->scale (-inf where there is none): a caller
 * can flag near ties from them, e.g. |s_k - s_k+1| <= 1e-3 max(|s_k|, |s_k+1|).
 * bsum/gsum must hold every block/group before the segment's last block
 * (call hga_build_summaries for the segment first).
 * workspace: at least hga_route_workspace_size() bytes of device memory.
 */
HGA_API hga_status_t hga_route(const hga_config_t* cfg, const void* q, int64_t q_begin, int32_t s_len,
                       int64_t ctx_cap, const float* bsum, const float* gsum,
                       int32_t* sel_blk, int32_t* sel_grp, float* scores_out, void* workspace,
                       size_t ws_bytes, void* stream);

/*
 * Step a4 -- exact-token attention forward [A], [B].  Query t of head h'
 * (KV head h'/G, query block j, global position p = q_begin + t) attends to
 *   { 8g+i : g in sel_grp[b,h,j], i < 8 }  U  { own-block tokens at positions <= p }
 * with softmax scale cfg->scale:  O = softmax(q K^T * scale) V,
 * LSE = log(sum exp(q k * scale)).  K/V are read from the whole-context buffers.
 */
HGA_API hga_status_t hga_attn_fwd(const hga_config_t* cfg, const void* q, const void* k, const void* v,
                          int64_t ctx_cap, int64_t q_begin, int32_t s_len,
                          const int32_t* sel_grp, void* o, float* lse, void* stream);

/*
 * hga_route without a caller-provided workspace.  The paper has no
 * counterpart: this is a library convenience for callers that cannot call
 * cudaMalloc -- for example a plugin running inside a host runtime that owns
 * every byte of device memory and hands its extensions no allocator, or code
 * that must not allocate after start-up because cudaMalloc can synchronise
 * the device and has unbounded latency.  Such callers still pass every input
 * and output buffer; only the router's scratch (the mean queries and the
 * candidate chunks' finalists)
 * comes from a fixed array inside the library.
 *
 * The array is HGA_NOALLOC_SCRATCH_BYTES (4 MiB) of device memory that every
 * GPU which loads the library holds until the process exits.  A call whose
 * hga_route_workspace_size() exceeds it returns HGA_ERR_WORKSPACE and
 * launches nothing (for the Qwen3-8B shape -- 32 query / 8 KV heads, d = 128,
 * 2048-token segments, batch 1 -- contexts up to 950,272 tokens fit).
 *
 * The first call on each device looks up the array's device address (with
 * that device current) and caches it; make that first call before any stream
 * capture.  Every call on a device shares the one array and it keeps the
 * last call's contents; nothing in it needs to start at zero, because each
 * call writes every scratch element before reading it.  Calls that can
 * overlap on the GPU (different streams, or several host threads) race on
 * the array: serialise them.  Results are identical to hga_route.
 */
#define HGA_NOALLOC_SCRATCH_BYTES (4u << 20)
HGA_API hga_status_t hga_route_noalloc(const hga_config_t* cfg, const void* q, int64_t q_begin,
                                       int32_t s_len, int64_t ctx_cap, const float* bsum,
                                       const float* gsum, int32_t* sel_blk, int32_t* sel_grp,
                                       void* stream);

/* Bytes of device workspace hga_attn_bwd and hga_attn_fwd_bwd need for this
 * segment: D = rowsum(dO * O) as [B, Hq, S] fp32, 256 bytes for the work
 * counter of the tensor-core dK/dV kernel, two arrays of per-item
 * completion flags ([B, Hkv, S/64] int32 each) used by hga_attn_fwd_bwd, and
 * the inverted selection the dQ kernel writes for the dK/dV kernel ([B, Hkv,
 * S/64 key blocks, S/64 query blocks] int32: which groups of each block of
 * the segment each query block attends); every section starts on a 256-byte
 * boundary. */
HGA_API size_t hga_attn_bwd_workspace_size(const hga_config_t* cfg, int32_t s_len);

/*
 * Step a5 -- backward under segment-wise backprop [A], [B].  Gradients of
 * sum(dO * O) for the forward above, recomputed from the saved LSE:
 *   D = rowsum(dO * O);  P = exp(q k * scale - LSE);  dS = P (dO v - D)
 *   dQ = scale * sum_k dS k                               (every attended key)
 *   dK = scale * sum dS q,  dV = sum P dO                 (active-segment keys only,
 *        summed over the G heads and every query block that attends to them)
 * History keys (positions < q_begin) are detached: no gradient is produced for
 * them.  dq, dk, dv are written, not accumulated.  workspace: at least
 * hga_attn_bwd_workspace_size() bytes of device memory.
 */
HGA_API hga_status_t hga_attn_bwd(const hga_config_t* cfg, const void* q, const void* k, const void* v,
                          int64_t ctx_cap, int64_t q_begin, int32_t s_len,
                          const int32_t* sel_grp, const void* o, const float* lse,
                          const void* d_o, void* dq, void* dk, void* dv, void* workspace,
                          size_t ws_bytes, void* stream);

/*
 * Steps a4 + a5 in one call: hga_attn_fwd then hga_attn_bwd for the same
 * segment, with the same arguments and results (o, lse, dq, dk, dv).  On the
 * tensor-core path the three kernels overlap: the dQ work of a query block
 * starts as soon as that block's forward is done, and the dK/dV work of a
 * key block as soon as D of the query blocks that attend to it is, through
 * per-item completion flags in the workspace instead of whole-grid waits.
 * The flag sections of the workspace must be zero before its first use in
 * this call (e.g. one cudaMemset of the whole workspace after allocating
 * it); each call leaves them holding its own token, which later calls never
 * reuse.  Not to be called concurrently with another call on the same
 * workspace.
 */
HGA_API hga_status_t hga_attn_fwd_bwd(const hga_config_t* cfg, const void* q, const void* k,
                              const void* v, int64_t ctx_cap, int64_t q_begin, int32_t s_len,
                              const int32_t* sel_grp, void* o, float* lse, const void* d_o,
                              void* dq, void* dk, void* dv, void* workspace, size_t ws_bytes,
                              void* stream);

/* Bytes of device workspace hga_segment_fwd_bwd needs: the backward
 * workspace (hga_attn_bwd_workspace_size), one more array of per-item flags
 * ([B, Hkv, S/64] int32, 256-byte aligned) and the routing workspace
 * (hga_route_workspace_size, rounded up to 256 bytes), in that order. */
HGA_API size_t hga_segment_workspace_size(const hga_config_t* cfg, int32_t s_len, int64_t q_begin);

/*
 * Steps a3 + a4 + a5 in one call: hga_route, then hga_attn_fwd_bwd, for one
 * segment, with the same arguments and results (sel_blk, sel_grp, o, lse, dq,
 * dk, dv; sel_blk may be NULL).  Where the routing runs as one kernel (up to
 * 512 key blocks of context) and the attention on the tensor-core path, the
 * forward of a query block starts as soon as that block's selection is
 * written, through a third array of per-item flags; otherwise the steps run
 * one after another.  bsum and gsum are the summaries of the context
 * (hga_summaries), as for hga_route.  The flag sections follow the rule of
 * hga_attn_fwd_bwd: zero before the workspace's first use, never used by two
 * calls at once.  workspace: at least hga_segment_workspace_size() bytes of
 * device memory, 16-byte aligned.
 */
HGA_API hga_status_t hga_segment_fwd_bwd(const hga_config_t* cfg, const void* q, const void* k,
                                         const void* v, int64_t ctx_cap, int64_t q_begin,
                                         int32_t s_len, const float* bsum, const float* gsum,
                                         int32_t* sel_blk, int32_t* sel_grp, void* o, float* lse,
                                         const void* d_o, void* dq, void* dk, void* dv,
                                         void* workspace, size_t ws_bytes, void* stream);

/*
 * Step a7 -- the host tier [A] ("older KV is detached into RAM or NVMe, and
 * HGA loads a bounded set of exact historical tokens for each query block").
 * History K/V stay in pinned host memory (k_host, v_host: whole-context
 * [batch, n_kv_heads, ctx_cap, head_dim], allocated with cudaHostAlloc or
 * registered with cudaHostRegister, device-mapped; pageable memory is
 * rejected with HGA_ERR_INVALID_ARG).  For the segment starting at q_begin,
 * every history group (index < q_begin/8) that any query block of the segment
 * selected in sel_grp is copied once, per (batch, KV head), in ascending
 * order, into rows [8u, 8u+8) of the device staging buffers k_stage/v_stage
 * ([batch, n_kv_heads, stage_cap, head_dim]); u is its slot.  sel_stage
 * ([batch, n_kv_heads, s_len/64, topk_groups]) receives the selection in
 * staging indices: a history group -> its slot; a group of the active segment
 * g -> (stage_cap - s_len)/8 + g - q_begin/8; -1 stays -1.  The caller places
 * the active segment's K/V at staging rows [stage_cap - s_len, stage_cap), so
 * hga_attn_fwd / hga_attn_bwd with (k_stage, v_stage, stage_cap,
 * q_begin' = stage_cap - s_len, sel_stage) compute exactly what they compute on
 * the whole-context buffers.  n_unique ([batch, n_kv_heads] int32, optional)
 * receives the number of groups copied per head: 4 KiB each for bf16, d=128.
 * stage_cap must be a multiple of 64 and >= hga_tier_stage_rows().
 */
HGA_API int64_t hga_tier_stage_rows(const hga_config_t* cfg, int64_t q_begin, int32_t s_len);
HGA_API size_t hga_tier_workspace_size(const hga_config_t* cfg, int32_t s_len, int64_t q_begin);
HGA_API hga_status_t hga_tier_gather(const hga_config_t* cfg, const void* k_host,
                                     const void* v_host, int64_t ctx_cap, int64_t q_begin,
                                     int32_t s_len, const int32_t* sel_grp, void* k_stage,
                                     void* v_stage, int64_t stage_cap, int32_t* sel_stage,
                                     int32_t* n_unique, void* workspace, size_t ws_bytes,
                                     void* stream);

/*
 * Step a6 for the host tier: the active segment's K/V (staging rows
 * [stage_cap - s_len, stage_cap)) join the host history at rows
 * [q_begin, q_begin + s_len) of k_host / v_host (pinned).  One strided
 * device-to-host copy per tensor on `stream` (copy engine, asynchronous).
 */
HGA_API hga_status_t hga_tier_append(const hga_config_t* cfg, const void* k_stage,
                                     const void* v_stage, int64_t stage_cap, void* k_host,
                                     void* v_host, int64_t ctx_cap, int64_t q_begin,
                                     int32_t s_len, void* stream);

/*
 * Strictly causal routing.  The seventnews page, section "一个真正的警告：
 * 因果泄露" (causal leakage): a block's routing decision uses the scores of
 * several query positions, so earlier tokens can learn something about later
 * ones; a strictly causal variant is in development.  Here a query block keeps
 * one shared selection but is routed with the mean query of the 64 tokens
 * before it, so every query the decision uses is earlier than every token it
 * serves.  Candidates and both levels are those of hga_route.
 *
 * qsum [batch, n_kv_heads, ctx_cap/64, head_dim] float32 holds the resident
 * mean query of every block (mean over its 64 tokens and the G heads of the KV
 * head), like bsum holds the mean key.  hga_build_query_summaries writes the
 * rows of the segment's blocks q_begin/64 .. (q_begin+s_len)/64 - 1 from its
 * Q.  hga_route_causal writes those rows too, then routes query block j
 * (global block J = q_begin/64 + j) with row J - 1: for j = 0 that row comes
 * from the previous segment, so route the segments of a sequence in order (or
 * build the row of block q_begin/64 - 1 first).  The first block of a
 * sequence has no candidates and reads no row.  Writes sel_grp and, if not
 * NULL, sel_blk, as hga_route; workspace as hga_route_workspace_size().
 */
HGA_API hga_status_t hga_build_query_summaries(const hga_config_t* cfg, const void* q,
                                               int64_t q_begin, int32_t s_len, int64_t ctx_cap,
                                               float* qsum, void* stream);
HGA_API hga_status_t hga_route_causal(const hga_config_t* cfg, const void* q, int64_t q_begin,
                                      int32_t s_len, int64_t ctx_cap, const float* bsum,
                                      const float* gsum, float* qsum, int32_t* sel_blk,
                                      int32_t* sel_grp, void* workspace, size_t ws_bytes,
                                      void* stream);

/*
 * The upstream pass of a segment, in one read of its projection outputs ([B]
 * "HGA的不同之处": the router scores the existing projected keys; the
 * workloads apply RoPE, base 1e6, before the summaries).  For the s_len tokens
 * starting at global position q_begin:
 *   q_proj [batch, s_len, n_q_heads, head_dim], k_proj and v_proj [batch,
 *   s_len, n_kv_heads, head_dim], token-major; q_row_stride (kv_row_stride)
 *   elements from one token's Q (K and V) row to the next: n_q_heads*head_dim
 *   (n_kv_heads*head_dim) for separate tensors, the fused QKV width for both
 *   when k_proj/v_proj point into the same rows as q_proj; element type
 *   cfg->dtype, each stride times the element size a multiple of 16 bytes
 *   (HGA_ERR_INVALID_ARG otherwise, or if a stride is below its row width);
 *   Q and K are rotated (rotate-half RoPE: for i < d/2, theta_i =
 *   base^(-2i/d), angle p*theta_i at the global position p; rope_base = 0
 *   skips the rotation), V is not;
 *   q_out [batch, n_q_heads, s_len, head_dim] receives Q; k, v (the
 *   whole-context buffers) receive rows [q_begin, q_begin + s_len);
 *   gsum, bsum receive the segment's group and block summaries and qsum
 *   [batch, n_kv_heads, ctx_cap/64, head_dim] float32 its block mean queries
 *   (mean over 64 tokens and the G heads), all of the stored (rounded) values.
 * One launch; it replaces hga_build_summaries and, with
 * hga_route_summarized, every read of Q and K by the routing.
 */
HGA_API hga_status_t hga_prepare_segment(const hga_config_t* cfg, const void* q_proj,
                                         const void* k_proj, const void* v_proj,
                                         int64_t q_row_stride, int64_t kv_row_stride,
                                         int64_t q_begin, int32_t s_len,
                                         int64_t ctx_cap, float rope_base, void* q_out, void* k,
                                         void* v, float* gsum, float* bsum, float* qsum,
                                         void* stream);

/*
 * hga_route (causal = 0) or hga_route_causal (causal = 1) from the resident
 * summaries alone: query block j (global block J) is routed with row J
 * (causal: J - 1) of qsum, which hga_prepare_segment or
 * hga_build_query_summaries wrote; Q is not read.  Results equal those calls'
 * when qsum holds the block means they form.  workspace as
 * hga_route_workspace_size().
 */
HGA_API hga_status_t hga_route_summarized(const hga_config_t* cfg, int64_t q_begin,
                                          int32_t s_len, int64_t ctx_cap, const float* bsum,
                                          const float* gsum, const float* qsum, int32_t causal,
                                          int32_t* sel_blk, int32_t* sel_grp, void* workspace,
                                          size_t ws_bytes, void* stream);

/*
 * Decode -- one new token per sequence [A] ("HGA can also be used for
 * retrieval and generation"), routed and attended as in [B] with the query
 * block reduced to that one token.  For sequence b the token sits at global
 * position pos[b] (device array of `batch` int64; 0 <= pos[b] < ctx_cap).
 * Per (b, KV head h), with J = pos[b] / 64 the token's own block:
 *   qbar = mean of its query over the G heads of h;
 *   level 1: score_c = qbar . bsum[b,h,c] for c in [0, J), keep the top
 *            min(topk_blocks, J) (ties: lower c);
 *   level 2: the 8 groups of each kept block, keep the top
 *            min(topk_groups, 8*kept) (ties: lower g);
 *   attention of each of the G heads over { 8g+i : g selected, i < 8 } U
 *   { 64J .. pos[b] } (its own key included), scale cfg->scale.
 * Layouts: q, o [batch, n_q_heads, head_dim] (cfg->dtype); lse
 * [batch, n_q_heads] float32, natural log; K/V the whole-context buffers
 * [batch, n_kv_heads, ctx_cap, head_dim] with the new token's K/V already
 * written at row pos[b]; bsum/gsum as for hga_route, holding every complete
 * block before the token's own block (call hga_build_summaries for a block
 * once its 64 tokens are in K; rebuilding a range is harmless).  sel_blk
 * [batch, n_kv_heads, topk_blocks] and sel_grp [batch, n_kv_heads,
 * topk_groups] (int32, ascending, -1 padded) are written when not NULL.
 * G = n_q_heads / n_kv_heads must be 1, 2, 4 or 8 (else HGA_ERR_UNSUPPORTED).
 * A position outside [0, ctx_cap) leaves that sequence's outputs untouched and
 * latches HGA_ERR_DEVICE_CHECK.  One launch; no workspace.
 */
HGA_API hga_status_t hga_decode(const hga_config_t* cfg, const void* q, const void* k,
                                const void* v, int64_t ctx_cap, const int64_t* pos,
                                const float* bsum, const float* gsum, int32_t* sel_blk,
                                int32_t* sel_grp, void* o, float* lse, void* stream);

/*
 * Step a7, third tier: history K/V in files on NVMe ([A]: older KV is
 * detached into RAM or NVMe; seventnews, section "意义何在": NVMe-backed
 * tiered storage).  A K or V file holds the whole context in the layout of
 * the device buffers, [batch, n_kv_heads, ctx_cap, head_dim] elements, so a
 * group is one contiguous run of 8*head_dim elements.  Per segment:
 *
 * hga_tier_plan (device, asynchronous): the planning half of
 *   hga_tier_gather: sel_stage receives the selection in staging indices (as
 *   there); slot_group ([batch, n_kv_heads, slot_cap] int32) the distinct
 *   selected history groups of each head in ascending order, n_unique
 *   ([batch, n_kv_heads] int32) their number.  slot_cap >=
 *   min(s_len/64 * topk_groups, q_begin/8); stage_cap as for hga_tier_gather.
 *
 * hga_tier_read_groups (host, synchronous): with slot_group and n_unique
 *   copied to host memory, reads every listed group of every head from the
 *   files fd_k / fd_v into host staging buffers laid out like the device
 *   staging ([batch, n_kv_heads, stage_cap, head_dim]; slot u at rows
 *   [8u, 8u+8)), one pread per run of consecutive groups, on n_threads
 *   threads.  The caller then copies rows [0, 8*n_unique) of each head to
 *   the device staging (one 2-D copy per tensor).  HGA_ERR_IO if a read fails
 *   or ends early; HGA_ERR_INVALID_ARG for a group or count out of range.
 *
 * hga_tier_write_segment (host, synchronous): writes the segment's rows
 *   [q_begin, q_begin + s_len) of every head from host buffers ([batch,
 *   n_kv_heads, seg_rows, head_dim], the segment at rows [0, s_len)) into the
 *   files, one pwrite per head and tensor on n_threads threads.
 *
 * The file descriptors are the caller's (opened for reading / writing; with
 * O_DIRECT the buffers, offsets and sizes must meet the device's alignment:
 * groups are 2 KiB at bf16, d = 128).
 */
HGA_API hga_status_t hga_tier_plan(const hga_config_t* cfg, int64_t q_begin, int32_t s_len,
                                   const int32_t* sel_grp, int64_t stage_cap, int32_t* sel_stage,
                                   int32_t* slot_group, int32_t* n_unique, int64_t slot_cap,
                                   void* stream);
HGA_API hga_status_t hga_tier_read_groups(const hga_config_t* cfg, int fd_k, int fd_v,
                                          int64_t ctx_cap, const int32_t* slot_group,
                                          const int32_t* n_unique, int64_t slot_cap,
                                          void* k_stage_host, void* v_stage_host,
                                          int64_t stage_cap, int32_t n_threads);
HGA_API hga_status_t hga_tier_write_segment(const hga_config_t* cfg, int fd_k, int fd_v,
                                            int64_t ctx_cap, int64_t q_begin, int32_t s_len,
                                            const void* k_seg_host, const void* v_seg_host,
                                            int64_t seg_rows, int32_t n_threads);

/*
 * Reads and clears the calling device's latched device-side status
 * (HGA_OK, HGA_ERR_DEVICE_CHECK or HGA_ERR_TIMEOUT).  Synchronises `stream`.
 */
HGA_API hga_status_t hga_get_device_status(void* stream);


/* ------------------------------------------------------------------------
 * Diagnostics: launch counting and per-kernel timing.
 *
 * Every kernel launch of the library increments a process-wide counter.
 * The hot-path kernels (summaries, routing, tensor-core attention) are
 * launched with programmatic stream serialization: each may be scheduled
 * while the kernel before it on the stream drains, and waits for that
 * kernel's completion on the device before touching memory.
 * When timing is enabled, each launch is bracketed by two CUDA events
 * recorded on its stream (as external event nodes while the stream is being
 * captured into a CUDA graph, so graph replays are timed too).  Events come
 * from a pool created by hga_timing_enable (host-side event objects, no
 * device memory); launches beyond the pool are not timed.
 * ------------------------------------------------------------------------ */

/* Kernel kinds reported by the timing facility. */
typedef enum {
  HGA_K_SUMMARIES = 0,
  HGA_K_QBAR = 1,
  HGA_K_BLOCK_TOPK = 2,
  HGA_K_SELECT = 3,
  HGA_K_FWD_SIMT = 4,
  HGA_K_BWD_DQ_SIMT = 5,
  HGA_K_BWD_DKDV_SIMT = 6,
  HGA_K_FWD_TC = 7,
  HGA_K_BWD_DQ_TC = 8,
  HGA_K_BWD_DKDV_TC = 9,
  HGA_K_TIER_DEDUP = 10,
  HGA_K_TIER_COPY = 11,
  HGA_K_ROUTE_FUSED = 12,
  HGA_K_DECODE = 13,
  HGA_K_QSUM = 14,
  HGA_K_PREPARE = 15,
  HGA_K_COUNT = 16
} hga_kernel_kind_t;

/* Name of a kernel kind ("attn_fwd_simt", ...). */
HGA_API const char* hga_kernel_name(int kind);

/* Number of kernels this library has launched in this process. */
HGA_API uint64_t hga_launch_count(void);

/* slots > 0: enable timing with a pool of `slots` event pairs (created on
 * first use, reused afterwards); 0: disable.  Rewinds the pool cursor, so the
 * next launches use slots 0, 1, ... again. */
HGA_API hga_status_t hga_timing_enable(int32_t slots);

/* Waits for the event pairs of the slots used since the last
 * hga_timing_enable and adds their durations to the per-kind totals.  Eager
 * use: enable, launch, collect.  Graph use: enable, capture (the captured
 * launches keep their slots), then replay + collect as often as wanted. */
HGA_API hga_status_t hga_timing_collect(void);

/* Accumulated milliseconds and timed launches of one kernel kind. */
HGA_API hga_status_t hga_timing_get(int kind, double* ms, uint64_t* launches);

/* Zeroes the per-kind totals. */
HGA_API void hga_timing_reset(void);

/* Restricts timing to the kinds whose bit (1u << kind) is set in `mask`
 * (initially all).  Launches of other kinds are counted but not bracketed,
 * so they keep their programmatic dependency on the kernel before them
 * (an event between two kernels orders them fully). */
HGA_API void hga_timing_kinds(uint32_t mask);

#ifdef __cplusplus
}
#endif

#endif /* HGA_H */
