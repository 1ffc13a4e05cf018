"""CPU oracle for the HGA hot path -- TEST INFRASTRUCTURE ONLY.

Only the tests, the smoke check and the benchmark's CPU-baseline leg may import
this module.  The library (libhga and its Python binding) never calls it, and it
shares no code with the CUDA path: it imports numpy and nothing else.

It is a plain, slow, float64 restatement of what the pages describe, one step
after the other, with no blocking, fusion or reordering.  Sources (the HGA
pages, all about "Long-Context Fine-Tuning with Limited VRAM"):

  [P2]  adnankhan.ai notes "Long-Context Fine-Tuning with Limited VRAM",
        section "Raw Abstract / Excerpt" (bounded set of exact historical
        tokens per query block; only the active segment is differentiable,
        older KV is detached).
  [P3a] seventnews "BMW如何通过重新设计注意力机制，在16 GB GPU上实现16K上下文",
        section "HGA的不同之处" (what HGA does differently): 64-token blocks
        with a compact summary each; queries score the summaries, the top-k
        blocks are opened at the level of 8-token groups, and only the
        selected groups' exact-token K/V enter attention; the router has no
        learned weights and scores the existing projected keys; summaries are
        never attention values.
  [P3b] same page, same section, last paragraph: 2048-token segments, forward
        and backward per segment, no gradient across segment boundaries, later
        segments still attend to earlier exact tokens through routing.
  [P5]  gist.science retelling, section "解决方案" (the solution): 64-token
        block summary cards and an 8-token group summary cache.

Readings adopted where the pages are silent (each one is the plainest reading
the rest supports):

  R1  summary of a block / group = mean of its post-RoPE keys, per KV head;
  R2  routing score of a candidate = mean, over the query block's 64 queries
      and the G query heads sharing the KV head, of q.s/sqrt(d); by linearity
      this equals qbar.s/sqrt(d) with qbar the mean query;
  R3  candidates of query block j = every complete block strictly before the
      query block's own block (history and earlier blocks of the segment);
  R4  level 2 opens only the selected blocks: their groups compete for the
      top-k group slots;
  R5  ties go to the lower index (block index at level 1, global group index
      at level 2); fewer candidates than k -> take all, pad with -1; the
      selection is a set, reported in ascending order;
  R6  attention of a query at global position p = softmax over the union of
      the selected groups' tokens and its own block's tokens at positions <= p,
      scale 1/sqrt(d), natural-log LSE;
  R7  one selection per (batch, KV head, query block), shared by the G heads;
  R8  under segment-wise backprop the history K/V are detached: history keys
      give dQ only, keys of the active segment give dQ, dK and dV; no gradient
      flows through the discrete routing or the summaries;
  R9  near ties: when the k-th and (k+1)-th sorted scores of a level differ by
      at most 1e-3 relative, the row is flagged; a flagged row's attention is
      checked with the GPU's own selection.

Parity pins (tests/test_oracle_pins.py): brute force of R2-R5 on tiny inputs,
closed forms and hand-computed golden fixtures for R1, equality with dense
causal attention (torch SDPA in float64, autograd for gradients) when top-k
covers every candidate, equality with masked SDPA for general selections,
finite differences, softmax rows summing to one, and the keyset bound.
"""

from __future__ import annotations

import math

import numpy as np

BLOCK = 64      # tokens per block                       [P3a], [P5]
GROUP = 8       # tokens per group                       [P3a], [P5]
QBLOCK = 64     # queries per query block (reading R1..R7 share this size)
GROUPS_PER_BLOCK = BLOCK // GROUP
TIE_REL = 1e-3


# ----------------------------------------------------------------------------
# step a1: summaries (R1)
# ----------------------------------------------------------------------------

def build_summaries(k: np.ndarray, t_begin: int, t_end: int):
    """Group and block summaries of keys in [t_begin, t_end).

    k: [B, Hkv, T, d] float64 post-RoPE keys.  Returns (gsum, bsum) with
    gsum[b,h,i] = mean of the 8 keys of group t_begin/8 + i and
    bsum[b,h,i] = mean of the 64 keys of block t_begin/64 + i.
    """
    assert t_begin % BLOCK == 0 and t_end % BLOCK == 0 and t_end <= k.shape[2]
    B, H, _, d = k.shape
    seg = k[:, :, t_begin:t_end, :]
    n = t_end - t_begin
    gsum = seg.reshape(B, H, n // GROUP, GROUP, d).mean(axis=3)
    bsum = seg.reshape(B, H, n // BLOCK, BLOCK, d).mean(axis=3)
    return gsum, bsum


# ----------------------------------------------------------------------------
# steps a2 + a3: two-level routing (R2..R5, R7, R9)
# ----------------------------------------------------------------------------

def _topk_lower_index(scores: np.ndarray, idx: np.ndarray, k: int):
    """Order candidates by (-score, index); return (chosen indices, sorted scores)."""
    order = np.lexsort((idx, -scores))
    return idx[order[:k]], scores[order]


def _near_tie(sorted_scores: np.ndarray, k: int) -> bool:
    if k >= len(sorted_scores) or k == 0:
        return False
    a, b = sorted_scores[k - 1], sorted_scores[k]
    return abs(a - b) <= TIE_REL * max(abs(a), abs(b))


def route(q: np.ndarray, bsum: np.ndarray, gsum: np.ndarray, q_begin: int,
          topk_blocks: int, topk_groups: int, n_kv_heads: int):
    """Two-level weight-free routing of one segment's query blocks.

    q: [B, Hq, S, d] float64 (the segment, first token at global q_begin).
    bsum: [B, Hkv, >= J_max, d] block summaries by global block index.
    gsum: [B, Hkv, >= 8 J_max, d] group summaries by global group index.
    Returns sel_blk [B,Hkv,n_qb,k_b] int32, sel_grp [B,Hkv,n_qb,k_g] int32
    (ascending, -1 padded) and near_tie [B,Hkv,n_qb] bool.
    """
    B, Hq, S, d = q.shape
    G = Hq // n_kv_heads
    n_qb = S // QBLOCK
    sel_blk = np.full((B, n_kv_heads, n_qb, topk_blocks), -1, np.int32)
    sel_grp = np.full((B, n_kv_heads, n_qb, topk_groups), -1, np.int32)
    near_tie = np.zeros((B, n_kv_heads, n_qb), bool)
    inv_sqrt_d = 1.0 / math.sqrt(d)
    for b in range(B):
        for h in range(n_kv_heads):
            for j in range(n_qb):
                own = (q_begin + QBLOCK * j) // BLOCK          # the query block's own block
                qblk = q[b, h * G:(h + 1) * G, QBLOCK * j:QBLOCK * (j + 1), :]
                qbar = qblk.reshape(-1, d).mean(axis=0)        # R2: mean over queries and heads
                # level 1: candidates are the complete blocks before `own` (R3)
                cand = np.arange(own)
                s1 = (bsum[b, h, :own, :] @ qbar) * inv_sqrt_d
                kb = min(topk_blocks, own)
                blocks, s1_sorted = _topk_lower_index(s1, cand, kb)
                blocks = np.sort(blocks)
                # level 2: the groups of the selected blocks compete (R4)
                groups = (blocks[:, None] * GROUPS_PER_BLOCK
                          + np.arange(GROUPS_PER_BLOCK)[None, :]).reshape(-1)
                s2 = (gsum[b, h, groups, :] @ qbar) * inv_sqrt_d
                kg = min(topk_groups, len(groups))
                chosen, s2_sorted = _topk_lower_index(s2, groups, kg)
                chosen = np.sort(chosen)
                sel_blk[b, h, j, :kb] = blocks
                sel_grp[b, h, j, :kg] = chosen
                near_tie[b, h, j] = _near_tie(s1_sorted, kb) or _near_tie(s2_sorted, kg)
    return sel_blk, sel_grp, near_tie


# ----------------------------------------------------------------------------
# keysets (R6)
# ----------------------------------------------------------------------------

def routed_keys(sel_row: np.ndarray) -> np.ndarray:
    """Token positions of the selected groups (ascending, padding dropped)."""
    g = sel_row[sel_row >= 0].astype(np.int64)
    return (g[:, None] * GROUP + np.arange(GROUP)[None, :]).reshape(-1)


def keyset(q_begin: int, j: int, r: int, sel_row: np.ndarray) -> np.ndarray:
    """All key positions attended by query r (0..63) of query block j."""
    own0 = ((q_begin + QBLOCK * j) // BLOCK) * BLOCK
    p = q_begin + QBLOCK * j + r
    own = np.arange(own0, p + 1)
    return np.concatenate([routed_keys(sel_row), own])


def _block_keys(q_begin: int, j: int, sel_row: np.ndarray):
    """Union of the query block's keys plus a [64, n] mask of which query sees which."""
    own0 = ((q_begin + QBLOCK * j) // BLOCK) * BLOCK
    routed = routed_keys(sel_row)
    keys = np.concatenate([routed, own0 + np.arange(BLOCK)])
    pos_q = q_begin + QBLOCK * j + np.arange(QBLOCK)
    visible = np.ones((QBLOCK, len(keys)), bool)
    visible[:, len(routed):] = keys[None, len(routed):] <= pos_q[:, None]
    return keys, visible


# ----------------------------------------------------------------------------
# step a4: forward (R6, R7)
# ----------------------------------------------------------------------------

def attn_fwd(q, k, v, q_begin: int, sel_grp: np.ndarray, n_kv_heads: int):
    """Exact-token attention of one segment over its selection.

    q: [B,Hq,S,d], k/v: [B,Hkv,T,d] float64; sel_grp [B,Hkv,n_qb,k_g].
    Returns o [B,Hq,S,d] and lse [B,Hq,S] (natural log).
    """
    B, Hq, S, d = q.shape
    G = Hq // n_kv_heads
    scale = 1.0 / math.sqrt(d)
    o = np.zeros_like(q)
    lse = np.zeros((B, Hq, S))
    for b in range(B):
        for h in range(n_kv_heads):
            for j in range(S // QBLOCK):
                keys, visible = _block_keys(q_begin, j, sel_grp[b, h, j])
                kk, vv = k[b, h, keys, :], v[b, h, keys, :]
                for hq in range(h * G, (h + 1) * G):
                    rows = slice(QBLOCK * j, QBLOCK * (j + 1))
                    s = (q[b, hq, rows, :] @ kk.T) * scale
                    s = np.where(visible, s, -np.inf)
                    m = s.max(axis=1, keepdims=True)
                    p = np.exp(s - m)
                    l = p.sum(axis=1, keepdims=True)
                    o[b, hq, rows, :] = (p @ vv) / l
                    lse[b, hq, rows] = (m + np.log(l))[:, 0]
    return o, lse


# ----------------------------------------------------------------------------
# step a5: backward under segment-wise backprop (R8)
# ----------------------------------------------------------------------------

def attn_bwd(q, k, v, do, q_begin: int, sel_grp: np.ndarray, n_kv_heads: int):
    """Gradients of sum(dO * O) for one segment.

    Returns dq [B,Hq,S,d] and, for the active segment's keys only,
    dk, dv [B,Hkv,S,d] (positions q_begin .. q_begin+S-1).  History keys are
    detached, so their gradient is not produced.
    """
    B, Hq, S, d = q.shape
    G = Hq // n_kv_heads
    scale = 1.0 / math.sqrt(d)
    T = k.shape[2]
    dq = np.zeros_like(q)
    dk_full = np.zeros((B, n_kv_heads, T, d))
    dv_full = np.zeros((B, n_kv_heads, T, d))
    for b in range(B):
        for h in range(n_kv_heads):
            for j in range(S // QBLOCK):
                keys, visible = _block_keys(q_begin, j, sel_grp[b, h, j])
                kk, vv = k[b, h, keys, :], v[b, h, keys, :]
                for hq in range(h * G, (h + 1) * G):
                    rows = slice(QBLOCK * j, QBLOCK * (j + 1))
                    qq, dd = q[b, hq, rows, :], do[b, hq, rows, :]
                    s = np.where(visible, (qq @ kk.T) * scale, -np.inf)
                    m = s.max(axis=1, keepdims=True)
                    p = np.exp(s - m)
                    p = p / p.sum(axis=1, keepdims=True)       # softmax probabilities
                    oo = p @ vv
                    dp = dd @ vv.T
                    D = (dd * oo).sum(axis=1, keepdims=True)
                    ds = p * (dp - D)
                    dq[b, hq, rows, :] = (ds @ kk) * scale
                    np.add.at(dk_full[b, h], keys, (ds.T @ qq) * scale)
                    np.add.at(dv_full[b, h], keys, p.T @ dd)
    act = slice(q_begin, q_begin + S)
    return dq, dk_full[:, :, act, :], dv_full[:, :, act, :]


# ----------------------------------------------------------------------------
# step a7: host tier -- which history groups cross PCIe, and the selection in
# staging indices (the adnankhan.ai notes, "Raw Abstract / Excerpt": older KV
# is detached into RAM or NVMe; HGA loads a bounded set of exact historical
# tokens per query block)
# ----------------------------------------------------------------------------

def tier_stage(sel_grp: np.ndarray, q_begin: int, s_len: int, stage_cap: int):
    """Per (b, KV head): the distinct history groups (index < q_begin/8) any
    query block of the segment selected, ascending -- these are copied once --
    and the selection rewritten to staging indices: history group -> its rank
    among them, active-segment group g -> (stage_cap - s_len)/8 + g - q_begin/8,
    -1 -> -1.  Returns (list of per-(b,h) unique arrays, sel_stage)."""
    B, H = sel_grp.shape[:2]
    n_hist = q_begin // GROUP
    act0 = (stage_cap - s_len) // GROUP
    uniques = [[None] * H for _ in range(B)]
    out = np.full_like(sel_grp, -1)
    for b in range(B):
        for h in range(H):
            sel = sel_grp[b, h]
            hist = np.unique(sel[(sel >= 0) & (sel < n_hist)])
            uniques[b][h] = hist
            rank = {int(g): i for i, g in enumerate(hist)}
            for idx, g in np.ndenumerate(sel):
                if g < 0:
                    continue
                out[b, h][idx] = rank[int(g)] if g < n_hist else act0 + (int(g) - n_hist)
    return uniques, out


# ----------------------------------------------------------------------------
# one segment of the segment-wise loop (a1 .. a5 in order)
# ----------------------------------------------------------------------------

def segment_step(q, k, v, do, q_begin: int, gsum, bsum, topk_blocks: int,
                 topk_groups: int, n_kv_heads: int, backward: bool = True):
    """Summarise the segment's keys into gsum/bsum (in place, global indices),
    route, attend, and (optionally) backpropagate.  Returns a dict."""
    S = q.shape[2]
    g, bl = build_summaries(k, q_begin, q_begin + S)
    gsum[:, :, q_begin // GROUP:(q_begin + S) // GROUP] = g
    bsum[:, :, q_begin // BLOCK:(q_begin + S) // BLOCK] = bl
    sel_blk, sel_grp, tie = route(q, bsum, gsum, q_begin, topk_blocks, topk_groups,
                                  n_kv_heads)
    o, lse = attn_fwd(q, k, v, q_begin, sel_grp, n_kv_heads)
    out = dict(sel_blk=sel_blk, sel_grp=sel_grp, near_tie=tie, o=o, lse=lse)
    if backward:
        dq, dk, dv = attn_bwd(q, k, v, do, q_begin, sel_grp, n_kv_heads)
        out.update(dq=dq, dk=dk, dv=dv)
    return out


# ----------------------------------------------------------------------------
# decode: one new token per sequence routed against the resident summaries
# (the adnankhan.ai notes, "Raw Abstract / Excerpt": HGA can also be used for
# generation).  Readings:
#   D1  the "query block" of a decode step is the one new token: qbar is the
#       mean of its query over the G heads of the KV head (R2 with 1 row);
#   D2  candidates are the complete blocks before the token's own block
#       (R3): [0, pos // 64); the own block is not complete, so its summary
#       is never scored;
#   D3  the token attends to the selected groups' tokens and to its own
#       block's tokens at positions <= pos (R6), its own K/V included (the
#       caller writes them into the context before the step).
# ----------------------------------------------------------------------------

def decode_route(q_tok: np.ndarray, bsum: np.ndarray, gsum: np.ndarray, pos,
                 topk_blocks: int, topk_groups: int, n_kv_heads: int):
    """Routing of one token per sequence.  q_tok: [B, Hq, d] float64; pos:
    global position of each sequence's token.  Returns sel_blk [B,Hkv,k_b],
    sel_grp [B,Hkv,k_g] (ascending, -1 padded) and near_tie [B,Hkv]."""
    B, Hq, d = q_tok.shape
    G = Hq // n_kv_heads
    sel_blk = np.full((B, n_kv_heads, topk_blocks), -1, np.int32)
    sel_grp = np.full((B, n_kv_heads, topk_groups), -1, np.int32)
    near_tie = np.zeros((B, n_kv_heads), bool)
    inv_sqrt_d = 1.0 / math.sqrt(d)
    for b in range(B):
        own = int(pos[b]) // BLOCK                         # D2
        for h in range(n_kv_heads):
            qbar = q_tok[b, h * G:(h + 1) * G, :].mean(axis=0)      # D1
            s1 = (bsum[b, h, :own, :] @ qbar) * inv_sqrt_d
            kb = min(topk_blocks, own)
            blocks, s1_sorted = _topk_lower_index(s1, np.arange(own), kb)
            blocks = np.sort(blocks)
            groups = (blocks[:, None] * GROUPS_PER_BLOCK
                      + np.arange(GROUPS_PER_BLOCK)[None, :]).reshape(-1)
            s2 = (gsum[b, h, groups, :] @ qbar) * inv_sqrt_d
            kg = min(topk_groups, len(groups))
            chosen, s2_sorted = _topk_lower_index(s2, groups, kg)
            sel_blk[b, h, :kb] = blocks
            sel_grp[b, h, :kg] = np.sort(chosen)
            near_tie[b, h] = _near_tie(s1_sorted, kb) or _near_tie(s2_sorted, kg)
    return sel_blk, sel_grp, near_tie


def decode_attn(q_tok: np.ndarray, k: np.ndarray, v: np.ndarray, pos, sel_grp: np.ndarray,
                n_kv_heads: int):
    """Attention of one token per sequence over its selection (D3).
    Returns o [B, Hq, d] and lse [B, Hq] (natural log)."""
    B, Hq, d = q_tok.shape
    G = Hq // n_kv_heads
    scale = 1.0 / math.sqrt(d)
    o = np.zeros_like(q_tok)
    lse = np.zeros((B, Hq))
    for b in range(B):
        p = int(pos[b])
        own0 = (p // BLOCK) * BLOCK
        for h in range(n_kv_heads):
            keys = np.concatenate([routed_keys(sel_grp[b, h]), np.arange(own0, p + 1)])
            kk, vv = k[b, h, keys, :], v[b, h, keys, :]
            for hq in range(h * G, (h + 1) * G):
                s = (kk @ q_tok[b, hq]) * scale
                m = s.max()
                w = np.exp(s - m)
                o[b, hq] = (w @ vv) / w.sum()
                lse[b, hq] = m + math.log(w.sum())
    return o, lse


# ----------------------------------------------------------------------------
# strictly causal routing (seventnews page, section "一个真正的警告：因果泄露":
# because a block's routing decision uses the scores of several query
# positions, earlier tokens can learn something about later ones; a strictly
# causal variant is in development).  Reading C1: a query block keeps one
# shared selection, but it is routed with the mean query of the 64 tokens
# just before it (the previous block, global block J-1), so that every query
# the decision uses is earlier than every token it serves.  Candidates and
# both levels are as in route() (R3..R5).  The first block of a sequence has
# no candidates, so it needs no earlier queries.
# ----------------------------------------------------------------------------

def query_summaries(q: np.ndarray, n_kv_heads: int) -> np.ndarray:
    """Mean query of every 64-token block per KV head: q [B, Hq, S, d] (S a
    multiple of 64) -> [B, Hkv, S/64, d], the mean over the block's 64 tokens
    and the G heads of the KV head (R2)."""
    B, Hq, S, d = q.shape
    G = Hq // n_kv_heads
    return q.reshape(B, n_kv_heads, G, S // QBLOCK, QBLOCK, d).mean(axis=(2, 4))


def route_causal(q_prev_mean: np.ndarray, bsum: np.ndarray, gsum: np.ndarray, q_begin: int,
                 n_qb: int, topk_blocks: int, topk_groups: int):
    """Causal routing of the segment's n_qb query blocks (C1).  q_prev_mean
    [B, Hkv, n_qb, d]: for query block j, the mean query of global block
    q_begin/64 + j - 1 (any value where that block does not exist).  Returns
    sel_blk, sel_grp (ascending, -1 padded) and near_tie, as route()."""
    B, H, _, d = q_prev_mean.shape
    sel_blk = np.full((B, H, n_qb, topk_blocks), -1, np.int32)
    sel_grp = np.full((B, H, n_qb, topk_groups), -1, np.int32)
    near_tie = np.zeros((B, H, n_qb), bool)
    inv_sqrt_d = 1.0 / math.sqrt(d)
    for b in range(B):
        for h in range(H):
            for j in range(n_qb):
                own = q_begin // BLOCK + j
                qbar = q_prev_mean[b, h, j]
                s1 = (bsum[b, h, :own, :] @ qbar) * inv_sqrt_d
                kb = min(topk_blocks, own)
                blocks, s1_sorted = _topk_lower_index(s1, np.arange(own), kb)
                blocks = np.sort(blocks)
                groups = (blocks[:, None] * GROUPS_PER_BLOCK
                          + np.arange(GROUPS_PER_BLOCK)[None, :]).reshape(-1)
                s2 = (gsum[b, h, groups, :] @ qbar) * inv_sqrt_d
                kg = min(topk_groups, len(groups))
                chosen, s2_sorted = _topk_lower_index(s2, groups, kg)
                sel_blk[b, h, j, :kb] = blocks
                sel_grp[b, h, j, :kg] = np.sort(chosen)
                near_tie[b, h, j] = _near_tie(s1_sorted, kb) or _near_tie(s2_sorted, kg)
    return sel_blk, sel_grp, near_tie


# ----------------------------------------------------------------------------
# the upstream pass of a segment: from the Q/K/V projection outputs to the
# tensors and summaries the path reads (the seventnews page, section
# "HGA的不同之处": the router scores the existing projected keys; the
# workloads apply RoPE, base 1e6, before the summaries).  Readings:
#   U1  the projection outputs are token-major, [B, S, H, d] per tensor;
#   U2  RoPE is the rotate-half form: for i < d/2, with theta_i =
#       base^(-2i/d) and angle p * theta_i at global position p,
#       (x_i, x_{i+d/2}) -> (x_i cos - x_{i+d/2} sin, x_{i+d/2} cos + x_i sin);
#       V is not rotated;
#   U3  Q, K and V are stored in the path's element type (bf16: round to
#       nearest even), and the summaries and block mean queries are taken of
#       the stored values.
# ----------------------------------------------------------------------------

def rope(x: np.ndarray, pos0: int, base: float) -> np.ndarray:
    """Rotate-half RoPE (U2) of x [..., S, d] at positions pos0 .. pos0+S-1."""
    d = x.shape[-1]
    half = d // 2
    theta = base ** (-2.0 * np.arange(half) / d)
    ang = (pos0 + np.arange(x.shape[-2]))[:, None] * theta[None, :]
    c, s = np.cos(ang), np.sin(ang)
    x1, x2 = x[..., :half], x[..., half:]
    return np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=-1)


def round_bf16(x: np.ndarray) -> np.ndarray:
    """float64 -> nearest bfloat16 (8-bit significand, ties to even), as float64."""
    x = np.asarray(x, np.float64)
    m, e = np.frexp(x)                       # x = m * 2^e, 0.5 <= |m| < 1
    scaled = np.ldexp(m, 8)                  # 8 significant bits above the point
    return np.ldexp(np.round(scaled), e - 8)     # np.round: half to even


def prepare_segment(q_proj, k_proj, v_proj, q_begin: int, rope_base, n_kv_heads: int,
                    dtype: str):
    """q_proj [B, S, Hq, d], k_proj / v_proj [B, S, Hkv, d] float64 (U1).
    Returns q [B, Hq, S, d], k, v [B, Hkv, S, d] as stored (U2, U3), the
    segment's gsum / bsum (R1, global indices from q_begin/8 and q_begin/64)
    and qsum [B, Hkv, S/64, d] (the block mean queries)."""
    q = np.transpose(q_proj, (0, 2, 1, 3))
    k = np.transpose(k_proj, (0, 2, 1, 3))
    v = np.transpose(v_proj, (0, 2, 1, 3))
    if rope_base is not None:
        q, k = rope(q, q_begin, rope_base), rope(k, q_begin, rope_base)
    if dtype == "bf16":
        q, k, v = round_bf16(q), round_bf16(k), round_bf16(v)
    else:
        q, k, v = (np.asarray(t, np.float32).astype(np.float64) for t in (q, k, v))
    S = q.shape[2]
    gsum, bsum = build_summaries(k, 0, S)
    return q, k, v, gsum, bsum, query_summaries(q, n_kv_heads)
