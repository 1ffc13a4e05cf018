"""Helpers shared by the parity tests: run the CUDA path through the C ABI on
seeded synthetic inputs and run the oracle on the same inputs."""

from __future__ import annotations

import numpy as np

import oracle
from hierarchical_routed_sparse_hga_b200 import synth

# tolerances: float32 path max-abs 1e-4; bf16 path 2e-2 of the tensor's max |oracle|
F32_ABS = 1e-4
BF16_REL = 2e-2
LSE_ABS = 1e-4
SUMMARY_REL = 1e-5
TIE_REL = 1e-3      # the near-tie window of the routing scores


def torch_dtype(w):
    import torch
    return torch.bfloat16 if w.dtype == "bf16" else torch.float32


def to_device(arr, w, device="cuda"):
    """Storage numpy array (uint16 bf16 bits or float32) -> CUDA tensor."""
    import torch
    if w.dtype == "bf16":
        t = torch.from_numpy(np.ascontiguousarray(arr).view(np.int16)).view(torch.bfloat16)
    else:
        t = torch.from_numpy(np.ascontiguousarray(arr, dtype=np.float32))
    return t.to(device)


def to_f64(t):
    import torch
    return t.detach().to(torch.float64).cpu().numpy()


def config_of(w, flags=0):
    from hierarchical_routed_sparse_hga_b200 import HGA_BF16, HGA_F32, Config
    return Config(w.batch, w.n_q_heads, w.n_kv_heads, w.head_dim, w.topk_blocks,
                  w.topk_groups, HGA_BF16 if w.dtype == "bf16" else HGA_F32, flags)


def assert_close(gpu, ref, w, what, rel=None, abs_=None):
    gpu = np.asarray(gpu, np.float64)
    ref = np.asarray(ref, np.float64)
    assert gpu.shape == ref.shape, (what, gpu.shape, ref.shape)
    err = np.max(np.abs(gpu - ref)) if ref.size else 0.0
    if abs_ is not None:
        bound = abs_
    elif rel is not None:
        bound = rel * max(np.max(np.abs(ref)), 1e-30)
    elif w.dtype == "f32":
        bound = F32_ABS
    else:
        bound = BF16_REL * max(np.max(np.abs(ref)), 1e-30)
    assert err <= bound, f"{what}: max err {err:.3e} > {bound:.3e}"
    return err


def _valid_topk(chosen, cand, scores, k, what):
    """One flagged row: `chosen` (GPU indices, -1 padded) must be a valid top-k
    of `cand` under `scores` (float64, same order as cand): right size,
    ascending and unique, inside the candidates, and no rejected candidate
    scoring above a chosen one by more than the 1e-3 relative tie window."""
    kk = min(k, len(cand))
    got = [int(c) for c in chosen if c >= 0]
    assert len(got) == kk and all(c == -1 for c in chosen[kk:]), (what, "size", chosen)
    assert all(a < b for a, b in zip(got, got[1:])), (what, "not ascending/unique", got)
    pos = {int(c): i for i, c in enumerate(cand)}
    assert all(c in pos for c in got), (what, "outside the candidate set", got)
    picked = np.zeros(len(cand), bool)
    picked[[pos[c] for c in got]] = True
    if picked.all() or not picked.any():
        return got
    lo, hi = scores[picked].min(), scores[~picked].max()
    assert lo >= hi - TIE_REL * max(abs(lo), abs(hi)), (what, "rejected beats chosen", lo, hi)
    return got


def check_selection(gpu_blk, gpu_grp, q64, bsum, gsum, q_begin, w, n_kv, what=""):
    """Selections against the oracle: bit-exact on every row the oracle does
    not flag as a near tie; on flagged rows the GPU's choice must be one of
    the valid answers at both levels (scored in float64 from the oracle's
    summaries).  Returns (flagged rows, flagged rows where the GPU differs)."""
    sb, sg, tie = oracle.route(q64, bsum, gsum, q_begin, w.topk_blocks, w.topk_groups, n_kv)
    gpu_blk, gpu_grp = np.asarray(gpu_blk), np.asarray(gpu_grp)
    for name, g, r in (("sel_blk", gpu_blk, sb), ("sel_grp", gpu_grp, sg)):
        bad = np.any(g != r, axis=-1) & ~tie
        assert not bad.any(), f"{what}{name}: {int(bad.sum())} unflagged rows differ, " \
                              f"first at {np.argwhere(bad)[0].tolist()}"
    G = q64.shape[1] // n_kv
    differ = 0
    for b, h, j in np.argwhere(tie):
        J = (q_begin + 64 * j) // 64
        qbar = q64[b, h * G:(h + 1) * G, 64 * j:64 * (j + 1)].reshape(-1, q64.shape[-1]).mean(0)
        blocks = _valid_topk(gpu_blk[b, h, j], np.arange(J), bsum[b, h, :J] @ qbar,
                             w.topk_blocks, f"{what}sel_blk{(b, h, j)}")
        groups = np.array([8 * c + i for c in blocks for i in range(8)], np.int64)
        _valid_topk(gpu_grp[b, h, j], groups, gsum[b, h, groups] @ qbar, w.topk_groups,
                    f"{what}sel_grp{(b, h, j)}")
        differ += int(np.any(gpu_grp[b, h, j] != sg[b, h, j]) or
                      np.any(gpu_blk[b, h, j] != sb[b, h, j]))
    return int(tie.sum()), differ


class Segmenter:
    """Runs a workload segment by segment on the GPU (HgaLayer) and, for the
    segments asked for, on the oracle with the same inputs."""

    def __init__(self, w, kv_heads=None, flags=0, causal=False):
        import torch
        from hierarchical_routed_sparse_hga_b200 import HgaLayer
        self.w = w
        self.causal = causal
        self.heads = list(range(w.n_kv_heads)) if kv_heads is None else list(kv_heads)
        G = w.group_heads
        self.q_heads = [h * G + g for h in self.heads for g in range(G)]
        k_np, v_np = synth.keys(w), synth.values(w)
        self.k64 = synth.widen(k_np[:, self.heads], w.dtype)
        self.v64 = synth.widen(v_np[:, self.heads], w.dtype)
        self.layer = HgaLayer(config_of(w, flags), w.ctx_len, w.seg_len,
                              k=to_device(k_np, w), v=to_device(v_np, w))
        # history before the first query-carrying segment is summarised up front
        first = w.segments()[0]
        if first:
            from hierarchical_routed_sparse_hga_b200 import hga_build_summaries
            hga_build_summaries(self.layer.cfg, self.layer.k, w.ctx_len, 0, first,
                                self.layer.gsum, self.layer.bsum)
            if causal:
                # the mean query of the block just before the first segment
                # (the earlier segment's queries)
                prev = first - w.seg_len
                self.layer.build_query_summaries(to_device(synth.queries(w, prev), w), prev)
        torch.cuda.synchronize()

    def run_segment(self, q_begin, backward=None):
        import torch
        w = self.w
        backward = w.backward if backward is None else backward
        q_np = synth.queries(w, q_begin)
        q = to_device(q_np, w)
        d_o = to_device(synth.douts(w, q_begin), w) if backward else None
        self.layer.segment(q, q_begin, d_o, causal=self.causal)
        torch.cuda.synchronize()
        L = self.layer
        hs, qs = self.heads, self.q_heads
        out = dict(q64=synth.widen(q_np[:, qs], w.dtype),
                   sel_blk=L.sel_blk[:, hs].cpu().numpy(), sel_grp=L.sel_grp[:, hs].cpu().numpy(),
                   o=to_f64(L.o[:, qs]), lse=to_f64(L.lse[:, qs]),
                   gsum=to_f64(L.gsum[:, hs]), bsum=to_f64(L.bsum[:, hs]),
                   qsum=to_f64(L.qsum[:, hs]))
        if backward:
            out.update(do64=synth.widen(synth.douts(w, q_begin)[:, qs], w.dtype),
                       dq=to_f64(L.dq[:, qs]), dk=to_f64(L.dk[:, hs]), dv=to_f64(L.dv[:, hs]))
        return out


def compare_segment(w, gpu, q_begin, n_kv, k64, v64, backward):
    """Oracle on the same inputs (heads already sliced); asserts parity."""
    T_end = q_begin + w.seg_len
    g_ref, b_ref = oracle.build_summaries(k64, 0, T_end)
    assert_close(gpu["gsum"][:, :, :T_end // 8], g_ref, w, "gsum", rel=SUMMARY_REL)
    assert_close(gpu["bsum"][:, :, :T_end // 64], b_ref, w, "bsum", rel=SUMMARY_REL)
    flagged, differ = check_selection(gpu["sel_blk"], gpu["sel_grp"], gpu["q64"], b_ref,
                                      g_ref, q_begin, w, n_kv)
    # attention is checked on the GPU's selection (equal to the oracle's on
    # every unflagged row, a valid top-k on the flagged ones)
    o, lse = oracle.attn_fwd(gpu["q64"], k64, v64, q_begin, gpu["sel_grp"], n_kv)
    assert_close(gpu["o"], o, w, "o")
    assert_close(gpu["lse"], lse, w, "lse", abs_=LSE_ABS)
    if backward:
        dq, dk, dv = oracle.attn_bwd(gpu["q64"], k64, v64, gpu["do64"], q_begin,
                                     gpu["sel_grp"], n_kv)
        assert_close(gpu["dq"], dq, w, "dq")
        assert_close(gpu["dk"], dk, w, "dk")
        assert_close(gpu["dv"], dv, w, "dv")
    return flagged, differ


def check_decode_selection(gpu_blk, gpu_grp, q_tok, bsum, gsum, pos, w, n_kv, what=""):
    """check_selection for decode steps ([B, Hkv, k] selections, one token per
    sequence at pos[b]).  Returns (flagged rows, flagged rows that differ)."""
    sb, sg, tie = oracle.decode_route(q_tok, bsum, gsum, pos, w.topk_blocks, w.topk_groups,
                                      n_kv)
    gpu_blk, gpu_grp = np.asarray(gpu_blk), np.asarray(gpu_grp)
    for name, g, r in (("sel_blk", gpu_blk, sb), ("sel_grp", gpu_grp, sg)):
        bad = np.any(g != r, axis=-1) & ~tie
        assert not bad.any(), f"{what}{name}: {int(bad.sum())} unflagged rows differ, " \
                              f"first at {np.argwhere(bad)[0].tolist()}"
    G = q_tok.shape[1] // n_kv
    differ = 0
    for b, h in np.argwhere(tie):
        J = int(pos[b]) // 64
        qbar = q_tok[b, h * G:(h + 1) * G].mean(0)
        blocks = _valid_topk(gpu_blk[b, h], np.arange(J), bsum[b, h, :J] @ qbar,
                             w.topk_blocks, f"{what}sel_blk{(b, h)}")
        groups = np.array([8 * c + i for c in blocks for i in range(8)], np.int64)
        _valid_topk(gpu_grp[b, h], groups, gsum[b, h, groups] @ qbar, w.topk_groups,
                    f"{what}sel_grp{(b, h)}")
        differ += int(np.any(gpu_grp[b, h] != sg[b, h]) or np.any(gpu_blk[b, h] != sb[b, h]))
    return int(tie.sum()), differ


def compare_segment_causal(w, gpu, q_prev_mean, q_begin, n_kv, k64, v64, backward):
    """Causal routing against the oracle: the summaries, the segment's
    resident block mean queries, the selections (routed with the previous
    block's mean query, q_prev_mean [B, Hkv, n_qb, d] from the oracle) and
    the attention on the GPU's selection."""
    T_end = q_begin + w.seg_len
    g_ref, b_ref = oracle.build_summaries(k64, 0, T_end)
    assert_close(gpu["bsum"][:, :, :T_end // 64], b_ref, w, "bsum", rel=SUMMARY_REL)
    J0 = q_begin // 64
    qs_ref = oracle.query_summaries(gpu["q64"], n_kv)
    assert_close(gpu["qsum"][:, :, J0:J0 + w.seg_len // 64], qs_ref, w, "qsum", rel=SUMMARY_REL)
    sb, sg, tie = oracle.route_causal(q_prev_mean, b_ref, g_ref, q_begin, w.seg_len // 64,
                                      w.topk_blocks, w.topk_groups)
    for name, g, r in (("sel_blk", gpu["sel_blk"], sb), ("sel_grp", gpu["sel_grp"], sg)):
        bad = np.any(g != r, axis=-1) & ~tie
        assert not bad.any(), f"causal {name}: {int(bad.sum())} unflagged rows differ"
    differ = 0
    for b, h, j in np.argwhere(tie):
        J = J0 + j
        qbar = q_prev_mean[b, h, j]
        blocks = _valid_topk(gpu["sel_blk"][b, h, j], np.arange(J), b_ref[b, h, :J] @ qbar,
                             w.topk_blocks, f"causal sel_blk{(b, h, j)}")
        groups = np.array([8 * c + i for c in blocks for i in range(8)], np.int64)
        _valid_topk(gpu["sel_grp"][b, h, j], groups, g_ref[b, h, groups] @ qbar, w.topk_groups,
                    f"causal sel_grp{(b, h, j)}")
        differ += int(np.any(gpu["sel_grp"][b, h, j] != sg[b, h, j]))
    o, lse = oracle.attn_fwd(gpu["q64"], k64, v64, q_begin, gpu["sel_grp"], n_kv)
    assert_close(gpu["o"], o, w, "o")
    assert_close(gpu["lse"], lse, w, "lse", abs_=LSE_ABS)
    if backward:
        dq, dk, dv = oracle.attn_bwd(gpu["q64"], k64, v64, gpu["do64"], q_begin,
                                     gpu["sel_grp"], n_kv)
        assert_close(gpu["dq"], dq, w, "dq")
        assert_close(gpu["dk"], dk, w, "dk")
        assert_close(gpu["dv"], dv, w, "dv")
    return int(tie.sum()), differ
