"""Strictly causal routing through the C ABI against the oracle: each query
block routed with the mean query of the 64 tokens before it.  Selections
bit-exact except on near-tie rows (where the GPU's must be a valid top-k),
attention forward and backward on the GPU's selection within the usual
tolerances, the resident block mean queries within 1e-5 relative."""

import dataclasses

import numpy as np
import pytest

import oracle
from hierarchical_routed_sparse_hga_b200 import synth

from hga_testlib import Segmenter, compare_segment_causal

pytestmark = pytest.mark.gpu

WL = synth.workloads()


def run_causal(w, segments=None, kv_heads=None):
    seg = Segmenter(w, kv_heads=kv_heads, causal=True)
    n_kv = len(seg.heads)
    want = set(w.segments() if segments is None else segments)
    prev_mean = None            # oracle mean query of the block before each segment
    first = w.segments()[0]
    if first:
        q_prev = synth.widen(synth.queries(w, first - w.seg_len)[:, seg.q_heads], w.dtype)
        prev_mean = oracle.query_summaries(q_prev, n_kv)[:, :, -1]
    flagged = differ = rows = 0
    for q_begin in w.segments():
        out = seg.run_segment(q_begin)
        qs = oracle.query_summaries(out["q64"], n_kv)        # [B, Hkv, n_qb, d]
        first_row = prev_mean if prev_mean is not None else np.zeros_like(qs[:, :, 0])
        q_prev_mean = np.concatenate([first_row[:, :, None], qs[:, :, :-1]], axis=2)
        if q_begin in want:
            f, dif = compare_segment_causal(w, out, q_prev_mean, q_begin, n_kv, seg.k64,
                                            seg.v64, w.backward)
            flagged += f
            differ += dif
            rows += w.batch * n_kv * (w.seg_len // 64)
        prev_mean = qs[:, :, -1]
    print(f"[{w.name} causal] near-tie rows: {flagged} of {rows} flagged, "
          f"{differ} with another valid selection on the GPU")
    assert differ <= max(2, rows // 20)


def test_causal_qwen3_fwdbwd_16k_all_segments():
    # the benchmark's workload with causal routing: 8 segments from token 0
    run_causal(WL["qwen3_fwdbwd_16k"])


def test_causal_routing_at_131k():
    # the last segment of the 131072-token context (2047 candidate blocks),
    # two KV heads checked
    w = dataclasses.replace(WL["qwen3_fwdbwd_16k"], name="qwen3_fwd_131k_last",
                            ctx_len=131072, first_seg=63, backward=False)
    run_causal(w, kv_heads=[1, 4])


def test_causal_history_before_first_segment():
    # one segment after 14336 history tokens: the block before it comes from
    # hga_build_query_summaries over the previous segment's queries
    run_causal(WL["qwen3_fwd_16k"])


def test_causal_long_context_three_kernel_routing():
    # past 512 candidate blocks (the three-kernel routing), last segment of
    # a 36864-token context, two KV heads checked
    w = dataclasses.replace(WL["qwen3_fwdbwd_16k"], name="qwen3_fwdbwd_36k_last",
                            ctx_len=36864, first_seg=17)
    run_causal(w, kv_heads=[2, 7])


@pytest.mark.parametrize("kw", [
    dict(n_q_heads=4, n_kv_heads=1, head_dim=64, ctx_len=576, seg_len=192, topk_blocks=5,
         topk_groups=13, dtype="f32", first_seg=0),
    dict(batch=2, n_q_heads=8, n_kv_heads=2, head_dim=128, ctx_len=1024, seg_len=256,
         topk_blocks=3, topk_groups=12, dtype="bf16", scaled=True, rope_base=1e6, first_seg=0),
])
def test_causal_custom_shapes(kw):
    run_causal(synth.custom(seed=13, **kw))


def test_causal_selection_ignores_later_queries():
    # the selections of a segment's first half do not change when the
    # queries of its second half do (they reach only later query blocks)
    import torch
    w = WL["qwen3_fwdbwd_16k"]
    from hga_testlib import to_device
    seg = Segmenter(w, causal=True)
    L = seg.layer
    for q_begin in w.segments()[:-1]:
        seg.run_segment(q_begin, backward=False)
    q_begin = w.segments()[-1]
    q = to_device(synth.queries(w, q_begin), w)
    L.summarize(q_begin)
    L.route_causal(q, q_begin)
    torch.cuda.synchronize()
    a = L.sel_grp.clone()
    q2 = q.clone()
    q2[:, :, 1024:] = -q2[:, :, 1024:]
    L.route_causal(q2, q_begin)
    torch.cuda.synchronize()
    assert torch.equal(a[:, :, :17], L.sel_grp[:, :, :17])      # blocks 0..16 use rows < 1024
    assert not torch.equal(a[:, :, 17:], L.sel_grp[:, :, 17:])
