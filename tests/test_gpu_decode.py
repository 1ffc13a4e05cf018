"""Decode (one new token per sequence) through the C ABI against the oracle.

Selections are compared bit-exactly except on rows the oracle flags as near
ties, where the GPU's choice must be a valid top-k; outputs within 2e-2 of the
tensor's max |oracle| (bf16) or 1e-4 absolute (float32); LSE 1e-4 absolute.
"""

import numpy as np
import pytest

import oracle
from hierarchical_routed_sparse_hga_b200 import synth

from hga_testlib import assert_close, check_decode_selection, config_of, to_device, to_f64

pytestmark = pytest.mark.gpu


def run_decode(w, positions, heads=None):
    """Runs hga_decode on workload w's context at the given positions and
    checks it against the oracle on the KV heads `heads` (default: all)."""
    import torch
    from hierarchical_routed_sparse_hga_b200 import hga_build_summaries, hga_decode
    heads = list(range(w.n_kv_heads)) if heads is None else heads
    G = w.group_heads
    q_heads = [h * G + g for h in heads for g in range(G)]
    cfg = config_of(w)
    dev = torch.device("cuda", 0)
    k_np = synth.keys(w, heads)
    v_np = synth.values(w, heads)
    shape = (w.batch, w.n_kv_heads, w.ctx_len, w.head_dim)
    tdt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    k = torch.zeros(shape, dtype=tdt, device=dev)
    v = torch.zeros(shape, dtype=tdt, device=dev)
    k[:, heads] = to_device(k_np, w)
    v[:, heads] = to_device(v_np, w)
    gsum = torch.zeros((w.batch, w.n_kv_heads, w.ctx_len // 8, w.head_dim), device=dev)
    bsum = torch.zeros((w.batch, w.n_kv_heads, w.ctx_len // 64, w.head_dim), device=dev)
    hga_build_summaries(cfg, k, w.ctx_len, 0, w.ctx_len, gsum, bsum)
    q_np = synth.decode_queries(w, positions)
    q = to_device(q_np, w)
    pos = torch.tensor(positions, dtype=torch.int64, device=dev)
    sel_blk = torch.full((w.batch, w.n_kv_heads, w.topk_blocks), -9, dtype=torch.int32,
                         device=dev)
    sel_grp = torch.full((w.batch, w.n_kv_heads, w.topk_groups), -9, dtype=torch.int32,
                         device=dev)
    o = torch.zeros((w.batch, w.n_q_heads, w.head_dim), dtype=tdt, device=dev)
    lse = torch.zeros((w.batch, w.n_q_heads), device=dev)
    hga_decode(cfg, q, k, v, w.ctx_len, pos, bsum, gsum, sel_blk, sel_grp, o, lse)
    torch.cuda.synchronize()
    k64, v64 = synth.widen(k_np, w.dtype), synth.widen(v_np, w.dtype)
    q64 = synth.widen(q_np, w.dtype)[:, q_heads]
    g_ref, b_ref = oracle.build_summaries(k64, 0, w.ctx_len)
    sb = sel_blk[:, heads].cpu().numpy()
    sg = sel_grp[:, heads].cpu().numpy()
    flagged, differ = check_decode_selection(sb, sg, q64, b_ref, g_ref, positions, w, len(heads))
    print(f"[{w.name} decode] near-tie rows: {flagged} of {w.batch * len(heads)} flagged, "
          f"{differ} with another valid selection on the GPU")
    o_ref, lse_ref = oracle.decode_attn(q64, k64, v64, positions, sg, len(heads))
    assert_close(to_f64(o[:, q_heads]), o_ref, w, "o")
    assert_close(to_f64(lse[:, q_heads]), lse_ref, w, "lse", abs_=1e-4)
    return sel_blk, sel_grp, o, lse


def test_decode_qwen3_shape():
    # the first block (no candidates), block boundaries on both sides, the
    # last token of the context
    w = synth.custom(batch=6, n_q_heads=32, n_kv_heads=8, head_dim=128, ctx_len=8192,
                     seg_len=2048, topk_blocks=16, topk_groups=64, dtype="bf16", scaled=True,
                     rope_base=1e6, seed=31)
    run_decode(w, [8191, 5, 4096, 4095, 64 * 77 + 40, 64 * 16])


def test_decode_qwen3_131k_sampled_heads():
    # the 131072-token context, two KV heads checked (the others hold zeros)
    w = synth.custom(batch=2, n_q_heads=32, n_kv_heads=8, head_dim=128, ctx_len=131072,
                     seg_len=2048, topk_blocks=16, topk_groups=64, dtype="bf16", scaled=True,
                     rope_base=1e6, seed=33)
    run_decode(w, [131071, 70000], heads=[1, 6])


@pytest.mark.parametrize("kw", [
    # float32, d = 64, G = 1, ragged k_g, more k_b than candidates
    dict(batch=3, n_q_heads=2, n_kv_heads=2, head_dim=64, ctx_len=1024, topk_blocks=5,
         topk_groups=13, dtype="f32"),
    # G = 8, everything selected (dense)
    dict(batch=2, n_q_heads=8, n_kv_heads=1, head_dim=128, ctx_len=640, topk_blocks=64,
         topk_groups=256, dtype="bf16"),
    # G = 2, bf16, d = 64
    dict(batch=2, n_q_heads=4, n_kv_heads=2, head_dim=64, ctx_len=2048, topk_blocks=8,
         topk_groups=32, dtype="bf16", scaled=True, rope_base=1e6),
])
def test_decode_custom_shapes(kw):
    w = synth.custom(seg_len=64, seed=12, **kw)
    T = w.ctx_len
    positions = [T - 1, 64 * 3 + 1, 63][:w.batch]
    run_decode(w, positions)


def test_decode_block_boundary_positions():
    # the token alone in its block: the very first token (no candidates, it
    # attends to itself only), the first token of block 1 (one candidate),
    # and two later block starts
    w = synth.custom(batch=4, n_q_heads=4, n_kv_heads=2, head_dim=128, ctx_len=1024,
                     seg_len=64, topk_blocks=4, topk_groups=16, dtype="bf16", scaled=True,
                     rope_base=1e6, seed=14)
    run_decode(w, [0, 64, 64 * 7, 1024 - 64])


def test_decode_is_deterministic():
    w = synth.custom(batch=2, n_q_heads=32, n_kv_heads=8, head_dim=128, ctx_len=4096,
                     seg_len=2048, topk_blocks=16, topk_groups=64, dtype="bf16", scaled=True,
                     rope_base=1e6, seed=35)
    a = run_decode(w, [4095, 3000])
    b = run_decode(w, [4095, 3000])
    for x, y in zip(a, b):
        assert bool((x == y).all())


def test_decode_position_out_of_range_is_latched():
    import torch
    from hierarchical_routed_sparse_hga_b200 import (HGA_BF16, HGA_ERR_DEVICE_CHECK, HGA_OK,
                                                     Config, hga_decode,
                                                     hga_get_device_status)
    dev = torch.device("cuda", 0)
    cfg = Config(2, 8, 2, 128, 4, 16, HGA_BF16)
    T = 512
    k = torch.zeros((2, 2, T, 128), dtype=torch.bfloat16, device=dev)
    gsum = torch.zeros((2, 2, T // 8, 128), device=dev)
    bsum = torch.zeros((2, 2, T // 64, 128), device=dev)
    q = torch.zeros((2, 8, 128), dtype=torch.bfloat16, device=dev)
    o = torch.full((2, 8, 128), 7.0, dtype=torch.bfloat16, device=dev)
    lse = torch.full((2, 8), 7.0, device=dev)
    pos = torch.tensor([T, 100], dtype=torch.int64, device=dev)
    hga_decode(cfg, q, k, k, T, pos, bsum, gsum, None, None, o, lse)
    assert hga_get_device_status() == HGA_ERR_DEVICE_CHECK
    assert hga_get_device_status() == HGA_OK
    assert bool((o[0] == 7.0).all()) and bool((lse[0] == 7.0).all())   # untouched
    assert bool((lse[1] != 7.0).all())                                   # the valid one ran
