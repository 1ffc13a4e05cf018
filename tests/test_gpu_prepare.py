"""The upstream pass (hga_prepare_segment) and routing from the resident
summaries (hga_route_summarized) through the C ABI against the oracle.

RoPE is computed in float32 on the GPU and in float64 by the oracle, and
both round to bf16: elements may differ by one bf16 unit in the last place
where the exact value sits next to a rounding boundary; that share must stay
below 1e-3.  Everything downstream (summaries, block mean queries, routing,
attention) is checked against the oracle run on the GPU's stored Q and K,
with the usual tolerances and near-tie rule."""

import numpy as np
import pytest

import oracle
from hierarchical_routed_sparse_hga_b200 import synth

from hga_testlib import (SUMMARY_REL, assert_close, check_selection, config_of,
                         compare_segment_causal, to_device, to_f64)

pytestmark = pytest.mark.gpu


def rope_mismatch(gpu, ref, x_in, what):
    """The GPU's stored values against the oracle's: each element within one
    bf16 step of its value plus the float32 rounding bound of the rotation
    (a few units of 2^-24 of the rotated pair's magnitude |x_i| + |x_{i+d/2}|,
    which matters where the rotation cancels toward zero); and rare."""
    gpu, ref = np.asarray(gpu), np.asarray(ref)
    half = x_in.shape[-1] // 2
    pair = np.abs(x_in[..., :half]) + np.abs(x_in[..., half:])
    mag = np.concatenate([pair, pair], axis=-1)
    step = np.ldexp(1.0, np.frexp(np.maximum(np.abs(gpu), np.abs(ref)))[1] - 8)
    tol = step + 16 * 2.0 ** -24 * mag
    err = np.abs(gpu - ref)
    worst = np.unravel_index(np.argmax(err - tol), err.shape)
    assert np.all(err <= tol), (what, worst, gpu[worst], ref[worst], mag[worst])
    frac = float((gpu != ref).mean())
    assert frac < 1e-3, (what, frac)
    return frac


def run_prepare(w, check_segments, causal=False, rope=True):
    import torch
    from hierarchical_routed_sparse_hga_b200 import HgaLayer
    cfg = config_of(w)
    dev = torch.device("cuda", 0)
    L = HgaLayer(cfg, w.ctx_len, w.seg_len, device=dev)
    G, S = w.group_heads, w.seg_len
    base = w.rope_base if rope else None
    q_out = torch.empty((w.batch, w.n_q_heads, S, w.head_dim), dtype=L.k.dtype, device=dev)
    k_ref = np.zeros((w.batch, w.n_kv_heads, w.ctx_len, w.head_dim))
    v_ref = np.zeros_like(k_ref)
    prev_mean = None
    for s0 in range(0, w.ctx_len, S):
        qp, kp, vp = synth.projections(w, s0)
        L.prepare(to_device(qp, w), to_device(kp, w), to_device(vp, w),
                  w.n_q_heads * w.head_dim, w.n_kv_heads * w.head_dim, s0, base, q_out)
        torch.cuda.synchronize()
        q64, k64, v64, g_o, b_o, qs_o = oracle.prepare_segment(
            synth.widen(qp, w.dtype), synth.widen(kp, w.dtype), synth.widen(vp, w.dtype), s0,
            base, w.n_kv_heads, w.dtype)
        q_gpu = to_f64(q_out)
        k_gpu = to_f64(L.k[:, :, s0:s0 + S])
        x_q = np.transpose(synth.widen(qp, w.dtype), (0, 2, 1, 3))
        x_k = np.transpose(synth.widen(kp, w.dtype), (0, 2, 1, 3))
        rope_mismatch(q_gpu, q64, x_q, "q")
        rope_mismatch(k_gpu, k64, x_k, "k")
        assert np.array_equal(to_f64(L.v[:, :, s0:s0 + S]), v64)
        k_ref[:, :, s0:s0 + S] = k_gpu
        v_ref[:, :, s0:s0 + S] = v64
        # summaries and block means of the GPU's stored values
        g_r, b_r = oracle.build_summaries(k_gpu, 0, S)
        assert_close(to_f64(L.gsum[:, :, s0 // 8:(s0 + S) // 8]), g_r, w, "gsum", rel=SUMMARY_REL)
        assert_close(to_f64(L.bsum[:, :, s0 // 64:(s0 + S) // 64]), b_r, w, "bsum",
                     rel=SUMMARY_REL)
        qs_r = oracle.query_summaries(q_gpu, w.n_kv_heads)
        assert_close(to_f64(L.qsum[:, :, s0 // 64:(s0 + S) // 64]), qs_r, w, "qsum",
                     rel=SUMMARY_REL)
        if s0 in check_segments:
            L.route_summarized(s0, causal)
            L.forward(q_out, s0)
            torch.cuda.synchronize()
            sel_blk = L.sel_blk.cpu().numpy()
            sel_grp = L.sel_grp.cpu().numpy()
            g_all, b_all = oracle.build_summaries(k_ref, 0, s0 + S)
            gpu = dict(q64=q_gpu, sel_blk=sel_blk, sel_grp=sel_grp, o=to_f64(L.o),
                       lse=to_f64(L.lse), bsum=to_f64(L.bsum), qsum=to_f64(L.qsum))
            if causal:
                first = prev_mean if prev_mean is not None else np.zeros_like(qs_r[:, :, 0])
                q_prev = np.concatenate([first[:, :, None], qs_r[:, :, :-1]], axis=2)
                compare_segment_causal(w, gpu, q_prev, s0, w.n_kv_heads, k_ref, v_ref, False)
            else:
                check_selection(sel_blk, sel_grp, q_gpu, b_all, g_all, s0, w, w.n_kv_heads)
                o, lse = oracle.attn_fwd(q_gpu, k_ref, v_ref, s0, sel_grp, w.n_kv_heads)
                assert_close(gpu["o"], o, w, "o")
                assert_close(gpu["lse"], lse, w, "lse", abs_=1e-4)
        prev_mean = qs_r[:, :, -1]


def qwen3(ctx, seed=41, **kw):
    return synth.custom(n_q_heads=32, n_kv_heads=8, head_dim=128, ctx_len=ctx, seg_len=2048,
                        topk_blocks=16, topk_groups=64, dtype="bf16", scaled=True,
                        rope_base=1e6, seed=seed, **kw)


def test_prepare_and_route_from_summaries_qwen3_16k():
    run_prepare(qwen3(16384), check_segments={2048, 14336})


def test_prepare_and_causal_route_from_summaries():
    run_prepare(qwen3(8192, seed=42), check_segments={2048, 6144}, causal=True)


def test_prepare_long_context_three_kernel_routing():
    # the last segment of 36864 tokens: routing past 512 candidate blocks
    run_prepare(qwen3(36864, seed=43), check_segments={34816})


def test_prepare_without_rope_float32_is_layout_only():
    import torch
    w = synth.custom(batch=2, n_q_heads=4, n_kv_heads=2, head_dim=64, ctx_len=512, seg_len=256,
                     topk_blocks=3, topk_groups=9, dtype="f32", seed=44)
    run_prepare(w, check_segments={256}, rope=False)
    from hierarchical_routed_sparse_hga_b200 import HgaLayer
    L = HgaLayer(config_of(w), w.ctx_len, w.seg_len)
    qp, kp, vp = synth.projections(w, 256)
    q_out = torch.empty((2, 4, 256, 64), device="cuda")
    L.prepare(to_device(qp, w), to_device(kp, w), to_device(vp, w), 4 * 64, 2 * 64, 256, None,
              q_out)
    torch.cuda.synchronize()
    assert np.array_equal(q_out.cpu().numpy(), np.transpose(qp, (0, 2, 1, 3)))
    assert np.array_equal(L.k[:, :, 256:].cpu().numpy(), np.transpose(kp, (0, 2, 1, 3)))


def test_prepare_from_fused_qkv_rows():
    # one [B, S, (Hq + 2 Hkv) * d] projection output, K and V pointing into it
    import torch
    from hierarchical_routed_sparse_hga_b200 import HgaLayer
    w = qwen3(4096, seed=45)
    L1 = HgaLayer(config_of(w), w.ctx_len, w.seg_len)
    L2 = HgaLayer(config_of(w), w.ctx_len, w.seg_len)
    qp, kp, vp = (to_device(t, w) for t in synth.projections(w, 2048))
    B, S = w.batch, w.seg_len
    fused = torch.cat([qp.reshape(B, S, -1), kp.reshape(B, S, -1), vp.reshape(B, S, -1)], dim=2)
    stride = fused.shape[2]
    qo1 = torch.empty((B, 32, S, 128), dtype=torch.bfloat16, device="cuda")
    qo2 = torch.empty_like(qo1)
    L1.prepare(qp, kp, vp, 32 * 128, 8 * 128, 2048, 1e6, qo1)
    nq = 32 * 128
    L2.prepare(fused, fused.data_ptr() + nq * 2, fused.data_ptr() + (nq + 8 * 128) * 2, stride,
               stride, 2048, 1e6, qo2)
    torch.cuda.synchronize()
    assert torch.equal(qo1, qo2) and torch.equal(L1.k, L2.k) and torch.equal(L1.v, L2.v)
    assert torch.equal(L1.gsum, L2.gsum) and torch.equal(L1.qsum, L2.qsum)
