"""Host tier (history K/V in pinned host memory) against the all-HBM path and
the oracle's dedup/remap: bit-identical outputs, exact indices."""

import numpy as np
import pytest

import oracle
from hierarchical_routed_sparse_hga_b200 import synth

from hga_testlib import config_of, to_device

pytestmark = pytest.mark.gpu


def run_tier_vs_hbm(w):
    import torch
    from hierarchical_routed_sparse_hga_b200 import HgaLayer, HgaTieredLayer
    k_np, v_np = synth.keys(w), synth.values(w)
    k_dev, v_dev = to_device(k_np, w), to_device(v_np, w)
    cfg = config_of(w)
    hbm = HgaLayer(cfg, w.ctx_len, w.seg_len, k=k_dev, v=v_dev)
    tier = HgaTieredLayer(cfg, w.ctx_len, w.seg_len)
    S = w.seg_len
    for q_begin in w.segments():
        q = to_device(synth.queries(w, q_begin), w)
        do = to_device(synth.douts(w, q_begin), w)
        hbm.segment(q, q_begin, do)
        tier.active_k().copy_(k_dev[:, :, q_begin:q_begin + S])
        tier.active_v().copy_(v_dev[:, :, q_begin:q_begin + S])
        tier.segment(q, q_begin, do)
        torch.cuda.synchronize()
        sel = hbm.sel_grp.cpu().numpy()
        assert np.array_equal(tier.sel_grp.cpu().numpy(), sel)
        uniq, sel_st = oracle.tier_stage(sel, q_begin, S, tier.stage_cap)
        assert np.array_equal(tier.sel_stage.cpu().numpy(), sel_st), q_begin
        counts = tier.n_unique.cpu().numpy()
        ks = tier.k_stage.cpu()
        for b in range(w.batch):
            for h in range(w.n_kv_heads):
                u = uniq[b][h]
                assert counts[b, h] == len(u)
                rows = (u[:, None] * 8 + np.arange(8)[None, :]).reshape(-1)
                assert torch.equal(ks[b, h, :len(rows)], k_dev[b, h, rows].cpu())
        for name in ("o", "lse", "dq", "dk", "dv"):
            assert torch.equal(getattr(tier, name), getattr(hbm, name)), (name, q_begin)
    # the host history now holds the whole sequence
    assert torch.equal(tier.k_host.to(k_dev.device), k_dev)


def test_tier_bf16_tensor_core_path():
    run_tier_vs_hbm(synth.custom(batch=2, n_q_heads=8, n_kv_heads=2, head_dim=128,
                                 ctx_len=3072, seg_len=1024, topk_blocks=4, topk_groups=12,
                                 dtype="bf16", scaled=True, rope_base=1e6, seed=13))


def test_tier_f32_path():
    run_tier_vs_hbm(synth.custom(batch=1, n_q_heads=2, n_kv_heads=1, head_dim=64,
                                 ctx_len=1536, seg_len=512, topk_blocks=3, topk_groups=10,
                                 dtype="f32", seed=14))


def test_tier_rejects_pageable_host_memory():
    import torch
    from hierarchical_routed_sparse_hga_b200 import (HGA_ERR_INVALID_ARG, HgaError,
                                                     HgaTieredLayer, hga_tier_gather)
    w = synth.custom(n_q_heads=4, n_kv_heads=1, head_dim=128, ctx_len=1024, seg_len=512,
                     topk_blocks=2, topk_groups=8, dtype="bf16")
    tier = HgaTieredLayer(config_of(w), w.ctx_len, w.seg_len)
    pageable = np.zeros(tier.k_host.numel(), np.uint16)
    with pytest.raises(HgaError) as e:
        hga_tier_gather(tier.cfg, pageable.ctypes.data, pageable.ctypes.data, w.ctx_len, 512,
                        w.seg_len, tier.sel_grp, tier.k_stage, tier.v_stage, tier.stage_cap,
                        tier.sel_stage, tier.n_unique, tier.tier_ws)
    assert e.value.status == HGA_ERR_INVALID_ARG
    torch.cuda.synchronize()


def test_file_tier_equals_hbm_path(tmp_path):
    # history K/V in files: every segment's selected groups read back from
    # the files give the same selections and bit-identical outputs as the
    # all-HBM path, and the files end up holding the whole sequence
    import os

    import torch
    from hierarchical_routed_sparse_hga_b200 import HgaFileTieredLayer, HgaLayer
    w = synth.custom(batch=2, n_q_heads=8, n_kv_heads=2, head_dim=128, ctx_len=3072,
                     seg_len=512, topk_blocks=4, topk_groups=16, dtype="bf16", scaled=True,
                     rope_base=1e6, seed=52, first_seg=0)
    k_np, v_np = synth.keys(w), synth.values(w)
    k_dev, v_dev = to_device(k_np, w), to_device(v_np, w)
    cfg = config_of(w)
    hbm = HgaLayer(cfg, w.ctx_len, w.seg_len, k=k_dev, v=v_dev)
    nbytes = k_dev.numel() * k_dev.element_size()
    fds = []
    for name in ("k.bin", "v.bin"):
        fd = os.open(str(tmp_path / name), os.O_RDWR | os.O_CREAT, 0o600)
        os.ftruncate(fd, nbytes)
        fds.append(fd)
    try:
        tier = HgaFileTieredLayer(cfg, w.ctx_len, w.seg_len, fds[0], fds[1], n_threads=4)
        S = w.seg_len
        for q_begin in w.segments():
            q = to_device(synth.queries(w, q_begin), w)
            do = to_device(synth.douts(w, q_begin), w)
            hbm.segment(q, q_begin, do)
            tier.active_k().copy_(k_dev[:, :, q_begin:q_begin + S])
            tier.active_v().copy_(v_dev[:, :, q_begin:q_begin + S])
            tier.segment(q, q_begin, do)
            torch.cuda.synchronize()
            sel = hbm.sel_grp.cpu().numpy()
            assert np.array_equal(tier.sel_grp.cpu().numpy(), sel)
            _, sel_st = oracle.tier_stage(sel, q_begin, S, tier.stage_cap)
            assert np.array_equal(tier.sel_stage.cpu().numpy(), sel_st), q_begin
            for name in ("o", "lse", "dq", "dk", "dv"):
                assert torch.equal(getattr(tier, name), getattr(hbm, name)), (name, q_begin)
        assert tier.bytes_read > 0
        for fd, ref in zip(fds, (k_np, v_np)):
            raw = os.pread(fd, nbytes, 0)
            assert np.array_equal(np.frombuffer(raw, np.uint16).reshape(ref.shape), ref)
    finally:
        for fd in fds:
            os.close(fd)
