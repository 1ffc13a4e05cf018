"""The file (NVMe) tier's host side on the CPU: segments written with
hga_tier_write_segment and groups read back with hga_tier_read_groups, for
the unique history groups the oracle's tier_stage lists, must reproduce the
history rows bit for bit; attention of the oracle on the staged rows equals
attention on the whole context; bad lists and short files are rejected."""

import os
import tempfile

import numpy as np
import pytest

import oracle
import hierarchical_routed_sparse_hga_b200 as hga
from hierarchical_routed_sparse_hga_b200 import synth


def files(nbytes):
    d = tempfile.mkdtemp()
    fds = []
    for name in ("k.bin", "v.bin"):
        fd = os.open(os.path.join(d, name), os.O_RDWR | os.O_CREAT, 0o600)
        os.ftruncate(fd, nbytes)
        fds.append(fd)
    return fds


@pytest.fixture
def case():
    w = synth.custom(batch=2, n_q_heads=4, n_kv_heads=2, head_dim=16, ctx_len=640, seg_len=128,
                     topk_blocks=3, topk_groups=7, seed=51, first_seg=0)
    k, v = synth.keys(w), synth.values(w)          # float32 storage [B, Hkv, T, d]
    cfg = hga.Config(w.batch, w.n_q_heads, w.n_kv_heads, 64, w.topk_blocks, w.topk_groups,
                     hga.HGA_F32)
    return w, k, v, cfg


def widen_d(a, d=64):
    """The library's head_dim must be 64 or 128: pad the tiny case's rows."""
    out = np.zeros(a.shape[:-1] + (d,), a.dtype)
    out[..., :a.shape[-1]] = a
    return out


def test_write_then_read_groups_roundtrip(case):
    w, k, v, cfg = case
    k, v = widen_d(k), widen_d(v)
    B, H, T, d = k.shape
    fd_k, fd_v = files(k.nbytes)
    try:
        S = w.seg_len
        for s0 in range(0, T, S):                   # every segment appended in order
            hga.hga_tier_write_segment(cfg, fd_k, fd_v, T, s0, S,
                                       np.ascontiguousarray(k[:, :, s0:s0 + S]),
                                       np.ascontiguousarray(v[:, :, s0:s0 + S]), S, 3)
        q_begin = 512
        rng = np.random.default_rng(3)
        n_hist = q_begin // 8
        sel = np.full((B, H, 2, 7), -1, np.int32)
        for b in range(B):
            for h in range(H):
                for j in range(2):
                    # runs of consecutive groups and isolated ones, some shared
                    g = np.unique(np.concatenate([np.arange(10, 14), rng.integers(0, n_hist, 3)]))
                    sel[b, h, j, :len(g[:7])] = np.sort(g[:7])
        stage_cap = 64 * 8 + S
        uniq, _ = oracle.tier_stage(sel, q_begin, S, stage_cap)
        slot_cap = 16
        slot_group = np.zeros((B, H, slot_cap), np.int32)
        n_unique = np.zeros((B, H), np.int32)
        for b in range(B):
            for h in range(H):
                slot_group[b, h, :len(uniq[b][h])] = uniq[b][h]
                n_unique[b, h] = len(uniq[b][h])
        ks = np.full((B, H, stage_cap - S, d), np.nan, np.float32)
        vs = np.full_like(ks, np.nan)
        hga.hga_tier_read_groups(cfg, fd_k, fd_v, T, slot_group, n_unique, slot_cap, ks, vs,
                                 stage_cap - S, 4)
        for b in range(B):
            for h in range(H):
                u = uniq[b][h]
                rows = (u[:, None] * 8 + np.arange(8)[None, :]).reshape(-1)
                assert np.array_equal(ks[b, h, :len(rows)], k[b, h, rows])
                assert np.array_equal(vs[b, h, :len(rows)], v[b, h, rows])
                assert np.isnan(ks[b, h, len(rows):]).all()      # nothing else written
    finally:
        os.close(fd_k)
        os.close(fd_v)


def test_staged_rows_give_the_same_attention(case):
    # the oracle's attention on the rows read back equals it on the context
    w, k32, v32, cfg = case
    k, v = widen_d(k32), widen_d(v32)
    B, H, T, d = k.shape
    S, q_begin = w.seg_len, 512
    fd_k, fd_v = files(k.nbytes)
    try:
        hga.hga_tier_write_segment(cfg, fd_k, fd_v, T, 0, q_begin, np.ascontiguousarray(
            k[:, :, :q_begin]), np.ascontiguousarray(v[:, :, :q_begin]), q_begin, 2)
        k64, v64 = k32.astype(np.float64), v32.astype(np.float64)
        q = synth.widen(synth.queries(w, q_begin), "f32")
        g, bl = oracle.build_summaries(k64, 0, T)
        _, sg, _ = oracle.route(q, bl, g, q_begin, 3, 7, 2)
        stage_cap = ((min(2 * 7, q_begin // 8) * 8 + 63) // 64) * 64 + S
        uniq, sel_st = oracle.tier_stage(sg, q_begin, S, stage_cap)
        slot_cap = 14
        slot_group = np.zeros((B, H, slot_cap), np.int32)
        n_unique = np.array([[len(uniq[b][h]) for h in range(H)] for b in range(B)], np.int32)
        for b in range(B):
            for h in range(H):
                slot_group[b, h, :n_unique[b, h]] = uniq[b][h]
        ks = np.zeros((B, H, stage_cap, d), np.float32)
        vs = np.zeros_like(ks)
        hga.hga_tier_read_groups(cfg, fd_k, fd_v, T, slot_group, n_unique, slot_cap, ks, vs,
                                 stage_cap, 3)
        ks[:, :, stage_cap - S:] = k[:, :, q_begin:]
        vs[:, :, stage_cap - S:] = v[:, :, q_begin:]
        o1, l1 = oracle.attn_fwd(q, k64, v64, q_begin, sg, 2)
        o2, l2 = oracle.attn_fwd(q, ks[..., :16].astype(np.float64),
                                 vs[..., :16].astype(np.float64), stage_cap - S, sel_st, 2)
        assert np.allclose(o1, o2, rtol=0, atol=1e-13) and np.allclose(l1, l2, rtol=0, atol=1e-13)
    finally:
        os.close(fd_k)
        os.close(fd_v)


def test_file_tier_rejects_bad_lists_and_short_files(case):
    w, k, v, cfg = case
    k, v = widen_d(k), widen_d(v)
    B, H, T, d = k.shape
    fd_k, fd_v = files(k.nbytes // 2)                # files cover only half the context
    try:
        ks = np.zeros((B, H, 64, d), np.float32)
        vs = np.zeros_like(ks)
        sg = np.zeros((B, H, 4), np.int32)

        def status(slot_group, n_unique, fdk=fd_k):
            with pytest.raises(hga.HgaError) as e:
                hga.hga_tier_read_groups(cfg, fdk, fd_v, T, slot_group, n_unique, 4, ks, vs,
                                         64, 2)
            return e.value.status

        n = np.ones((B, H), np.int32)
        assert status(np.full_like(sg, T // 8), n) == hga.HGA_ERR_INVALID_ARG   # beyond ctx
        assert status(sg, np.full((B, H), 5, np.int32)) == hga.HGA_ERR_INVALID_ARG  # > slot_cap
        assert status(np.full_like(sg, 70), n) == hga.HGA_ERR_IO                # past EOF
        assert status(sg, n, fdk=-1) == hga.HGA_ERR_INVALID_ARG
    finally:
        os.close(fd_k)
        os.close(fd_v)
