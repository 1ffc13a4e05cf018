"""Segment-wise driver of the HGA hot path over one layer's context.

HgaLayer owns the device buffers of one attention layer (whole-context K/V,
the resident group/block summaries, the route and backward workspaces and the
per-segment outputs), all allocated once with torch, and runs one segment as

    hga_build_summaries -> hga_route -> hga_attn_fwd [-> hga_attn_bwd]

through the C ABI.  The K/V of the active segment live at their final place in
the context buffer, so "appending the segment to history" after the step is
just moving q_begin forward: later segments read the same tokens, detached
(the backward writes gradients for the active segment's keys only).
"""

from __future__ import annotations

import torch

from . import _lib
from ._lib import HGA_BF16, HGA_F32, Config

_TORCH_DTYPE = {HGA_BF16: torch.bfloat16, HGA_F32: torch.float32}


class HgaLayer:
    def __init__(self, cfg: Config, ctx_cap: int, seg_len: int, device="cuda",
                 k=None, v=None):
        self.cfg = cfg
        self.ctx_cap = ctx_cap
        self.seg_len = seg_len
        self.device = torch.device(device)
        dt = _TORCH_DTYPE[cfg.dtype]
        B, Hq, Hkv, d = cfg.batch, cfg.n_q_heads, cfg.n_kv_heads, cfg.head_dim
        n_qb = seg_len // 64
        shape_kv = (B, Hkv, ctx_cap, d)
        self.k = k if k is not None else torch.zeros(shape_kv, dtype=dt, device=self.device)
        self.v = v if v is not None else torch.zeros(shape_kv, dtype=dt, device=self.device)
        self.gsum = torch.zeros((B, Hkv, ctx_cap // 8, d), dtype=torch.float32,
                                device=self.device)
        self.bsum = torch.zeros((B, Hkv, ctx_cap // 64, d), dtype=torch.float32,
                                device=self.device)
        ws = max(_lib.hga_route_workspace_size(cfg, seg_len, ctx_cap - seg_len), 256)
        self.route_ws = torch.empty(ws, dtype=torch.uint8, device=self.device)
        self.bwd_ws = torch.empty(max(_lib.hga_attn_bwd_workspace_size(cfg, seg_len), 256),
                                  dtype=torch.uint8, device=self.device)
        self.sel_blk = torch.empty((B, Hkv, n_qb, cfg.topk_blocks), dtype=torch.int32,
                                   device=self.device)
        self.sel_grp = torch.empty((B, Hkv, n_qb, cfg.topk_groups), dtype=torch.int32,
                                   device=self.device)
        self.o = torch.empty((B, Hq, seg_len, d), dtype=dt, device=self.device)
        self.lse = torch.empty((B, Hq, seg_len), dtype=torch.float32, device=self.device)
        self.dq = torch.empty_like(self.o)
        self.dk = torch.empty((B, Hkv, seg_len, d), dtype=dt, device=self.device)
        self.dv = torch.empty_like(self.dk)

    # -- the four calls of one segment ------------------------------------
    def summarize(self, q_begin: int, stream=None):
        _lib.hga_build_summaries(self.cfg, self.k, self.ctx_cap, q_begin,
                                 q_begin + self.seg_len, self.gsum, self.bsum, stream)

    def route(self, q, q_begin: int, stream=None):
        _lib.hga_route(self.cfg, q, q_begin, self.seg_len, self.ctx_cap, self.bsum,
                       self.gsum, self.sel_blk, self.sel_grp, self.route_ws, stream=stream)

    def forward(self, q, q_begin: int, stream=None):
        _lib.hga_attn_fwd(self.cfg, q, self.k, self.v, self.ctx_cap, q_begin, self.seg_len,
                          self.sel_grp, self.o, self.lse, stream)

    def backward(self, q, d_o, q_begin: int, stream=None):
        _lib.hga_attn_bwd(self.cfg, q, self.k, self.v, self.ctx_cap, q_begin, self.seg_len,
                          self.sel_grp, self.o, self.lse, d_o, self.dq, self.dk, self.dv,
                          self.bwd_ws, stream=stream)

    def segment(self, q, q_begin: int, d_o=None, stream=None):
        """One segment: summaries, routing, forward and (if d_o) backward."""
        self.summarize(q_begin, stream)
        self.route(q, q_begin, stream)
        self.forward(q, q_begin, stream)
        if d_o is not None:
            self.backward(q, d_o, q_begin, stream)
