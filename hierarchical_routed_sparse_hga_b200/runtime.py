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
        # resident mean query of every block, for causal routing
        self.qsum = torch.zeros((B, Hkv, ctx_cap // 64, d), dtype=torch.float32,
                                device=self.device)
        ws = max(_lib.hga_route_workspace_size(cfg, seg_len, ctx_cap - seg_len), 256)
        self.route_ws = torch.empty(ws, dtype=torch.uint8, device=self.device)
        # zeroed once: hga_attn_fwd_bwd's completion flags live in it
        self.bwd_ws = torch.zeros(max(_lib.hga_attn_bwd_workspace_size(cfg, seg_len), 256),
                                  dtype=torch.uint8, device=self.device)
        # zeroed once: hga_segment_fwd_bwd's completion flags live in it
        self.seg_ws = torch.zeros(
            max(_lib.hga_segment_workspace_size(cfg, seg_len, ctx_cap - seg_len), 256),
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

    def route(self, q, q_begin: int, stream=None, scores_out=None):
        _lib.hga_route(self.cfg, q, q_begin, self.seg_len, self.ctx_cap, self.bsum,
                       self.gsum, self.sel_blk, self.sel_grp, self.route_ws, stream=stream,
                       scores_out=scores_out)

    def build_query_summaries(self, q, q_begin: int, stream=None):
        _lib.hga_build_query_summaries(self.cfg, q, q_begin, self.seg_len, self.ctx_cap,
                                       self.qsum, stream)

    def route_causal(self, q, q_begin: int, stream=None):
        _lib.hga_route_causal(self.cfg, q, q_begin, self.seg_len, self.ctx_cap, self.bsum,
                              self.gsum, self.qsum, self.sel_blk, self.sel_grp, self.route_ws,
                              stream=stream)

    def prepare(self, q_proj, k_proj, v_proj, q_row_stride: int, kv_row_stride: int,
                q_begin: int, rope_base, q_out, stream=None):
        """The segment's upstream pass (hga_prepare_segment): RoPE of the
        projections, Q into q_out, K/V into the context, summaries and block
        mean queries into gsum, bsum, qsum."""
        _lib.hga_prepare_segment(self.cfg, q_proj, k_proj, v_proj, q_row_stride, kv_row_stride,
                                 q_begin, self.seg_len, self.ctx_cap, rope_base, q_out, self.k, self.v,
                                 self.gsum, self.bsum, self.qsum, stream)

    def route_summarized(self, q_begin: int, causal=False, stream=None):
        _lib.hga_route_summarized(self.cfg, q_begin, self.seg_len, self.ctx_cap, self.bsum,
                                  self.gsum, self.qsum, causal, self.sel_blk, self.sel_grp,
                                  self.route_ws, stream=stream)

    def segment_from_projections(self, q_proj, k_proj, v_proj, q_row_stride: int,
                                 kv_row_stride: int, q_begin: int, rope_base, q_out, d_o=None,
                                 causal=False, stream=None, out=None):
        """One segment from its projection outputs: the upstream pass, routing
        from the resident summaries, then the forward and (if d_o) backward."""
        self.prepare(q_proj, k_proj, v_proj, q_row_stride, kv_row_stride, q_begin, rope_base,
                     q_out, stream)
        self.route_summarized(q_begin, causal, stream)
        if d_o is None:
            self.forward(q_out, q_begin, stream, out)
        else:
            self.forward_backward(q_out, d_o, q_begin, stream, out)

    def make_outputs(self):
        """A fresh set of per-segment outputs (o, lse, dq, dk, dv), for callers
        that keep one segment's results while the next one is computed."""
        return (torch.empty_like(self.o), torch.empty_like(self.lse), torch.empty_like(self.dq),
                torch.empty_like(self.dk), torch.empty_like(self.dv))

    def _out(self, out):
        return (self.o, self.lse, self.dq, self.dk, self.dv) if out is None else out

    def forward(self, q, q_begin: int, stream=None, out=None):
        o, lse = self._out(out)[:2]
        _lib.hga_attn_fwd(self.cfg, q, self.k, self.v, self.ctx_cap, q_begin, self.seg_len,
                          self.sel_grp, o, lse, stream)

    def backward(self, q, d_o, q_begin: int, stream=None, out=None):
        o, lse, dq, dk, dv = self._out(out)
        _lib.hga_attn_bwd(self.cfg, q, self.k, self.v, self.ctx_cap, q_begin, self.seg_len,
                          self.sel_grp, o, lse, d_o, dq, dk, dv, self.bwd_ws, stream=stream)

    def forward_backward(self, q, d_o, q_begin: int, stream=None, out=None):
        o, lse, dq, dk, dv = self._out(out)
        _lib.hga_attn_fwd_bwd(self.cfg, q, self.k, self.v, self.ctx_cap, q_begin, self.seg_len,
                              self.sel_grp, o, lse, d_o, dq, dk, dv, self.bwd_ws, stream=stream)

    def route_forward_backward(self, q, d_o, q_begin: int, stream=None, out=None):
        o, lse, dq, dk, dv = self._out(out)
        _lib.hga_segment_fwd_bwd(self.cfg, q, self.k, self.v, self.ctx_cap, q_begin,
                                 self.seg_len, self.bsum, self.gsum, self.sel_blk, self.sel_grp,
                                 o, lse, d_o, dq, dk, dv, self.seg_ws, stream=stream)

    def decode(self, q_tok, pos, o, lse, sel_blk=None, sel_grp=None, stream=None):
        """One new token per sequence (hga_decode): q_tok [B, Hq, d] at global
        positions pos (int64 device tensor [B]); the token's K/V must already
        be in self.k / self.v at pos, and every complete block before its own
        block summarised.  Writes o [B, Hq, d] and lse [B, Hq]."""
        _lib.hga_decode(self.cfg, q_tok, self.k, self.v, self.ctx_cap, pos, self.bsum,
                        self.gsum, sel_blk, sel_grp, o, lse, stream)

    def segment(self, q, q_begin: int, d_o=None, stream=None, out=None, causal=False):
        """One segment: summaries, routing, forward and (if d_o) backward
        (chained, so that the forward of each query block starts as soon as
        its selection is written and its backward as soon as its forward is
        done).  Results go to `out` (from make_outputs) if given, else to the
        layer's own o, lse, dq, dk, dv.  causal=True routes each query block
        with the previous block's mean query (hga_route_causal; segments in
        order), then runs the forward and backward chained."""
        self.summarize(q_begin, stream)
        if causal:
            self.route_causal(q, q_begin, stream)
            if d_o is None:
                self.forward(q, q_begin, stream, out)
            else:
                self.forward_backward(q, d_o, q_begin, stream, out)
        elif d_o is None:
            self.route(q, q_begin, stream)
            self.forward(q, q_begin, stream, out)
        else:
            self.route_forward_backward(q, d_o, q_begin, stream, out)


class HgaTieredLayer:
    """One layer with its history K/V in pinned host memory.

    Summaries stay in HBM.  Per segment: summaries of the active keys (from the
    staging buffer), routing, the host-tier gather of the selected history
    groups into HBM staging (hga_tier_gather), attention forward/backward on
    the staging buffer, and finally the append of the segment's K/V to the
    host history.  The caller writes the active segment's K/V into
    `active_k()` / `active_v()` before calling `segment`.
    """

    def __init__(self, cfg: Config, ctx_cap: int, seg_len: int, device="cuda",
                 k_host=None, v_host=None):
        self.cfg, self.ctx_cap, self.seg_len = cfg, ctx_cap, seg_len
        self.device = torch.device(device)
        dt = _TORCH_DTYPE[cfg.dtype]
        B, Hq, Hkv, d = cfg.batch, cfg.n_q_heads, cfg.n_kv_heads, cfg.head_dim
        n_qb = seg_len // 64
        shape = (B, Hkv, ctx_cap, d)
        self.k_host = k_host if k_host is not None else torch.zeros(shape, dtype=dt).pin_memory()
        self.v_host = v_host if v_host is not None else torch.zeros(shape, dtype=dt).pin_memory()
        self.stage_cap = _lib.hga_tier_stage_rows(cfg, ctx_cap - seg_len, seg_len)
        self.k_stage = torch.zeros((B, Hkv, self.stage_cap, d), dtype=dt, device=self.device)
        self.v_stage = torch.zeros_like(self.k_stage)
        self.gsum = torch.zeros((B, Hkv, ctx_cap // 8, d), dtype=torch.float32,
                                device=self.device)
        self.bsum = torch.zeros((B, Hkv, ctx_cap // 64, d), dtype=torch.float32,
                                device=self.device)
        dev = self.device
        self.route_ws = torch.empty(max(_lib.hga_route_workspace_size(cfg, seg_len,
                                                                      ctx_cap - seg_len), 256),
                                    dtype=torch.uint8, device=dev)
        self.bwd_ws = torch.empty(max(_lib.hga_attn_bwd_workspace_size(cfg, seg_len), 256),
                                  dtype=torch.uint8, device=dev)
        self.tier_ws = torch.empty(max(_lib.hga_tier_workspace_size(cfg, seg_len,
                                                                    ctx_cap - seg_len), 256),
                                   dtype=torch.uint8, device=dev)
        self.sel_blk = torch.empty((B, Hkv, n_qb, cfg.topk_blocks), dtype=torch.int32, device=dev)
        self.sel_grp = torch.empty((B, Hkv, n_qb, cfg.topk_groups), dtype=torch.int32, device=dev)
        self.sel_stage = torch.empty_like(self.sel_grp)
        self.n_unique = torch.zeros((B, Hkv), dtype=torch.int32, device=dev)
        self.o = torch.empty((B, Hq, seg_len, d), dtype=dt, device=dev)
        self.lse = torch.empty((B, Hq, seg_len), dtype=torch.float32, device=dev)
        self.dq = torch.empty_like(self.o)
        self.dk = torch.empty((B, Hkv, seg_len, d), dtype=dt, device=dev)
        self.dv = torch.empty_like(self.dk)

    @property
    def q_begin_stage(self) -> int:
        return self.stage_cap - self.seg_len

    def active_k(self):
        return self.k_stage[:, :, self.q_begin_stage:, :]

    def active_v(self):
        return self.v_stage[:, :, self.q_begin_stage:, :]

    def _active_ptr(self, t):
        return t.data_ptr() + self.q_begin_stage * t.shape[-1] * t.element_size()

    def summarize(self, q_begin: int, stream=None):
        _lib.hga_build_summaries_seg(self.cfg, self._active_ptr(self.k_stage), self.stage_cap,
                                     q_begin, q_begin + self.seg_len, self.ctx_cap, self.gsum,
                                     self.bsum, stream)

    def gather(self, q_begin: int, stream=None):
        _lib.hga_tier_gather(self.cfg, self.k_host, self.v_host, self.ctx_cap, q_begin,
                             self.seg_len, self.sel_grp, self.k_stage, self.v_stage,
                             self.stage_cap, self.sel_stage, self.n_unique, self.tier_ws,
                             stream=stream)

    def append_history(self, q_begin: int, stream=None):
        """The segment's K/V join the host history (detached)."""
        _lib.hga_tier_append(self.cfg, self.k_stage, self.v_stage, self.stage_cap, self.k_host,
                             self.v_host, self.ctx_cap, q_begin, self.seg_len, stream)

    def segment(self, q, q_begin: int, d_o=None, stream=None, append=True):
        cfg, S, qs = self.cfg, self.seg_len, self.q_begin_stage
        self.summarize(q_begin, stream)
        _lib.hga_route(cfg, q, q_begin, S, self.ctx_cap, self.bsum, self.gsum, self.sel_blk,
                       self.sel_grp, self.route_ws, stream=stream)
        self.gather(q_begin, stream)
        _lib.hga_attn_fwd(cfg, q, self.k_stage, self.v_stage, self.stage_cap, qs, S,
                          self.sel_stage, self.o, self.lse, stream)
        if d_o is not None:
            _lib.hga_attn_bwd(cfg, q, self.k_stage, self.v_stage, self.stage_cap, qs, S,
                              self.sel_stage, self.o, self.lse, d_o, self.dq, self.dk, self.dv,
                              self.bwd_ws, stream=stream)
        if append:
            self.append_history(q_begin, stream)


class HgaFileTieredLayer(HgaTieredLayer):
    """The host tier with the history K/V in files (NVMe) instead of pinned
    RAM.  Per segment the selected history groups are planned on the GPU
    (hga_tier_plan), their list comes back to the host, the groups are read
    from the files into pinned staging buffers laid out like the device
    staging (hga_tier_read_groups, a pool of reader threads) and copied up
    in one 2-D copy per tensor; the finished segment's K/V are written to the
    files (hga_tier_write_segment).  fd_k / fd_v are open file descriptors
    (read and write) of files of batch * n_kv_heads * ctx_cap * head_dim
    elements; the caller owns them."""

    def __init__(self, cfg: Config, ctx_cap: int, seg_len: int, fd_k: int, fd_v: int,
                 device="cuda", n_threads: int = 8):
        super().__init__(cfg, ctx_cap, seg_len, device=device,
                         k_host=torch.empty(0), v_host=torch.empty(0))
        self.fd_k, self.fd_v, self.n_threads = fd_k, fd_v, n_threads
        B, Hkv, d = cfg.batch, cfg.n_kv_heads, cfg.head_dim
        dt = _TORCH_DTYPE[cfg.dtype]
        self.slot_cap = max(1, min((seg_len // 64) * cfg.topk_groups, (ctx_cap - seg_len) // 8))
        self.slot_group = torch.empty((B, Hkv, self.slot_cap), dtype=torch.int32,
                                      device=self.device)
        self.slot_group_host = torch.empty_like(self.slot_group, device="cpu").pin_memory()
        self.n_unique_host = torch.empty((B, Hkv), dtype=torch.int32).pin_memory()
        hist_rows = self.stage_cap - seg_len
        self.k_stage_host = torch.empty((B, Hkv, hist_rows, d), dtype=dt).pin_memory()
        self.v_stage_host = torch.empty_like(self.k_stage_host).pin_memory()
        self.k_seg_host = torch.empty((B, Hkv, seg_len, d), dtype=dt).pin_memory()
        self.v_seg_host = torch.empty_like(self.k_seg_host).pin_memory()
        self.bytes_read = 0

    def gather(self, q_begin: int, stream=None):
        if q_begin == 0:
            return _lib.hga_tier_plan(self.cfg, q_begin, self.seg_len, self.sel_grp,
                                      self.stage_cap, self.sel_stage, self.slot_group,
                                      self.n_unique, self.slot_cap, stream)
        s = torch.cuda.current_stream(self.device) if stream is None else stream
        _lib.hga_tier_plan(self.cfg, q_begin, self.seg_len, self.sel_grp, self.stage_cap,
                           self.sel_stage, self.slot_group, self.n_unique, self.slot_cap, s)
        with torch.cuda.stream(s):
            self.slot_group_host.copy_(self.slot_group, non_blocking=True)
            self.n_unique_host.copy_(self.n_unique, non_blocking=True)
        s.synchronize()
        hist_rows = self.stage_cap - self.seg_len
        _lib.hga_tier_read_groups(self.cfg, self.fd_k, self.fd_v, self.ctx_cap,
                                  self.slot_group_host, self.n_unique_host, self.slot_cap,
                                  self.k_stage_host, self.v_stage_host, hist_rows,
                                  self.n_threads)
        rows = 8 * int(self.n_unique_host.max())
        row_bytes = self.cfg.head_dim * self.k_stage.element_size()
        self.bytes_read += 2 * int(self.n_unique_host.sum()) * 8 * row_bytes
        if rows:
            with torch.cuda.stream(s):
                self.k_stage[:, :, :rows].copy_(self.k_stage_host[:, :, :rows], non_blocking=True)
                self.v_stage[:, :, :rows].copy_(self.v_stage_host[:, :, :rows], non_blocking=True)

    def append_history(self, q_begin: int, stream=None):
        s = torch.cuda.current_stream(self.device) if stream is None else stream
        with torch.cuda.stream(s):
            self.k_seg_host.copy_(self.active_k(), non_blocking=True)
            self.v_seg_host.copy_(self.active_v(), non_blocking=True)
        s.synchronize()
        _lib.hga_tier_write_segment(self.cfg, self.fd_k, self.fd_v, self.ctx_cap, q_begin,
                                    self.seg_len, self.k_seg_host, self.v_seg_host,
                                    self.seg_len, self.n_threads)
