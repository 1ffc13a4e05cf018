"""ctypes binding of libhga (argument marshalling only).

Every function here has the name and argument order of the C entry point in
include/hga.h.  Array arguments are CUDA torch tensors (contiguous) or raw
device addresses (int); the stream defaults to torch's current stream.  Every
step of the hot path runs in libhga's kernels: there is no other code path, and
a missing library raises instead of falling back.
"""

from __future__ import annotations

import ctypes
import dataclasses
import math
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libhga.so")

HGA_OK, HGA_ERR_INVALID_ARG, HGA_ERR_UNSUPPORTED, HGA_ERR_CUDA, HGA_ERR_TIMEOUT, \
    HGA_ERR_DEVICE_CHECK, HGA_ERR_WORKSPACE, HGA_ERR_IO = range(8)
HGA_F32, HGA_BF16 = 0, 1
HGA_FLAG_SIMT = 1

EXPORTS = ("hga_version", "hga_status_string", "hga_last_cuda_error", "hga_build_summaries",
           "hga_route_workspace_size", "hga_route", "hga_attn_fwd",
           "hga_attn_bwd_workspace_size", "hga_attn_bwd", "hga_attn_fwd_bwd",
           "hga_segment_workspace_size", "hga_segment_fwd_bwd",
           "hga_get_device_status",
           "hga_kernel_name", "hga_launch_count", "hga_timing_enable", "hga_timing_collect",
           "hga_timing_get", "hga_timing_reset", "hga_timing_kinds", "hga_route_noalloc",
           "hga_build_summaries_seg",
           "hga_tier_stage_rows", "hga_tier_workspace_size", "hga_tier_gather",
           "hga_tier_append", "hga_decode", "hga_build_query_summaries",
           "hga_route_causal", "hga_prepare_segment", "hga_route_summarized",
           "hga_tier_plan", "hga_tier_read_groups", "hga_tier_write_segment")
HGA_NOALLOC_SCRATCH_BYTES = 4 << 20
HGA_K_COUNT = 16


class HgaError(RuntimeError):
    def __init__(self, fn: str, status: int, text: str):
        super().__init__(f"{fn}: {text} (status {status})")
        self.status = status


class _Config(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("n_q_heads", ctypes.c_int32),
                ("n_kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("topk_blocks", ctypes.c_int32), ("topk_groups", ctypes.c_int32),
                ("dtype", ctypes.c_int32), ("flags", ctypes.c_uint32),
                ("scale", ctypes.c_float)]


@dataclasses.dataclass
class Config:
    """Mirror of hga_config_t."""
    batch: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    topk_blocks: int
    topk_groups: int
    dtype: int = HGA_BF16
    flags: int = 0
    scale: float | None = None

    def c(self) -> _Config:
        scale = self.scale if self.scale is not None else 1.0 / math.sqrt(self.head_dim)
        return _Config(self.batch, self.n_q_heads, self.n_kv_heads, self.head_dim,
                       self.topk_blocks, self.topk_groups, self.dtype, self.flags, scale)


_lib = None


def load() -> ctypes.CDLL:
    """Load the in-tree libhga.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"libhga.so is not built at {LIB_PATH}; run "
                          "`python -m hierarchical_routed_sparse_hga_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    P, I32, I64, SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
    CFG = ctypes.POINTER(_Config)
    sig = {
        "hga_version": (ctypes.c_char_p, []),
        "hga_status_string": (ctypes.c_char_p, [ctypes.c_int]),
        "hga_last_cuda_error": (ctypes.c_char_p, []),
        "hga_build_summaries": (ctypes.c_int, [CFG, P, I64, I64, I64, P, P, P]),
        "hga_route_workspace_size": (SZ, [CFG, I32, I64]),
        "hga_route": (ctypes.c_int, [CFG, P, I64, I32, I64, P, P, P, P, P, P, SZ, P]),
        "hga_attn_fwd": (ctypes.c_int, [CFG, P, P, P, I64, I64, I32, P, P, P, P]),
        "hga_attn_bwd_workspace_size": (SZ, [CFG, I32]),
        "hga_attn_bwd": (ctypes.c_int, [CFG, P, P, P, I64, I64, I32, P, P, P, P, P, P, P,
                                        P, SZ, P]),
        "hga_attn_fwd_bwd": (ctypes.c_int, [CFG, P, P, P, I64, I64, I32, P, P, P, P, P, P, P,
                                            P, SZ, P]),
        "hga_segment_workspace_size": (SZ, [CFG, I32, I64]),
        "hga_segment_fwd_bwd": (ctypes.c_int, [CFG, P, P, P, I64, I64, I32, P, P, P, P, P, P,
                                               P, P, P, P, P, SZ, P]),
        "hga_get_device_status": (ctypes.c_int, [P]),
        "hga_kernel_name": (ctypes.c_char_p, [ctypes.c_int]),
        "hga_launch_count": (ctypes.c_uint64, []),
        "hga_timing_enable": (ctypes.c_int, [I32]),
        "hga_timing_collect": (ctypes.c_int, []),
        "hga_timing_get": (ctypes.c_int, [ctypes.c_int, ctypes.POINTER(ctypes.c_double),
                                          ctypes.POINTER(ctypes.c_uint64)]),
        "hga_timing_reset": (None, []),
        "hga_timing_kinds": (None, [ctypes.c_uint32]),
        "hga_route_noalloc": (ctypes.c_int, [CFG, P, I64, I32, I64, P, P, P, P, P]),
        "hga_build_summaries_seg": (ctypes.c_int, [CFG, P, I64, I64, I64, I64, P, P, P]),
        "hga_tier_stage_rows": (I64, [CFG, I64, I32]),
        "hga_tier_workspace_size": (SZ, [CFG, I32, I64]),
        "hga_tier_gather": (ctypes.c_int, [CFG, P, P, I64, I64, I32, P, P, P, I64, P, P, P, SZ,
                                           P]),
        "hga_tier_append": (ctypes.c_int, [CFG, P, P, I64, P, P, I64, I64, I32, P]),
        "hga_decode": (ctypes.c_int, [CFG, P, P, P, I64, P, P, P, P, P, P, P, P]),
        "hga_build_query_summaries": (ctypes.c_int, [CFG, P, I64, I32, I64, P, P]),
        "hga_route_causal": (ctypes.c_int, [CFG, P, I64, I32, I64, P, P, P, P, P, P, SZ, P]),
        "hga_prepare_segment": (ctypes.c_int, [CFG, P, P, P, I64, I64, I64, I32, I64,
                                               ctypes.c_float,
                                               P, P, P, P, P, P, P]),
        "hga_route_summarized": (ctypes.c_int, [CFG, I64, I32, I64, P, P, P, I32, P, P, P, SZ,
                                                P]),
        "hga_tier_plan": (ctypes.c_int, [CFG, I64, I32, P, I64, P, P, P, I64, P]),
        "hga_tier_read_groups": (ctypes.c_int, [CFG, ctypes.c_int, ctypes.c_int, I64, P, P, I64,
                                                P, P, I64, I32]),
        "hga_tier_write_segment": (ctypes.c_int, [CFG, ctypes.c_int, ctypes.c_int, I64, I64,
                                                  I32, P, P, I64, I32]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype, fn.argtypes = res, args
    _lib = lib
    return lib


def _ptr(x):
    if x is None:
        return None
    if isinstance(x, int):
        return x
    if not x.is_cuda:
        raise ValueError("libhga takes device tensors")
    if not x.is_contiguous():
        raise ValueError("libhga takes contiguous tensors")
    return x.data_ptr()


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(fn: str, status: int):
    if status != HGA_OK:
        text = load().hga_status_string(status).decode()
        if status == HGA_ERR_CUDA:
            text += f" ({load().hga_last_cuda_error().decode()})"
        raise HgaError(fn, status, text)


def _nbytes(t):
    return t.numel() * t.element_size()


# ----------------------------------------------------------------------------
# entry points (same names as the C ABI)
# ----------------------------------------------------------------------------

def hga_last_cuda_error() -> str:
    return load().hga_last_cuda_error().decode()


def hga_version() -> str:
    return load().hga_version().decode()


def hga_status_string(status: int) -> str:
    return load().hga_status_string(status).decode()


def hga_build_summaries(cfg: Config, k, ctx_cap, t_begin, t_end, gsum, bsum, stream=None):
    c = cfg.c()
    _check("hga_build_summaries", load().hga_build_summaries(
        ctypes.byref(c), _ptr(k), ctx_cap, t_begin, t_end, _ptr(gsum), _ptr(bsum),
        _stream(stream)))


def hga_build_summaries_seg(cfg: Config, k_seg, seg_cap, t_begin, t_end, ctx_cap, gsum, bsum,
                            stream=None):
    c = cfg.c()
    _check("hga_build_summaries_seg", load().hga_build_summaries_seg(
        ctypes.byref(c), _ptr(k_seg), seg_cap, t_begin, t_end, ctx_cap, _ptr(gsum), _ptr(bsum),
        _stream(stream)))


def hga_tier_stage_rows(cfg: Config, q_begin, s_len) -> int:
    c = cfg.c()
    return int(load().hga_tier_stage_rows(ctypes.byref(c), q_begin, s_len))


def hga_tier_workspace_size(cfg: Config, s_len, q_begin) -> int:
    c = cfg.c()
    return int(load().hga_tier_workspace_size(ctypes.byref(c), s_len, q_begin))


def _host_ptr(x):
    """Pinned host tensor (or raw address) for the tier's host-side arrays."""
    if isinstance(x, int):
        return x
    if x.is_cuda or not x.is_pinned() or not x.is_contiguous():
        raise ValueError("hga_tier_gather takes contiguous pinned host tensors for K/V")
    return x.data_ptr()


def hga_tier_gather(cfg: Config, k_host, v_host, ctx_cap, q_begin, s_len, sel_grp, k_stage,
                    v_stage, stage_cap, sel_stage, n_unique, workspace, ws_bytes=None,
                    stream=None):
    c = cfg.c()
    ws_bytes = _nbytes(workspace) if ws_bytes is None else ws_bytes
    _check("hga_tier_gather", load().hga_tier_gather(
        ctypes.byref(c), _host_ptr(k_host), _host_ptr(v_host), ctx_cap, q_begin, s_len,
        _ptr(sel_grp), _ptr(k_stage), _ptr(v_stage), stage_cap, _ptr(sel_stage), _ptr(n_unique),
        _ptr(workspace), ws_bytes, _stream(stream)))


def hga_tier_append(cfg: Config, k_stage, v_stage, stage_cap, k_host, v_host, ctx_cap, q_begin,
                    s_len, stream=None):
    c = cfg.c()
    _check("hga_tier_append", load().hga_tier_append(
        ctypes.byref(c), _ptr(k_stage), _ptr(v_stage), stage_cap, _host_ptr(k_host),
        _host_ptr(v_host), ctx_cap, q_begin, s_len, _stream(stream)))


def hga_route_workspace_size(cfg: Config, s_len, q_begin) -> int:
    c = cfg.c()
    return int(load().hga_route_workspace_size(ctypes.byref(c), s_len, q_begin))


def hga_route(cfg: Config, q, q_begin, s_len, ctx_cap, bsum, gsum, sel_blk, sel_grp,
              workspace, ws_bytes=None, stream=None, scores_out=None):
    """scores_out (optional, [B, Hkv, s_len/64, 4] float32) is the C call's
    argument after sel_grp; a keyword here."""
    c = cfg.c()
    ws_bytes = _nbytes(workspace) if ws_bytes is None else ws_bytes
    _check("hga_route", load().hga_route(
        ctypes.byref(c), _ptr(q), q_begin, s_len, ctx_cap, _ptr(bsum), _ptr(gsum),
        _ptr(sel_blk), _ptr(sel_grp), _ptr(scores_out), _ptr(workspace), ws_bytes,
        _stream(stream)))


def hga_build_query_summaries(cfg: Config, q, q_begin, s_len, ctx_cap, qsum, stream=None):
    c = cfg.c()
    _check("hga_build_query_summaries", load().hga_build_query_summaries(
        ctypes.byref(c), _ptr(q), q_begin, s_len, ctx_cap, _ptr(qsum), _stream(stream)))


def hga_route_causal(cfg: Config, q, q_begin, s_len, ctx_cap, bsum, gsum, qsum, sel_blk, sel_grp,
                     workspace, ws_bytes=None, stream=None):
    c = cfg.c()
    ws_bytes = _nbytes(workspace) if ws_bytes is None else ws_bytes
    _check("hga_route_causal", load().hga_route_causal(
        ctypes.byref(c), _ptr(q), q_begin, s_len, ctx_cap, _ptr(bsum), _ptr(gsum), _ptr(qsum),
        _ptr(sel_blk), _ptr(sel_grp), _ptr(workspace), ws_bytes, _stream(stream)))


def hga_prepare_segment(cfg: Config, q_proj, k_proj, v_proj, q_row_stride, kv_row_stride, q_begin,
                        s_len, ctx_cap, rope_base, q_out, k, v, gsum, bsum, qsum, stream=None):
    c = cfg.c()
    _check("hga_prepare_segment", load().hga_prepare_segment(
        ctypes.byref(c), _ptr(q_proj), _ptr(k_proj), _ptr(v_proj), q_row_stride, kv_row_stride,
        q_begin, s_len,
        ctx_cap, float(rope_base or 0.0), _ptr(q_out), _ptr(k), _ptr(v), _ptr(gsum), _ptr(bsum),
        _ptr(qsum), _stream(stream)))


def hga_route_summarized(cfg: Config, q_begin, s_len, ctx_cap, bsum, gsum, qsum, causal, sel_blk,
                         sel_grp, workspace, ws_bytes=None, stream=None):
    c = cfg.c()
    ws_bytes = _nbytes(workspace) if ws_bytes is None else ws_bytes
    _check("hga_route_summarized", load().hga_route_summarized(
        ctypes.byref(c), q_begin, s_len, ctx_cap, _ptr(bsum), _ptr(gsum), _ptr(qsum),
        int(causal), _ptr(sel_blk), _ptr(sel_grp), _ptr(workspace), ws_bytes,
        _stream(stream)))


def _hptr(x):
    """Host memory (numpy array, CPU tensor or raw address) for the file tier."""
    if x is None or isinstance(x, int):
        return x
    if hasattr(x, "ctypes"):
        if not x.flags["C_CONTIGUOUS"]:
            raise ValueError("the file tier takes contiguous host arrays")
        return x.ctypes.data
    if x.is_cuda or not x.is_contiguous():
        raise ValueError("the file tier takes contiguous host tensors")
    return x.data_ptr()


def hga_tier_plan(cfg: Config, q_begin, s_len, sel_grp, stage_cap, sel_stage, slot_group,
                  n_unique, slot_cap, stream=None):
    c = cfg.c()
    _check("hga_tier_plan", load().hga_tier_plan(
        ctypes.byref(c), q_begin, s_len, _ptr(sel_grp), stage_cap, _ptr(sel_stage),
        _ptr(slot_group), _ptr(n_unique), slot_cap, _stream(stream)))


def hga_tier_read_groups(cfg: Config, fd_k, fd_v, ctx_cap, slot_group, n_unique, slot_cap,
                         k_stage_host, v_stage_host, stage_cap, n_threads=8):
    c = cfg.c()
    _check("hga_tier_read_groups", load().hga_tier_read_groups(
        ctypes.byref(c), fd_k, fd_v, ctx_cap, _hptr(slot_group), _hptr(n_unique), slot_cap,
        _hptr(k_stage_host), _hptr(v_stage_host), stage_cap, n_threads))


def hga_tier_write_segment(cfg: Config, fd_k, fd_v, ctx_cap, q_begin, s_len, k_seg_host,
                           v_seg_host, seg_rows, n_threads=8):
    c = cfg.c()
    _check("hga_tier_write_segment", load().hga_tier_write_segment(
        ctypes.byref(c), fd_k, fd_v, ctx_cap, q_begin, s_len, _hptr(k_seg_host),
        _hptr(v_seg_host), seg_rows, n_threads))


def hga_route_noalloc(cfg: Config, q, q_begin, s_len, ctx_cap, bsum, gsum, sel_blk, sel_grp,
                      stream=None):
    """hga_route with the library's built-in scratch array instead of a
    caller-provided workspace, for callers that cannot allocate device memory."""
    c = cfg.c()
    _check("hga_route_noalloc", load().hga_route_noalloc(
        ctypes.byref(c), _ptr(q), q_begin, s_len, ctx_cap, _ptr(bsum), _ptr(gsum),
        _ptr(sel_blk), _ptr(sel_grp), _stream(stream)))


def hga_decode(cfg: Config, q, k, v, ctx_cap, pos, bsum, gsum, sel_blk, sel_grp, o, lse,
               stream=None):
    """One new token per sequence at positions pos (int64 device tensor)."""
    c = cfg.c()
    _check("hga_decode", load().hga_decode(
        ctypes.byref(c), _ptr(q), _ptr(k), _ptr(v), ctx_cap, _ptr(pos), _ptr(bsum), _ptr(gsum),
        _ptr(sel_blk), _ptr(sel_grp), _ptr(o), _ptr(lse), _stream(stream)))


def hga_attn_fwd(cfg: Config, q, k, v, ctx_cap, q_begin, s_len, sel_grp, o, lse, stream=None):
    c = cfg.c()
    _check("hga_attn_fwd", load().hga_attn_fwd(
        ctypes.byref(c), _ptr(q), _ptr(k), _ptr(v), ctx_cap, q_begin, s_len, _ptr(sel_grp),
        _ptr(o), _ptr(lse), _stream(stream)))


def hga_attn_bwd_workspace_size(cfg: Config, s_len) -> int:
    c = cfg.c()
    return int(load().hga_attn_bwd_workspace_size(ctypes.byref(c), s_len))


def hga_attn_bwd(cfg: Config, q, k, v, ctx_cap, q_begin, s_len, sel_grp, o, lse, d_o, dq, dk,
                 dv, workspace, ws_bytes=None, stream=None):
    c = cfg.c()
    ws_bytes = _nbytes(workspace) if ws_bytes is None else ws_bytes
    _check("hga_attn_bwd", load().hga_attn_bwd(
        ctypes.byref(c), _ptr(q), _ptr(k), _ptr(v), ctx_cap, q_begin, s_len, _ptr(sel_grp),
        _ptr(o), _ptr(lse), _ptr(d_o), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(workspace), ws_bytes,
        _stream(stream)))


def hga_attn_fwd_bwd(cfg: Config, q, k, v, ctx_cap, q_begin, s_len, sel_grp, o, lse, d_o, dq,
                     dk, dv, workspace, ws_bytes=None, stream=None):
    """hga_attn_fwd then hga_attn_bwd in one call (the kernels overlap);
    the workspace's flag sections must be zero before its first use."""
    c = cfg.c()
    ws_bytes = _nbytes(workspace) if ws_bytes is None else ws_bytes
    _check("hga_attn_fwd_bwd", load().hga_attn_fwd_bwd(
        ctypes.byref(c), _ptr(q), _ptr(k), _ptr(v), ctx_cap, q_begin, s_len, _ptr(sel_grp),
        _ptr(o), _ptr(lse), _ptr(d_o), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(workspace), ws_bytes,
        _stream(stream)))


def hga_segment_workspace_size(cfg: Config, s_len, q_begin) -> int:
    c = cfg.c()
    return int(load().hga_segment_workspace_size(ctypes.byref(c), s_len, q_begin))


def hga_segment_fwd_bwd(cfg: Config, q, k, v, ctx_cap, q_begin, s_len, bsum, gsum, sel_blk,
                        sel_grp, o, lse, d_o, dq, dk, dv, workspace, ws_bytes=None,
                        stream=None):
    """hga_route then hga_attn_fwd_bwd in one call (the forward of a query
    block waits only for its own selection); sel_blk may be None; the
    workspace's flag sections must be zero before its first use."""
    c = cfg.c()
    ws_bytes = _nbytes(workspace) if ws_bytes is None else ws_bytes
    _check("hga_segment_fwd_bwd", load().hga_segment_fwd_bwd(
        ctypes.byref(c), _ptr(q), _ptr(k), _ptr(v), ctx_cap, q_begin, s_len, _ptr(bsum),
        _ptr(gsum), _ptr(sel_blk), _ptr(sel_grp), _ptr(o), _ptr(lse), _ptr(d_o), _ptr(dq),
        _ptr(dk), _ptr(dv), _ptr(workspace), ws_bytes, _stream(stream)))

def hga_get_device_status(stream=None) -> int:
    return int(load().hga_get_device_status(_stream(stream)))


# ----------------------------------------------------------------------------
# diagnostics
# ----------------------------------------------------------------------------

def hga_kernel_name(kind: int) -> str:
    return load().hga_kernel_name(kind).decode()


def hga_launch_count() -> int:
    return int(load().hga_launch_count())


def hga_timing_enable(slots: int):
    _check("hga_timing_enable", load().hga_timing_enable(slots))


def hga_timing_collect():
    _check("hga_timing_collect", load().hga_timing_collect())


def hga_timing_get(kind: int):
    ms, n = ctypes.c_double(), ctypes.c_uint64()
    _check("hga_timing_get", load().hga_timing_get(kind, ctypes.byref(ms), ctypes.byref(n)))
    return ms.value, int(n.value)


def hga_timing_reset():
    load().hga_timing_reset()


def hga_timing_kinds(mask: int):
    load().hga_timing_kinds(mask & 0xFFFFFFFF)


def timing_table() -> dict:
    """{kernel name: (total ms, timed launches)} for every kind timed so far."""
    out = {}
    for kind in range(HGA_K_COUNT):
        ms, n = hga_timing_get(kind)
        if n:
            out[hga_kernel_name(kind)] = (ms, n)
    return out
