"""The C ABI library on the CPU: it loads, exports every declared entry point,
and rejects bad arguments on the host before any launch (no GPU needed)."""

import ctypes
import os
import re

import pytest

import hierarchical_routed_sparse_hga_b200 as hga
from hierarchical_routed_sparse_hga_b200 import _lib

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                      "include", "hga.h")


def declared():
    text = open(HEADER).read()
    return set(re.findall(r"HGA_API\s+[\w\s\*]+?\b(hga_\w+)\s*\(", text))


def test_header_declares_what_the_binding_names():
    assert declared() == set(_lib.EXPORTS)


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(_lib.LIB_PATH)
    for name in declared():
        assert hasattr(lib, name), name


def test_version_and_status_strings():
    assert "sm_100a" in hga.hga_version()
    assert hga.hga_status_string(0) == "ok"
    assert hga.hga_status_string(6) == "workspace too small"


def cfg(**kw):
    base = dict(batch=1, n_q_heads=32, n_kv_heads=8, head_dim=128, topk_blocks=16,
                topk_groups=64)
    base.update(kw)
    return hga.Config(**base)


FAKE = 0x10000  # aligned, never dereferenced: every call below fails its host check


def status_of(fn, *args):
    with pytest.raises(hga.HgaError) as e:
        fn(*args)
    return e.value.status


def test_host_argument_checks():
    c = cfg()
    # null pointers
    assert status_of(hga.hga_build_summaries, c, 0, 16384, 0, 2048, FAKE, FAKE, 0) == 1
    # not a multiple of 64
    assert status_of(hga.hga_build_summaries, c, FAKE, 16384, 32, 2048, FAKE, FAKE, 0) == 1
    # misaligned pointer
    assert status_of(hga.hga_attn_fwd, c, FAKE + 4, FAKE, FAKE, 16384, 0, 2048, FAKE, FAKE,
                     FAKE, 0) == 1
    # unsupported head dim / GQA ratio / k
    assert status_of(hga.hga_attn_fwd, cfg(head_dim=96), FAKE, FAKE, FAKE, 16384, 0, 2048,
                     FAKE, FAKE, FAKE, 0) == 2
    assert status_of(hga.hga_attn_fwd, cfg(n_q_heads=80, n_kv_heads=8), FAKE, FAKE, FAKE,
                     16384, 0, 2048, FAKE, FAKE, FAKE, 0) == 2
    assert status_of(hga.hga_attn_fwd, cfg(topk_groups=0), FAKE, FAKE, FAKE, 16384, 0, 2048,
                     FAKE, FAKE, FAKE, 0) == 2
    # segment past the context
    assert status_of(hga.hga_attn_fwd, c, FAKE, FAKE, FAKE, 16384, 15360, 2048, FAKE, FAKE,
                     FAKE, 0) == 1
    # segment too long
    assert status_of(hga.hga_attn_fwd, c, FAKE, FAKE, FAKE, 16384, 0, 8192, FAKE, FAKE,
                     FAKE, 0) == 2
    # workspace too small
    need = hga.hga_route_workspace_size(c, 2048, 14336)
    assert status_of(hga.hga_route, c, FAKE, 14336, 2048, 16384, FAKE, FAKE, None, FAKE, FAKE,
                     need - 256, 0) == 6
    need = hga.hga_attn_bwd_workspace_size(c, 2048)
    assert status_of(hga.hga_attn_bwd, c, FAKE, FAKE, FAKE, 16384, 14336, 2048, FAKE, FAKE,
                     FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, need - 4, 0) == 6
    need = hga.hga_segment_workspace_size(c, 2048, 14336)
    assert status_of(hga.hga_segment_fwd_bwd, c, FAKE, FAKE, FAKE, 16384, 14336, 2048, FAKE,
                     FAKE, None, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, need - 16,
                     0) == 6
    # sel_grp is required
    assert status_of(hga.hga_segment_fwd_bwd, c, FAKE, FAKE, FAKE, 16384, 14336, 2048, FAKE,
                     FAKE, None, None, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, need, 0) == 1


def test_workspace_sizes():
    c = cfg()
    # q-bar: 8 KV heads x 32 query blocks x 128 floats; then, for the 2
    # candidate chunks of 128 blocks (255 candidates), the finalists' keys and
    # block indices: 8 x 32 x 2 x (16 + 1) each (each part 256-B aligned)
    assert hga.hga_route_workspace_size(c, 2048, 14336) == (8 * 32 * 128 * 4
                                                           + 2 * 8 * 32 * 2 * 17 * 4)
    # D = rowsum(dO * O) per query row, the dK/dV kernel's work counter, two
    # arrays of per-item flags (8 KV heads x 32 query blocks) for the fused
    # call, and the inverted selection (8 KV heads x 32 key blocks x 32 query blocks)
    assert hga.hga_attn_bwd_workspace_size(c, 2048) == (32 * 2048 * 4 + 256 + 2 * 8 * 32 * 4
                                                        + 8 * 32 * 32 * 4)
    assert hga.hga_route_workspace_size(cfg(head_dim=100), 2048, 0) == 0
    # the chained segment call: the backward workspace, a third flag array,
    # then the routing workspace
    assert hga.hga_segment_workspace_size(c, 2048, 14336) == (
        hga.hga_attn_bwd_workspace_size(c, 2048) + 8 * 32 * 4
        + hga.hga_route_workspace_size(c, 2048, 14336))
    assert hga.hga_segment_workspace_size(cfg(head_dim=100), 2048, 0) == 0


def test_diagnostics_without_gpu():
    assert hga.hga_kernel_name(0) == "summaries"
    assert hga.hga_kernel_name(99) == "unknown"
    assert hga.hga_launch_count() >= 0
    assert hga.timing_table() == {}


def prototypes():
    """name -> (return type, [parameter types]) from the header's HGA_API lines."""
    text = re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)
    out = {}
    for m in re.finditer(r"HGA_API\s+([\w\s\*]+?)\b(hga_\w+)\s*\(([^)]*)\)\s*;", text):
        ret, name, params = m.group(1).strip(), m.group(2), m.group(3).strip()
        types = []
        if params and params != "void":
            for p in params.split(","):
                p = " ".join(p.split())
                pname = re.search(r"(\w+)\s*$", p).group(1)
                types.append(p[: len(p) - len(pname)].strip())
        out[name] = (ret, types)
    return out


def ctype_of(c_type):
    """The ctypes class the binding must use for a C type of the header."""
    t = c_type.replace("const ", "").replace(" ", "")
    if t == "hga_config_t*":
        return ctypes.POINTER(_lib._Config)
    if t == "double*":
        return ctypes.POINTER(ctypes.c_double)
    if t == "uint64_t*":
        return ctypes.POINTER(ctypes.c_uint64)
    if t.endswith("*"):
        return ctypes.c_char_p if t == "char*" else ctypes.c_void_p
    return {"int64_t": ctypes.c_int64, "int32_t": ctypes.c_int32, "size_t": ctypes.c_size_t,
            "int": ctypes.c_int, "uint32_t": ctypes.c_uint32, "uint64_t": ctypes.c_uint64,
            "hga_status_t": ctypes.c_int, "float": ctypes.c_float, "void": None}[t]


def test_binding_signatures_match_the_header():
    # every argument's width and kind as the header declares it, in order:
    # a parameter added, dropped or reordered on one side fails here
    lib = _lib.load()
    protos = prototypes()
    assert set(protos) == declared()
    for name, (ret, params) in protos.items():
        fn = getattr(lib, name)
        want = [ctype_of(p) for p in params]
        got = list(fn.argtypes or [])
        assert len(got) == len(want), (name, len(got), len(want))
        for i, (g, w_) in enumerate(zip(got, want)):
            assert g == w_ or (w_ is ctypes.c_int and g is ctypes.c_int32), (name, i, g, w_)
        assert fn.restype == ctype_of(ret), (name, fn.restype, ret)


def test_decode_host_argument_checks():
    c = cfg()
    args = (FAKE, FAKE, FAKE, 16384, FAKE, FAKE, FAKE, None, None, FAKE, FAKE, 0)
    # G = 3 has no decode kernel; d = 96 none at all
    assert status_of(hga.hga_decode, cfg(n_q_heads=24), *args) == 2
    assert status_of(hga.hga_decode, cfg(head_dim=96), *args) == 2
    # context not a multiple of 64, a missing position array, a misaligned output
    assert status_of(hga.hga_decode, c, FAKE, FAKE, FAKE, 16380, *args[4:]) == 1
    assert status_of(hga.hga_decode, c, FAKE, FAKE, FAKE, 16384, 0, *args[5:]) == 1
    assert status_of(hga.hga_decode, c, *args[:9], FAKE + 8, FAKE, 0) == 1


def test_prepare_and_summarized_route_host_checks():
    c = cfg()
    a = (FAKE, FAKE, FAKE)
    outs = (FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 0)
    # strides below the row widths, or not a multiple of 16 bytes
    assert status_of(hga.hga_prepare_segment, c, *a, 32 * 128 - 8, 8 * 128, 0, 2048, 16384,
                     1e6, *outs) == 1
    assert status_of(hga.hga_prepare_segment, c, *a, 32 * 128, 8 * 128 - 8, 0, 2048, 16384,
                     1e6, *outs) == 1
    assert status_of(hga.hga_prepare_segment, c, *a, 32 * 128 + 4, 8 * 128, 0, 2048, 16384,
                     1e6, *outs) == 1
    # a negative RoPE base; a segment past the context
    assert status_of(hga.hga_prepare_segment, c, *a, 4096, 1024, 0, 2048, 16384, -1.0,
                     *outs) == 1
    assert status_of(hga.hga_prepare_segment, c, *a, 4096, 1024, 15360, 2048, 16384, 1e6,
                     *outs) == 1
    # routing from summaries needs the block means, and causal is 0 or 1
    need = hga.hga_route_workspace_size(c, 2048, 14336)
    assert status_of(hga.hga_route_summarized, c, 14336, 2048, 16384, FAKE, FAKE, None, 0, None,
                     FAKE, FAKE, need, 0) == 1
    assert status_of(hga.hga_route_summarized, c, 14336, 2048, 16384, FAKE, FAKE, FAKE, 2, None,
                     FAKE, FAKE, need, 0) == 1
    assert status_of(hga.hga_route_causal, c, FAKE, 14336, 2048, 16384, FAKE, FAKE, FAKE, None,
                     FAKE, FAKE, need - 256, 0) == 6


def test_noalloc_limit_on_the_host():
    # the no-workspace routing takes its scratch from a fixed 4 MiB array: for
    # the Qwen3-8B shape at batch 1 and 2048-token segments the largest
    # context it accepts is 950,272 tokens; past it the call returns
    # HGA_ERR_WORKSPACE before touching the GPU
    c = cfg()
    limit = 4 << 20
    assert hga.hga_route_workspace_size(c, 2048, 950272 - 2048) <= limit
    assert hga.hga_route_workspace_size(c, 2048, 950272) > limit
    assert status_of(hga.hga_route_noalloc, c, FAKE, 950272, 2048, 952320, FAKE, FAKE, None,
                     FAKE, 0) == 6
