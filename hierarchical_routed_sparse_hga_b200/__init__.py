"""B200-native HGA hot path: libhga (C ABI, sm_100a kernels) and its binding.

    from hierarchical_routed_sparse_hga_b200 import Config, HgaLayer
    from hierarchical_routed_sparse_hga_b200 import hga_route, hga_attn_fwd, ...

The shared library is loaded on first use; build it with
`python -m hierarchical_routed_sparse_hga_b200.build`.
"""
from ._lib import (EXPORTS, HGA_BF16, HGA_ERR_CUDA, HGA_ERR_DEVICE_CHECK,  # noqa: F401
                   HGA_ERR_INVALID_ARG, HGA_ERR_TIMEOUT, HGA_ERR_UNSUPPORTED,
                   HGA_ERR_IO, HGA_ERR_WORKSPACE, HGA_F32, HGA_FLAG_SIMT, HGA_K_COUNT, HGA_OK, Config,
                   HgaError,
                   hga_attn_bwd, hga_attn_bwd_workspace_size, hga_attn_fwd,
                   hga_attn_fwd_bwd, hga_decode, hga_segment_fwd_bwd, hga_segment_workspace_size,
                   hga_build_summaries, hga_build_summaries_seg, hga_tier_append, hga_tier_gather,
                   hga_tier_stage_rows, hga_tier_workspace_size, hga_get_device_status,
                   hga_kernel_name,
                   hga_launch_count, hga_route, hga_route_causal, hga_route_noalloc,
                   hga_build_query_summaries, hga_prepare_segment, hga_route_summarized,
                   hga_tier_plan, hga_tier_read_groups, hga_tier_write_segment,
                   hga_route_workspace_size, hga_status_string,
                   hga_timing_collect, hga_timing_enable, hga_timing_get, hga_timing_kinds,
                   hga_timing_reset,
                   hga_version, load, timing_table)


def __getattr__(name):
    # HgaLayer needs torch; import it lazily so CPU-only tools stay light
    if name in ("HgaLayer", "HgaTieredLayer", "HgaFileTieredLayer"):
        from . import runtime
        return getattr(runtime, name)
    raise AttributeError(name)
