"""hga_route_noalloc: routing for callers that cannot allocate device memory.

Some callers have no way to call cudaMalloc -- a plugin inside a host runtime
that owns all device memory and gives its extensions no allocator, or code
that must not allocate once running because cudaMalloc can synchronise the
device.  hga_route_noalloc serves them by taking the router's scratch (the
mean queries and the candidate chunks' finalists) from an array built into
the library instead of a caller-provided workspace.

The context here is long enough (more than 512 candidate blocks) that the
routing runs as its three-kernel form, which is the form that writes and
reads that scratch.  The test calls the entry point through the C ABI twice
in a row: first at the end of a 40960-token context, then on an earlier
segment with fewer candidates, so the second call's finalist rows are
shorter than the first call's and sit over its leftover contents.  Each
result must equal the workspace-taking hga_route's exactly (selections are
integer indices).

The file name sorts last so that a run which stops at the first failure has
already run every other test.
"""

import numpy as np
import pytest

from hierarchical_routed_sparse_hga_b200 import synth

pytestmark = pytest.mark.gpu


def test_route_noalloc_matches_route_on_two_calls_in_a_row():
    import torch
    from hierarchical_routed_sparse_hga_b200 import (HGA_BF16, Config, HgaLayer,
                                                     hga_build_summaries, hga_route,
                                                     hga_route_noalloc)

    w = synth.custom(n_q_heads=32, n_kv_heads=8, head_dim=128, ctx_len=40960, seg_len=2048,
                     topk_blocks=16, topk_groups=64, dtype="bf16", scaled=True,
                     rope_base=1e6, seed=21)
    dev = torch.device("cuda", 0)

    def bf16(a):
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(dev)

    cfg = Config(w.batch, w.n_q_heads, w.n_kv_heads, w.head_dim, w.topk_blocks,
                 w.topk_groups, HGA_BF16)
    layer = HgaLayer(cfg, w.ctx_len, w.seg_len, device=dev, k=bf16(synth.keys(w)),
                     v=bf16(synth.values(w)))
    hga_build_summaries(cfg, layer.k, w.ctx_len, 0, w.ctx_len, layer.gsum, layer.bsum)

    n_qb = w.seg_len // 64
    for q_begin in (38912, 34816):        # two calls in a row, the second with shorter rows
        assert q_begin // 64 > 512        # past the single-kernel routing's limit
        q = bf16(synth.queries(w, q_begin))
        ref_blk = torch.full((1, 8, n_qb, 16), -9, dtype=torch.int32, device=dev)
        ref_grp = torch.full((1, 8, n_qb, 64), -9, dtype=torch.int32, device=dev)
        hga_route(cfg, q, q_begin, w.seg_len, w.ctx_len, layer.bsum, layer.gsum, ref_blk,
                  ref_grp, layer.route_ws)
        blk = torch.full_like(ref_blk, -9)
        grp = torch.full_like(ref_grp, -9)
        hga_route_noalloc(cfg, q, q_begin, w.seg_len, w.ctx_len, layer.bsum, layer.gsum, blk,
                          grp)
        torch.cuda.synchronize(dev)
        assert torch.equal(blk, ref_blk), q_begin
        assert torch.equal(grp, ref_grp), q_begin
        assert (grp >= 0).all()           # every slot filled: 16 blocks x 8 groups >= 64
    # and no device-side check latched an error on the way
    from hierarchical_routed_sparse_hga_b200 import hga_get_device_status
    assert hga_get_device_status() == 0


def test_route_noalloc_rejects_work_beyond_its_scratch():
    from hierarchical_routed_sparse_hga_b200 import (HGA_ERR_WORKSPACE, Config, HgaError,
                                                     hga_route_noalloc)
    cfg = Config(1, 32, 8, 128, 16, 64)
    fake = 0x10000  # never dereferenced: the size check fails before any launch
    with pytest.raises(HgaError) as e:
        hga_route_noalloc(cfg, fake, 1015808, 2048, 1017856, fake, fake, None, fake, 0)
    assert e.value.status == HGA_ERR_WORKSPACE
