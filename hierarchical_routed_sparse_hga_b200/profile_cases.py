"""Small cases for profiling one kernel family at a time under ncu.

    python -m hierarchical_routed_sparse_hga_b200.profile_cases <case>

Each case draws its inputs on the device (seeded), builds them through the
package's binding and launches every kernel of its family at least three
times, so that a capture can skip the first launches.  The cases hold a few
GB of device memory at most, and their inputs are larger than L2 where the
kernel reads HBM, so DRAM counters keep their meaning.

  bench16k  the 16384-token fwd+bwd workload (Qwen3-8B attention shape: 32
            query / 8 KV heads, d = 128, bf16; 8 segments of 2048), two passes
  long128k  batch 2, the last segment of a 131072-token context (2047
            candidate blocks: the three-kernel routing), forward, three times
  decode    batch 8, one token at position 32767 of a 32768-token context
  prepare   batch 8, one segment of 2048 from the projection outputs, then
            the query summaries
  tier      host tier, batch 8 x 8192 tokens, 4 segments fwd+bwd
  simt      the CUDA-core kernels: float32, d = 64, 4 query heads / 1 KV
            head, batch 2, 4 segments of 1024 after 4096 history tokens
"""
import sys

import torch

from . import HGA_BF16, HGA_F32, Config, HgaLayer, HgaTieredLayer, hga_build_summaries, synth

CASES = ("bench16k", "long128k", "decode", "prepare", "tier", "simt")


def _qwen3(batch, ctx, **kw):
    return synth.custom(batch=batch, n_q_heads=32, n_kv_heads=8, head_dim=128, ctx_len=ctx,
                        seg_len=2048, topk_blocks=16, topk_groups=64, dtype="bf16", scaled=True,
                        rope_base=1e6, **kw)


def _cfg(w, dtype=HGA_BF16):
    return Config(w.batch, w.n_q_heads, w.n_kv_heads, w.head_dim, w.topk_blocks,
                  w.topk_groups, dtype)


def run(case, dev):
    if case == "bench16k":
        w = synth.workloads()["qwen3_fwdbwd_16k"]
        k, v, qs, dos = synth.device_inputs(w, dev)
        layer = HgaLayer(_cfg(w), w.ctx_len, w.seg_len, device=dev, k=k, v=v)
        for _ in range(2):
            for i, s0 in enumerate(w.segments()):
                layer.segment(qs[i], s0, dos[i])
    elif case == "long128k":
        w = _qwen3(2, 131072, seed=61, first_seg=64, backward=False)
        k, v, _, _ = synth.device_inputs(w, dev, backward=False)
        layer = HgaLayer(_cfg(w), w.ctx_len, w.seg_len, device=dev, k=k, v=v)
        q_begin = w.ctx_len - w.seg_len
        hga_build_summaries(layer.cfg, layer.k, w.ctx_len, 0, q_begin, layer.gsum, layer.bsum)
        g = torch.Generator(device=dev)
        g.manual_seed(61)
        q = (torch.randn((2, 32, 2048, 128), generator=g, device=dev) * 0.09).to(torch.bfloat16)
        for _ in range(3):
            layer.segment(q, q_begin)
    elif case == "decode":
        w = _qwen3(8, 32768, seed=60)
        pos = w.ctx_len - 1
        k, v, q = synth.device_decode_inputs(w, [pos] * 8, dev)
        layer = HgaLayer(_cfg(w), w.ctx_len, w.seg_len, device=dev, k=k, v=v)
        hga_build_summaries(layer.cfg, layer.k, w.ctx_len, 0, w.ctx_len, layer.gsum, layer.bsum)
        p = torch.full((8,), pos, dtype=torch.int64, device=dev)
        o = torch.empty((8, 32, 128), dtype=torch.bfloat16, device=dev)
        lse = torch.empty((8, 32), device=dev)
        for _ in range(3):
            layer.decode(q, p, o, lse)
    elif case == "prepare":
        w = _qwen3(8, 4096, seed=60)
        layer = HgaLayer(_cfg(w), w.ctx_len, w.seg_len, device=dev)
        g = torch.Generator(device=dev)
        g.manual_seed(60)
        qp = torch.randn((8, 2048, 32, 128), generator=g, device=dev).to(torch.bfloat16)
        kp = torch.randn((8, 2048, 8, 128), generator=g, device=dev).to(torch.bfloat16)
        vp = torch.randn((8, 2048, 8, 128), generator=g, device=dev).to(torch.bfloat16)
        q_out = torch.empty((8, 32, 2048, 128), dtype=torch.bfloat16, device=dev)
        for _ in range(3):
            layer.prepare(qp, kp, vp, 32 * 128, 8 * 128, 2048, 1e6, q_out)
            layer.build_query_summaries(q_out, 2048)
    elif case == "tier":
        w = _qwen3(8, 8192, seed=60)
        k, v, qs, dos = synth.device_inputs(w, dev)
        tier = HgaTieredLayer(_cfg(w), w.ctx_len, w.seg_len, device=dev)
        S = w.seg_len
        for i, s0 in enumerate(w.segments()):
            tier.active_k().copy_(k[:, :, s0:s0 + S])
            tier.active_v().copy_(v[:, :, s0:s0 + S])
            tier.segment(qs[i], s0, dos[i])
    elif case == "simt":
        w = synth.custom(batch=2, n_q_heads=4, n_kv_heads=1, head_dim=64, ctx_len=8192,
                         seg_len=1024, topk_blocks=8, topk_groups=32, dtype="f32", seed=62,
                         first_seg=4)
        k, v, qs, dos = synth.device_inputs(w, dev)
        layer = HgaLayer(_cfg(w, HGA_F32), w.ctx_len, w.seg_len, device=dev, k=k, v=v)
        hga_build_summaries(layer.cfg, layer.k, w.ctx_len, 0, 4096, layer.gsum, layer.bsum)
        for i, s0 in enumerate(w.segments()):
            layer.segment(qs[i], s0, dos[i])
    else:
        raise SystemExit(f"unknown case {case!r}; one of {', '.join(CASES)}")
    torch.cuda.synchronize(dev)


def main(argv=None):
    argv = sys.argv[1:] if argv is None else argv
    if len(argv) != 1:
        raise SystemExit(f"usage: python -m hierarchical_routed_sparse_hga_b200.profile_cases "
                         f"<{'|'.join(CASES)}>")
    run(argv[0], torch.device("cuda", 0))
    print("ok", argv[0])


if __name__ == "__main__":
    main()
