#!/usr/bin/env python
"""HGA attention fwd+bwd tokens/s per layer (Qwen3-8B attention shape).

One step = one pass of the whole hot path over one sequence of the workload:
for every segment, in order: summaries of the segment's keys, two-level
routing, exact-token attention forward, and (for training workloads) the
backward under segment-wise backprop.  The default workload is the 16384-token
sequence processed as 8 segments of 2048 with forward and backward
(32 query heads, 8 KV heads, d=128, bf16, top-16 blocks then top-64 groups).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl hga|reference]

With N > 1 (torchrun, one process per GPU) every rank runs its own sequence
(different seed): the units shard with no data-path exchange ("weak" scaling);
the only collective is the max over ranks of the timed duration.

Timing: W untimed warm-up steps; then K steps, each bracketed by CUDA events on
the launching stream, with a 512 MiB write between steps (outside the events)
to flush the 126 MB L2; barrier + synchronize around the whole loop.
Per-kernel durations come from libhga's own event brackets around each launch
inside the same timed steps.
"""

from __future__ import annotations

import argparse
import dataclasses
import datetime
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "HGA attn fwd+bwd tokens/s per layer (Qwen3-8B shape); % of TC/HBM roofline"
DEFAULT_WORKLOAD = "qwen3_fwdbwd_16k"
FP32_ALU_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12   # SMs x FP32 lanes x FMA x max clock


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=30)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", choices=["hga", "reference"], default="hga")
    p.add_argument("--workload", default=DEFAULT_WORKLOAD)
    p.add_argument("--eager", action="store_true",
                   help="launch every step from the host instead of replaying a CUDA graph")
    p.add_argument("--simt", action="store_true", help="force the CUDA-core attention kernels")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-clocks", action="store_true")
    p.add_argument("--no-extra", action="store_true",
                   help="skip the 131072-token forward and the decode measurements")
    p.add_argument("--tier-sweep", action="store_true",
                   help="host-tier sweep: top-k blocks {8,16,32} x context 1K..32K, batch 8")
    args = p.parse_args()
    args.graph = not args.eager
    return args


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        d = json.load(open(path))
        return dict(hbm=d["hbm_gbs"], tc=d["bf16_tflops"], tc_sustained=d["bf16_tflops_sustained"],
                    sm_max_mhz=d.get("sm_max_mhz", 1965.0), source="measured")
    return dict(hbm=6650.0, tc=1590.0, tc_sustained=1400.0, sm_max_mhz=1965.0, source="fallback")


# ----------------------------------------------------------------------------
# distributed plumbing (host logic; tested with gloo on CPU)
# ----------------------------------------------------------------------------

def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", str(rank)))
    return rank, world, local


def rank_workload(w, rank: int):
    """Each rank processes its own sequence: same shapes, seed offset by rank."""
    return dataclasses.replace(w, seed=w.seed + 1000 * rank)


def max_over_ranks(value: float, world: int, device=None) -> float:
    if world == 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(units_per_rank_step: float, steps: int, world: int, max_ms: float) -> float:
    """Whole-job rate: the units all ranks processed over the slowest rank's time."""
    return world * units_per_rank_step * steps / (max_ms / 1e3)


def barrier(world: int, device=None):
    if world > 1:
        import torch.distributed as dist
        dist.barrier(device_ids=[device.index] if device is not None and device.type == "cuda"
                     else None)


# ----------------------------------------------------------------------------
# clocks during the timed region
# ----------------------------------------------------------------------------

class ClockSampler:
    """SM clock and clock-event reasons sampled during the timed region (read
    only).  NVML polled every 5 ms from a thread; nvidia-smi at 100 ms if the
    NVML binding is missing."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    # NVML clock-event reason bits
    REASON_BITS = (("sw_power_cap", 0x4), ("hw_slowdown", 0x8),
                   ("sw_thermal_slowdown", 0x20), ("hw_thermal_slowdown", 0x40))

    def __init__(self, gpu_id=None):
        self.proc = self.thread = None
        self.samples = []
        try:
            import pynvml
            pynvml.nvmlInit()
            h = (pynvml.nvmlDeviceGetHandleByUUID(gpu_id) if gpu_id
                 else pynvml.nvmlDeviceGetHandleByIndex(0))
            self.nvml, self.handle = pynvml, h
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self.nvml = None
        if self.nvml is not None:
            import threading
            self.stop_evt = threading.Event()
            self.sample()
            self.thread = threading.Thread(target=self.poll, daemon=True)
            self.thread.start()
            return
        self.file = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
               "-lms", "100"]
        if gpu_id:
            cmd += ["-i", gpu_id]
        try:
            self.proc = subprocess.Popen(cmd, stdout=self.file, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def sample(self):
        nv, h = self.nvml, self.handle
        try:
            mhz = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
            get = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                nv.nvmlDeviceGetCurrentClocksThrottleReasons
            self.samples.append((float(mhz), int(get(h))))
        except Exception:
            pass

    def poll(self):
        while not self.stop_evt.wait(0.005):
            self.sample()

    def stop(self):
        if self.thread is not None:
            self.stop_evt.set()
            self.thread.join(timeout=5)
            self.sample()
            if not self.samples:
                return None
            reasons = {name for _, bits in self.samples for name, bit in self.REASON_BITS
                       if bits & bit}
            return {"sm_mhz": statistics.median(m for m, _ in self.samples),
                    "sm_max_mhz": float(self.max_mhz), "samples": len(self.samples),
                    "reasons": sorted(reasons), "source": "nvml, 5 ms"}
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.file.seek(0)
        rows = [r.split(",") for r in self.file.read().strip().splitlines() if r.strip()]
        os.unlink(self.file.name)
        sm, mx, reasons = [], [], set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for r in rows:
            r = [x.strip() for x in r]
            try:
                sm.append(float(r[1]))
                mx.append(float(r[2]))
            except (ValueError, IndexError):
                continue
            for name, val in zip(names, r[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(name)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "samples": len(sm),
                "reasons": sorted(reasons), "source": "nvidia-smi, 100 ms"}


# ----------------------------------------------------------------------------
# algorithmic work per kernel kind (the roofline numerators)
# ----------------------------------------------------------------------------

def segment_pairs(w, sel_grp, q_begin):
    """(all attended (query row, key) pairs, pairs on active-segment keys)."""
    import numpy as np
    G, d = w.group_heads, w.head_dim
    valid = sel_grp >= 0
    routed = valid.sum(axis=-1) * 8                          # keys per (b, h, j)
    active = (valid & (sel_grp * 8 >= q_begin)).sum(axis=-1) * 8
    own = 64 * 65 // 2                                       # causal pairs of one block
    rows = G * 64
    all_pairs = int((routed * rows).sum() + own * G * routed.size)
    act_pairs = int((active * rows).sum() + own * G * routed.size)
    return all_pairs, act_pairs


def kernel_work(name, w, sels, unique_groups=None, from_summaries=False):
    """Algorithmic work of ALL launches of kernel `name` over one step.
    Returns (amount, unit, bound): FLOP for contractions, bytes otherwise."""
    unique_groups = unique_groups or {}
    d, S, B = w.head_dim, w.seg_len, w.batch
    Hq, Hkv = w.n_q_heads, w.n_kv_heads
    el = 2 if w.dtype == "bf16" else 4
    n_qb = S // 64
    tot = 0.0
    for q_begin, sel in sels:
        pairs, act = segment_pairs(w, sel, q_begin)
        own0 = q_begin // 64
        Js = [own0 + j for j in range(n_qb)]
        kb = [min(w.topk_blocks, J) for J in Js]
        # each routing kernel counts only the segments whose path it runs:
        # one launch up to 512 candidate blocks, three kernels beyond
        one_launch = own0 + n_qb - 1 <= 512
        if (name == "route_fused" and not one_launch) or (
                name in ("route_qbar", "route_block_topk", "route_select") and one_launch):
            continue
        n_chunks = -(-(own0 + n_qb - 1) // 128)       # candidate chunks of 128 blocks
        if name.startswith("attn_fwd"):
            tot += 4 * d * pairs
        elif name.startswith("attn_bwd_dq"):
            tot += 6 * d * pairs
        elif name.startswith("attn_bwd_dkdv"):
            # the increment over dQ: dV = P^T dO and dK = dS^T Q, 2d each per
            # active pair (the kernel recomputes S and dP, 4d more, which the
            # dQ kernel's 6d already counts)
            tot += 4 * d * act
        elif name == "summaries":
            tot += B * Hkv * (S * d * el + (S // 8 + S // 64) * d * 4)
        elif name == "route_qbar":
            # Q once, q-bar written
            tot += B * (Hq * S * d * el + Hkv * n_qb * d * 4)
        elif name == "route_block_topk":
            # each block summary of the head once, q-bar, the finalists
            # (key and index, k_b + 1 per chunk and query block) written
            tot += B * Hkv * ((own0 + n_qb - 1) * d * 4 + n_qb * d * 4
                              + n_chunks * n_qb * (w.topk_blocks + 1) * 8)
        elif name == "route_select":
            # the finalists and q-bar read, the kept blocks' group summaries,
            # the two selections written
            tot += B * Hkv * sum(n_chunks * (w.topk_blocks + 1) * 8 + d * 4 + 8 * k * d * 4
                                 + 4 * (w.topk_blocks + w.topk_groups) for k in kb)
        elif name == "route_fused":
            # Q once (unless q-bar comes from the resident block means), each
            # block summary of the head once, the kept blocks' group
            # summaries, the two selections written
            tot += (0 if from_summaries else B * Hq * S * d * el) + B * Hkv * (
                (own0 + n_qb - 1) * d * 4
                + sum(8 * k * d * 4 + 4 * (w.topk_blocks + w.topk_groups) for k in kb))
        elif name == "tier_copy":
            tot += 2 * 2 * unique_groups.get(q_begin, 0) * 8 * d * el   # read host + write HBM
        elif name == "tier_dedup":
            tot += B * Hkv * n_qb * w.topk_groups * 8
    if name.startswith("attn"):
        return tot, "FLOP", "alu" if name.endswith("simt") else "tensor"
    if name == "tier_copy":
        return tot / 2, "B", "pcie"          # bytes that cross PCIe (the host reads)
    return tot, "B", "hbm"


# the source files each kernel's device code comes from, besides the shared
# device headers and the C header they include
KERNEL_SOURCE = {
    "summaries": ("summaries.cuh",), "route_fused": ("route.cuh",),
    "route_qbar": ("route.cuh",), "route_block_topk": ("route.cuh",),
    "route_select": ("route.cuh",), "query_summaries": ("route.cuh",),
    "attn_fwd_tc": ("attn_fwd_sm100.cuh",), "attn_bwd_dq_tc": ("attn_bwd_sm100.cuh",),
    "attn_bwd_dkdv_tc": ("attn_bwd_sm100.cuh",), "attn_fwd_simt": ("attn_simt.cuh",),
    "attn_bwd_dq_simt": ("attn_simt.cuh",), "attn_bwd_dkdv_simt": ("attn_simt.cuh",),
    "tier_dedup": ("tier.cuh",), "tier_copy": ("tier.cuh",),
    "decode": ("decode.cuh", "route.cuh"), "prepare": ("prepare.cuh",),
}
SHARED_SOURCES = ("hga_common.cuh", "sm100_ptx.cuh")


def source_hash(kernel=None):
    """Hash of the sources a kernel is compiled from (all of csrc/ when the
    kernel is not listed), so that a stored ncu figure is used only while
    they are unchanged."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "hierarchical_routed_sparse_hga_b200", "csrc")
    if kernel in KERNEL_SOURCE:
        paths = [os.path.join(csrc, f) for f in SHARED_SOURCES + KERNEL_SOURCE[kernel]]
        paths.append(os.path.join(ROOT, "include", "hga.h"))
    else:
        paths = [os.path.join(csrc, f) for f in sorted(os.listdir(csrc))]
    for f in paths:
        h.update(open(f, "rb").read())
    return h.hexdigest()[:16]


def measured_traffic(kernel, workload):
    """DRAM bytes per launch from the committed ncu summary, if it matches the
    current kernel sources; else None."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.json")
    if not os.path.exists(path):
        return None
    d = json.load(open(path))
    e = d.get(workload, {}).get(kernel)
    if not e or e.get("source_hash") != source_hash(kernel):
        return None
    return e.get("bytes_per_launch")


# ----------------------------------------------------------------------------
# the GPU arm
# ----------------------------------------------------------------------------

class Runner:
    def __init__(self, w, device, flags=0):
        import torch
        from hierarchical_routed_sparse_hga_b200 import HGA_BF16, HGA_F32, Config, HgaLayer
        from hierarchical_routed_sparse_hga_b200 import synth
        self.w, self.device = w, device
        self.dt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
        cfg = Config(w.batch, w.n_q_heads, w.n_kv_heads, w.head_dim, w.topk_blocks,
                     w.topk_groups, HGA_BF16 if w.dtype == "bf16" else HGA_F32, flags)

        def dev(a):
            return self.to_torch(a).to(device)

        self.k_host = self.to_torch(synth.keys(w)).pin_memory()
        self.v_host = self.to_torch(synth.values(w)).pin_memory()
        self.layer = HgaLayer(cfg, w.ctx_len, w.seg_len, device=device,
                              k=self.k_host.to(device), v=self.v_host.to(device))
        self.segs = w.segments()
        # each segment's K/V rows as one contiguous pinned block [B, Hkv, rows,
        # d] (the first segment's also holds the history before it), so that
        # each goes up in one copy per tensor
        self.kv_host_seg = []
        for i, q_begin in enumerate(self.segs):
            lo, hi = (0 if i == 0 else q_begin), q_begin + w.seg_len
            self.kv_host_seg.append((lo, hi, self.k_host[:, :, lo:hi].contiguous().pin_memory(),
                                     self.v_host[:, :, lo:hi].contiguous().pin_memory()))
        self.q_host = [self.to_torch(synth.queries(w, s)).pin_memory() for s in self.segs]
        self.q = [t.to(device) for t in self.q_host]
        if w.backward:
            self.do_host = [self.to_torch(synth.douts(w, s)).pin_memory() for s in self.segs]
            self.do = [t.to(device) for t in self.do_host]
        self.history_end = self.segs[0]
        if self.history_end:
            # history before the first query-carrying segment: resident summaries
            from hierarchical_routed_sparse_hga_b200 import hga_build_summaries
            hga_build_summaries(self.layer.cfg, self.layer.k, w.ctx_len, 0, self.history_end,
                                self.layer.gsum, self.layer.bsum)
        torch.cuda.synchronize(device)

    def to_torch(self, a):
        import numpy as np
        import torch
        if self.w.dtype == "bf16":
            return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16)
        return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32))

    def step(self, record_sel=None, causal=False):
        L = self.layer
        for i, q_begin in enumerate(self.segs):
            L.segment(self.q[i], q_begin, self.do[i] if self.w.backward else None,
                      causal=causal)
            if record_sel is not None:
                record_sel.append((q_begin, L.sel_grp.cpu().numpy()))

    def e2e_step(self, out_host):
        """Host buffers in, host buffers out, through the runtime: every
        segment's K/V rows, Q and dO go up on an upload stream (segment i's
        while segment i-1 computes), the segment runs on the current stream,
        and its outputs come down on a download stream while the next segment
        computes (two output sets alternate).  The step ends when the last
        outputs are on the host."""
        import torch
        L, w = self.layer, self.w
        if not hasattr(self, "s_up"):
            self.s_up = torch.cuda.Stream(self.device)
            self.s_down = torch.cuda.Stream(self.device)
            self.out_sets = [L.make_outputs() for _ in range(2)]
        comp = torch.cuda.current_stream(self.device)
        # this step's uploads overwrite what the previous step computed from
        self.s_up.wait_stream(comp)
        up_done = []
        with torch.cuda.stream(self.s_up):
            for i, q_begin in enumerate(self.segs):
                # the segment's K/V block in one copy per tensor (a contiguous
                # source; the rows land in the whole-context buffers through a
                # device-side copy, while a strided source would be staged
                # through the host)
                lo, hi, kh, vh = self.kv_host_seg[i]
                L.k[:, :, lo:hi].copy_(kh, non_blocking=True)
                L.v[:, :, lo:hi].copy_(vh, non_blocking=True)
                self.q[i].copy_(self.q_host[i], non_blocking=True)
                if w.backward:
                    self.do[i].copy_(self.do_host[i], non_blocking=True)
                ev = torch.cuda.Event()
                ev.record(self.s_up)
                up_done.append(ev)
        down_done = []
        for i, q_begin in enumerate(self.segs):
            comp.wait_event(up_done[i])
            if i >= 2:
                comp.wait_event(down_done[i - 2])       # its output set is free again
            out = self.out_sets[i & 1]
            L.segment(self.q[i], q_begin, self.do[i] if w.backward else None, out=out)
            ev = torch.cuda.Event()
            ev.record(comp)
            self.s_down.wait_event(ev)
            srcs = (out[0], out[2], out[3], out[4]) if w.backward else (out[0],)
            with torch.cuda.stream(self.s_down):
                for dst, src in zip(out_host[i], srcs):
                    dst.copy_(src, non_blocking=True)
                ev2 = torch.cuda.Event()
                ev2.record(self.s_down)
                down_done.append(ev2)
        comp.wait_stream(self.s_down)

    def io_bytes(self):
        nb = lambda t: t.numel() * t.element_size()  # noqa: E731
        h2d = sum(nb(kh) + nb(vh) for _, _, kh, vh in self.kv_host_seg)
        h2d += sum(nb(t) for t in self.q_host)
        L = self.layer
        outs = (L.o, L.dq, L.dk, L.dv) if self.w.backward else (L.o,)
        if self.w.backward:
            h2d += sum(nb(t) for t in self.do_host)
        d2h = len(self.segs) * sum(nb(t) for t in outs)
        return h2d, d2h


class TierRunner:
    """Host-tier workload: history K/V in pinned host memory, inputs drawn on
    the device (synth.device_inputs).  One step = every segment: place the
    segment's K/V in staging, summaries, route, tier gather over PCIe,
    forward, backward, append of the segment's K/V to the host history."""

    def __init__(self, w, device, flags=0):
        import torch
        from hierarchical_routed_sparse_hga_b200 import (HGA_BF16, HGA_F32, Config,
                                                         HgaTieredLayer, synth)
        self.w, self.device = w, device
        cfg = Config(w.batch, w.n_q_heads, w.n_kv_heads, w.head_dim, w.topk_blocks,
                     w.topk_groups, HGA_BF16 if w.dtype == "bf16" else HGA_F32, flags)
        self.k, self.v, self.q, self.do = synth.device_inputs(w, device, w.backward)
        self.layer = HgaTieredLayer(cfg, w.ctx_len, w.seg_len, device=device)
        self.segs = w.segments()
        torch.cuda.synchronize(device)

    def step(self, record_sel=None):
        L, S = self.layer, self.w.seg_len
        for i, q_begin in enumerate(self.segs):
            L.active_k().copy_(self.k[:, :, q_begin:q_begin + S])
            L.active_v().copy_(self.v[:, :, q_begin:q_begin + S])
            L.segment(self.q[i], q_begin, self.do[i] if self.w.backward else None)
            if record_sel is not None:
                record_sel.append((q_begin, L.sel_grp.cpu().numpy(),
                                   int(L.n_unique.sum().item())))

    def pcie_bytes(self, sels):
        """Bytes over PCIe per step: gathered groups (K+V) and appended segments."""
        w = self.w
        el = 2 if w.dtype == "bf16" else 4
        gathered = sum(u for _, _, u in sels) * 2 * 8 * w.head_dim * el
        appended = len(self.segs) * 2 * w.batch * w.n_kv_heads * w.seg_len * w.head_dim * el
        return gathered, appended


def pcie_probe(device, nbytes=256 << 20, reps=5):
    """Pinned host -> device copy bandwidth (GB/s), best of `reps`."""
    import torch
    h = torch.empty(nbytes, dtype=torch.uint8).pin_memory()
    d = torch.empty(nbytes, dtype=torch.uint8, device=device)
    best = 0.0
    for _ in range(reps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        d.copy_(h, non_blocking=True)
        e1.record()
        torch.cuda.synchronize(device)
        best = max(best, nbytes / (e0.elapsed_time(e1) / 1e3) / 1e9)
    return best


def dense_sdpa_tokens_per_s(w, device, reps=3):
    """Dense causal attention (torch SDPA, bf16) fwd+bwd over the whole
    context at the workload's shape: the in-run reference point."""
    import torch
    import torch.nn.functional as F
    B, H, T, d = w.batch, w.n_q_heads, w.ctx_len, w.head_dim
    q = torch.randn((B, H, T, d), device=device, dtype=torch.bfloat16, requires_grad=True)
    k = torch.randn((B, w.n_kv_heads, T, d), device=device, dtype=torch.bfloat16,
                    requires_grad=True)
    v = torch.randn_like(k, requires_grad=True)
    go = torch.randn((B, H, T, d), device=device, dtype=torch.bfloat16)

    def run():
        o = F.scaled_dot_product_attention(q, k, v, is_causal=True, enable_gqa=True)
        o.backward(go)

    run()
    torch.cuda.synchronize(device)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(reps):
        run()
    e1.record()
    torch.cuda.synchronize(device)
    return B * T * reps / (e0.elapsed_time(e1) / 1e3)


def run_tier_sweep(args, device):
    import torch
    from hierarchical_routed_sparse_hga_b200 import synth
    peak = pcie_probe(device)
    for kb in (8, 16, 32):
        for L in (1024, 2048, 4096, 8192, 16384, 32768):
            w = synth.custom(f"tier_b8_L{L}_kb{kb}", batch=8, n_q_heads=32, n_kv_heads=8,
                             head_dim=128, ctx_len=L, seg_len=min(2048, L), topk_blocks=kb,
                             topk_groups=4 * kb, dtype="bf16", scaled=True, rope_base=1e6,
                             seed=4)
            run = TierRunner(w, device)
            sels = []
            run.step(record_sel=sels)
            torch.cuda.synchronize(device)
            steps = 2
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            for _ in range(steps):
                run.step()
            e1.record()
            torch.cuda.synchronize(device)
            ms = e0.elapsed_time(e1) / steps
            gathered, appended = run.pcie_bytes(sels)
            dense = dense_sdpa_tokens_per_s(w, device)
            print(json.dumps({
                "sweep": "tier", "context": L, "topk_blocks": kb, "topk_groups": 4 * kb,
                "batch": 8, "seg_len": w.seg_len, "tokens_per_s": round(8 * L / (ms / 1e3), 1),
                "ms_per_step": round(ms, 3), "pcie_gather_bytes": gathered,
                "pcie_append_bytes": appended,
                "pcie_gbs": round((gathered + appended) / (ms / 1e3) / 1e9, 2),
                "pcie_probe_h2d_gbs": round(peak, 2),
                "dense_sdpa_tokens_per_s": round(dense, 1)}), flush=True)
            del run
            torch.cuda.empty_cache()


def run_gpu(args, rank, world, local):
    import numpy as np
    import torch
    from hierarchical_routed_sparse_hga_b200 import (HGA_FLAG_SIMT, HGA_K_COUNT,
                                                     hga_kernel_name, hga_launch_count,
                                                     hga_timing_collect, hga_timing_enable,
                                                     hga_timing_kinds, hga_timing_reset, synth,
                                                     timing_table)
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=device)
    if args.tier_sweep:
        run_tier_sweep(args, device)
        return
    w0 = synth.workloads()[args.workload]
    w = rank_workload(w0, rank)
    tiered = "tiered" in w.name
    run = (TierRunner if tiered else Runner)(w, device, HGA_FLAG_SIMT if args.simt else 0)
    tokens_per_step = w.batch * len(run.segs) * w.seg_len

    sels = []
    run.step(record_sel=sels)                       # first warm-up step records selections
    unique_groups = {rec[0]: rec[2] for rec in sels if len(rec) > 2}
    sels = [(rec[0], rec[1]) for rec in sels]
    for _ in range(max(args.warmup, 3) - 1):
        run.step()
    torch.cuda.synchronize(device)

    per_step_launches = None
    graph = None
    n0 = hga_launch_count()
    run.step()
    torch.cuda.synchronize(device)
    per_step_launches = hga_launch_count() - n0
    slots = per_step_launches + 16
    flush = torch.empty(512 << 20, dtype=torch.uint8, device=device)

    def capture():
        g = torch.cuda.CUDAGraph()
        cs = torch.cuda.Stream(device)
        cs.wait_stream(torch.cuda.current_stream(device))
        with torch.cuda.stream(cs):
            with torch.cuda.graph(g, stream=cs):
                run.step()
        torch.cuda.current_stream(device).wait_stream(cs)
        return g

    kinds = {hga_kernel_name(k): k for k in range(HGA_K_COUNT)}
    table_all = None
    table_dom = None
    gpu_id = None
    try:
        gpu_id = f"GPU-{torch.cuda.get_device_properties(device).uuid}"
    except Exception:
        pass
    if args.graph:
        # Events between two kernels cut their programmatic dependency (and
        # the per-item overlap of the fused forward + backward), so the
        # headline graph carries no per-kernel events.  Two other graphs give
        # the per-kernel numbers: one with every launch bracketed (the table,
        # 3 untimed replays) and one with only the dominant kernel bracketed
        # (its launch time for the roofline, over its own K timed steps).
        hga_timing_kinds(0xFFFFFFFF)
        hga_timing_enable(slots)
        g_all = capture()
        hga_timing_reset()
        for _ in range(3):
            flush.zero_()
            g_all.replay()
            hga_timing_collect()
        torch.cuda.synchronize(device)
        table_all = timing_table()
        del g_all
        dom_name = max(table_all, key=lambda k: table_all[k][0])
        hga_timing_kinds(1 << kinds[dom_name])
        hga_timing_enable(slots)
        g_dom = capture()
        hga_timing_reset()
        barrier(world, device)
        torch.cuda.synchronize(device)
        for _ in range(args.steps):
            flush.zero_()
            g_dom.replay()
            hga_timing_collect()
        torch.cuda.synchronize(device)
        table_dom = timing_table()
        del g_dom
        hga_timing_enable(0)
        hga_timing_kinds(0xFFFFFFFF)
        graph = capture()
        graph.replay()
        torch.cuda.synchronize(device)
    hga_timing_reset()

    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    sampler = None if args.no_clocks else ClockSampler(gpu_id)
    barrier(world, device)
    torch.cuda.synchronize(device)
    launches0 = hga_launch_count()
    for i in range(args.steps):
        flush.zero_()
        if graph is None:
            hga_timing_enable(slots)
        starts[i].record()
        if graph is not None:
            graph.replay()
        else:
            run.step()
        ends[i].record()
        if graph is None:
            hga_timing_collect()
    torch.cuda.synchronize(device)
    barrier(world, device)
    launches = hga_launch_count() - launches0
    if graph is not None:
        launches = per_step_launches * args.steps   # graph replays bypass the host counter
    clocks = sampler.stop() if sampler else None
    hga_timing_enable(0)
    hga_timing_kinds(0xFFFFFFFF)

    step_ms = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    total_ms = max_over_ranks(sum(step_ms), world, device)
    value = job_throughput(tokens_per_step, args.steps, world, total_ms)

    # per-kernel table and the dominant kernel's roofline: in graph mode the
    # table comes from the fully bracketed graph (3 untimed replays), the
    # dominant kernel's launch time from the timed replays
    pk = peaks()
    pcie_peak = []

    def roof(bound):
        """(peak, unit, scale to that unit, note) for a bound."""
        if bound == "tensor":
            # each launch is timed on its own (events around the kernel, a few
            # tens of microseconds), so the burst figure applies
            return pk["tc"], "TFLOP/s", 1e12, f"bf16 dense, burst ({pk['source']})"
        if bound == "alu":
            return (FP32_ALU_TFLOPS, "TFLOP/s", 1e12,
                    "fp32 FFMA: 148 SMs x 128 lanes x 2 x 1965 MHz")
        if bound == "pcie":
            if not pcie_peak:
                pcie_peak.append(round(pcie_probe(device), 2))
            return (pcie_peak[0], "GB/s", 1e9,
                    "pinned host-to-device cudaMemcpyAsync probe, 256 MiB, best of 5")
        return pk["hbm"], "GB/s", 1e9, f"HBM copy ({pk['source']})"

    table = table_dom if table_dom is not None else timing_table()
    shown, reps = (table_all, 3) if table_all is not None else (table, args.steps)
    kernels = {}
    tot_ms = max(sum(v[0] for v in shown.values()), 1e-12)
    for name, (ms, n) in shown.items():
        work, unit, bound = kernel_work(name, w, sels, unique_groups)
        per_launch = work / (n / reps)
        peak, punit, scale, _ = roof(bound)
        achieved = per_launch / (ms / n / 1e3) / scale
        kernels[name] = {"launches": n, "ms_total": round(ms, 4), "share": round(ms / tot_ms, 4),
                         "avg_us": round(ms / n * 1e3, 3), "bound": bound,
                         "achieved": round(achieved, 3), "unit": punit,
                         "frac": round(achieved / peak, 4)}
    dom = max(table, key=lambda k: table[k][0])
    dom_ms, dom_n = table[dom]
    work, unit, bound = kernel_work(dom, w, sels, unique_groups)
    work_per_launch = work / (dom_n / args.steps)
    avg_s = dom_ms / dom_n / 1e3
    peak, punit, scale, peak_note = roof(bound)
    achieved = work_per_launch / avg_s / scale
    roofline = {"kernel": dom, "bound": bound, "achieved": round(achieved, 3),
                "peak": peak, "unit": punit, "frac": round(achieved / peak, 4),
                "traffic": measured_traffic(dom, args.workload),
                "work_per_launch": work_per_launch, "work_unit": unit,
                "avg_launch_us": round(avg_s * 1e6, 3), "peak_source": peak_note,
                **({"peak_sustained": pk["tc_sustained"],
                    "frac_of_sustained": round(achieved / pk["tc_sustained"], 4)}
                   if bound == "tensor" else {}),
                "timed": ("CUDA events around each launch of this kernel only, over K graph "
                          "replays of their own before the headline ones (events between "
                          "kernels would cut the programmatic overlap the headline measures)"
                          if args.graph else "CUDA events around every launch of the timed "
                          "steps")}

    # end to end through the public API with pinned host buffers
    e2e = None
    if not args.no_e2e and not tiered:
        L = run.layer
        outs = (L.o, L.dq, L.dk, L.dv) if w.backward else (L.o,)
        out_host = [[torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in outs]
                    for _ in run.segs]
        run.e2e_step(out_host)
        torch.cuda.synchronize(device)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier(world, device)
        e0.record()
        for _ in range(args.steps):
            run.e2e_step(out_host)
        e1.record()
        torch.cuda.synchronize(device)
        barrier(world, device)
        e_ms = max_over_ranks(e0.elapsed_time(e1), world, device)
        h2d, d2h = run.io_bytes()
        e2e = {"value": round(job_throughput(tokens_per_step, args.steps, world, e_ms), 1),
               "unit": "tokens/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h}

    extra = None
    if world == 1 and not args.no_extra and not tiered:
        extra = run_extras(device, max(args.steps // 2, 5), pk, run)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(w0, budget_s=15.0)

    if rank == 0:
        line = {
            "metric": METRIC, "value": round(value, 1), "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(total_ms / args.steps, 4), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": w.dtype, "data": "synthetic",
            "config": workload_config(args.workload, w, world),
            "launch": {"graph": bool(args.graph), "attention": "simt" if args.simt else "auto"},
            "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e,
            "gpu_launches": int(launches), "clocks": clocks, "kernels": kernels,
            "extra": extra,
        }
        print(json.dumps(line), flush=True)
    if graph is not None:
        del graph
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


# ----------------------------------------------------------------------------
# extra measurements on one GPU: the 131072-token forward and decode
# ----------------------------------------------------------------------------

def decode_bytes(w, positions):
    """Algorithmic HBM bytes of one hga_decode call: per (sequence, KV head)
    the J block summaries, the 8 k_b group summaries of the kept blocks, the
    attended K/V rows (8 k_g routed + the own block up to the token), the G
    query rows in and the G output rows and LSE out."""
    d, G, el = w.head_dim, w.group_heads, (2 if w.dtype == "bf16" else 4)
    tot = 0
    for p in positions:
        J = p // 64
        kb = min(w.topk_blocks, J)
        kg = min(w.topk_groups, 8 * kb)
        rows = 8 * kg + (p - 64 * J + 1)
        tot += w.n_kv_heads * (J * d * 4 + 8 * kb * d * 4 + rows * d * el * 2
                               + 2 * G * d * el + G * 4)
    return tot


def run_extras(device, steps, pk, run=None):
    """The 131072-token forward (64 segments of 2048, the long-context
    workload) with its per-kernel table, and decode (one new token per
    sequence, batch 8 at position 131071, four layers' caches in turn so
    that the working set exceeds L2)."""
    import torch
    from hierarchical_routed_sparse_hga_b200 import (HGA_BF16, HGA_K_COUNT, Config, HgaLayer,
                                                     hga_build_summaries, hga_kernel_name,
                                                     hga_timing_collect, hga_timing_enable,
                                                     hga_timing_reset, synth, timing_table)
    out = {}
    flush = torch.empty(512 << 20, dtype=torch.uint8, device=device)

    def graph_of(fn):
        g = torch.cuda.CUDAGraph()
        cs = torch.cuda.Stream(device)
        cs.wait_stream(torch.cuda.current_stream(device))
        with torch.cuda.stream(cs):
            with torch.cuda.graph(g, stream=cs):
                fn()
        torch.cuda.current_stream(device).wait_stream(cs)
        return g

    # -- the same fwd+bwd workload with strictly causal routing ------------
    if run is not None and not run.w.name.startswith("qwen3_tiered"):
        run.step(causal=True)
        g = graph_of(lambda: run.step(causal=True))
        g.replay()
        ms = []
        for _ in range(steps):
            flush.zero_()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            g.replay()
            e1.record()
            torch.cuda.synchronize(device)
            ms.append(e0.elapsed_time(e1))
        del g
        tokens = run.w.batch * len(run.segs) * run.w.seg_len
        out["causal_routing"] = {
            "workload": run.w.name, "routing": "hga_route_causal (previous block's mean query)",
            "tokens_per_s": round(tokens / (statistics.mean(ms) / 1e3), 1),
            "ms_per_step": round(statistics.mean(ms), 4),
            "timing": "graph replay per step, CUDA events, L2 flushed between steps"}

    # -- the same fwd+bwd workload from the projection outputs ---------------
    if run is not None and not run.w.name.startswith("qwen3_tiered") and run.w.backward:
        w = run.w
        cfg = run.layer.cfg
        k, v, qs, dos = synth.device_inputs(w, device)
        segs = w.segments()
        S = w.seg_len
        # token-major [B, S, H, d] projection outputs of every segment
        qproj = [q.transpose(1, 2).contiguous() for q in qs]
        kproj = [k[:, :, s0:s0 + S].transpose(1, 2).contiguous() for s0 in segs]
        vproj = [v[:, :, s0:s0 + S].transpose(1, 2).contiguous() for s0 in segs]
        del k, v, qs
        Lp = HgaLayer(cfg, w.ctx_len, S, device=device)
        q_out = torch.empty((w.batch, w.n_q_heads, S, w.head_dim), dtype=torch.bfloat16,
                            device=device)

        def pstep():
            for i, s0 in enumerate(segs):
                Lp.segment_from_projections(qproj[i], kproj[i], vproj[i],
                                            w.n_q_heads * w.head_dim, w.n_kv_heads * w.head_dim,
                                            s0, w.rope_base, q_out, dos[i])

        pstep()
        hga_timing_enable(8 * len(segs) + 16)
        g_all = graph_of(pstep)
        hga_timing_reset()
        for _ in range(3):
            flush.zero_()
            g_all.replay()
            hga_timing_collect()
        torch.cuda.synchronize(device)
        ptable = timing_table()
        hga_timing_enable(0)
        del g_all
        g = graph_of(pstep)
        g.replay()
        ms = []
        for _ in range(steps):
            flush.zero_()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            g.replay()
            e1.record()
            torch.cuda.synchronize(device)
            ms.append(e0.elapsed_time(e1))
        del g
        el = 2
        B, Hq, Hkv, d = w.batch, w.n_q_heads, w.n_kv_heads, w.head_dim
        # per launch: read Q/K/V projections, write Q, K, V, the summaries and block means
        prep_bytes = (2 * B * S * (Hq + 2 * Hkv) * d * el
                      + B * Hkv * (S // 8 + 2 * (S // 64)) * d * 4)
        pk_ms, pk_n = ptable.get("prepare", (0.0, 0))
        prep = None
        if pk_n:
            ach = prep_bytes / (pk_ms / pk_n / 1e3) / 1e9
            prep = {"avg_us": round(pk_ms / pk_n * 1e3, 3), "bytes_per_launch": prep_bytes,
                    "achieved": round(ach, 1), "unit": "GB/s",
                    "frac": round(ach / pk["hbm"], 4)}
        tokens = B * len(segs) * S
        out["from_projections"] = {
            "workload": w.name,
            "step": "per segment: hga_prepare_segment (RoPE, layout, summaries, block means) -> "
                    "hga_route_summarized -> hga_attn_fwd_bwd; inputs are the token-major "
                    "projection outputs",
            "tokens_per_s": round(tokens / (statistics.mean(ms) / 1e3), 1),
            "ms_per_step": round(statistics.mean(ms), 4),
            "prepare_kernel": prep,
            "kernel_us_per_step": {n: round(v_[0] / 3 * 1e3, 2) for n, v_ in ptable.items()}}
        del Lp, qproj, kproj, vproj, dos
        torch.cuda.empty_cache()

    # -- 131072-token forward --------------------------------------------
    w = synth.workloads()["qwen3_fwd_128k"]
    cfg = Config(w.batch, w.n_q_heads, w.n_kv_heads, w.head_dim, w.topk_blocks, w.topk_groups,
                 HGA_BF16)
    k, v, qs, _ = synth.device_inputs(w, device, backward=False)
    layer = HgaLayer(cfg, w.ctx_len, w.seg_len, device=device, k=k, v=v)
    segs = w.segments()

    def step(record=None):
        for i, s0 in enumerate(segs):
            layer.segment(qs[i], s0)
            if record is not None:
                record.append((s0, layer.sel_grp.cpu().numpy()))

    sels = []
    step(sels)
    step()
    n_launch = 6 * len(segs)           # summaries, up to 3 routing kernels, forward
    hga_timing_enable(n_launch + 16)
    g_all = graph_of(step)
    hga_timing_reset()
    for _ in range(3):
        flush.zero_()
        g_all.replay()
        hga_timing_collect()
    torch.cuda.synchronize(device)
    table = timing_table()
    hga_timing_enable(0)
    del g_all
    g = graph_of(step)
    g.replay()
    ms = []
    for _ in range(steps):
        flush.zero_()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        g.replay()
        e1.record()
        torch.cuda.synchronize(device)
        ms.append(e0.elapsed_time(e1))
    del g
    step_ms = statistics.mean(ms)
    kernels = {}
    tot = max(sum(v_[0] for v_ in table.values()), 1e-12)
    for name, (kms, n) in table.items():
        work, unit, bound = kernel_work(name, w, sels)
        per_launch = work / (n / 3)
        peak = pk["tc"] if bound == "tensor" else pk["hbm"]
        scale = 1e12 if bound == "tensor" else 1e9
        ach = per_launch / (kms / n / 1e3) / scale
        kernels[name] = {"launches": n // 3, "share": round(kms / tot, 4),
                         "avg_us": round(kms / n * 1e3, 3), "bound": bound,
                         "achieved": round(ach, 3),
                         "unit": "TFLOP/s" if bound == "tensor" else "GB/s",
                         "frac": round(ach / peak, 4)}
    route_names = [n for n in kernels if n.startswith("route")]
    route_us = sum(table[n][0] for n in route_names) / 3 * 1e3
    route_bytes = sum(kernel_work(n, w, sels)[0] for n in route_names)
    out["long_context_fwd"] = {
        "workload": w.name, "seq_len": w.ctx_len, "segments": len(segs),
        "tokens_per_s": round(w.ctx_len / (step_ms / 1e3), 1), "ms_per_step": round(step_ms, 4),
        "timing": "graph replay per step, CUDA events, L2 flushed between steps; kernel "
                  "table from 3 replays with every launch bracketed",
        "routing": {"us_per_step": round(route_us, 2),
                    "achieved_gbs": round(route_bytes / (route_us / 1e6) / 1e9, 1),
                    "frac_of_hbm": round(route_bytes / (route_us / 1e6) / 1e9 / pk["hbm"], 4)},
        "kernels": kernels}
    del layer, k, v, qs
    torch.cuda.empty_cache()

    # -- the file (NVMe) tier on the batched tiered workload -------------------
    from hierarchical_routed_sparse_hga_b200 import HgaFileTieredLayer
    wt = synth.workloads()["qwen3_tiered_b8_32k"]
    cfg = Config(wt.batch, wt.n_q_heads, wt.n_kv_heads, wt.head_dim, wt.topk_blocks,
                 wt.topk_groups, HGA_BF16)
    k, v, qs, dos = synth.device_inputs(wt, device)
    tmp = tempfile.mkdtemp(prefix="hga_tier_")
    nbytes = k.numel() * k.element_size()
    fds = []
    for name in ("k.bin", "v.bin"):
        fd = os.open(os.path.join(tmp, name), os.O_RDWR | os.O_CREAT, 0o600)
        os.ftruncate(fd, nbytes)
        fds.append(fd)
    try:
        tier = HgaFileTieredLayer(cfg, wt.ctx_len, wt.seg_len, fds[0], fds[1], device=device,
                                  n_threads=16)
        S = wt.seg_len

        def tstep():
            for i, s0 in enumerate(wt.segments()):
                tier.active_k().copy_(k[:, :, s0:s0 + S])
                tier.active_v().copy_(v[:, :, s0:s0 + S])
                tier.segment(qs[i], s0, dos[i])

        tstep()
        tier.bytes_read = 0
        t_steps = 2
        torch.cuda.synchronize(device)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(t_steps):
            tstep()
        e1.record()
        torch.cuda.synchronize(device)
        t_ms = e0.elapsed_time(e1) / t_steps
        read = tier.bytes_read / t_steps
        out["file_tier"] = {
            "workload": wt.name, "batch": wt.batch, "seq_len": wt.ctx_len,
            "segments": len(wt.segments()),
            "tokens_per_s": round(wt.batch * wt.ctx_len / (t_ms / 1e3), 1),
            "ms_per_step": round(t_ms, 2), "file_bytes_read_per_step": int(read),
            "file_read_gbs_over_step": round(read / (t_ms / 1e3) / 1e9, 2),
            "timing": "CUDA events around whole steps; each segment's planned groups are read "
                      "from the files by 16 host threads (pread) between the GPU phases; the "
                      "files were just written, so the reads may be served by the page cache",
        }
        del tier
    finally:
        for fd in fds:
            os.close(fd)
        for name in ("k.bin", "v.bin"):
            os.unlink(os.path.join(tmp, name))
        os.rmdir(tmp)
    del k, v, qs, dos
    torch.cuda.empty_cache()

    # -- decode ------------------------------------------------------------
    wd = synth.custom("qwen3_decode_b8_128k", batch=8, n_q_heads=32, n_kv_heads=8, head_dim=128,
                      ctx_len=131072, seg_len=2048, topk_blocks=16, topk_groups=64,
                      dtype="bf16", scaled=True, rope_base=1e6, seed=40)
    n_layers = 4
    positions = [wd.ctx_len - 1] * wd.batch
    layers = []
    cfg = Config(wd.batch, wd.n_q_heads, wd.n_kv_heads, wd.head_dim, wd.topk_blocks,
                 wd.topk_groups, HGA_BF16)
    for li in range(n_layers):
        k, v, q_tok = synth.device_decode_inputs(dataclasses.replace(wd, seed=40 + li),
                                                 positions, device)
        L = HgaLayer(cfg, wd.ctx_len, wd.seg_len, device=device, k=k, v=v)
        hga_build_summaries(cfg, L.k, wd.ctx_len, 0, wd.ctx_len, L.gsum, L.bsum)
        layers.append((L, q_tok))
    pos = torch.tensor(positions, dtype=torch.int64, device=device)
    o = torch.empty((wd.batch, wd.n_q_heads, wd.head_dim), dtype=torch.bfloat16, device=device)
    lse = torch.empty((wd.batch, wd.n_q_heads), device=device)
    reps = 20

    def dstep():
        for L, q_tok in layers:
            L.decode(q_tok, pos, o, lse)

    for _ in range(3):
        dstep()
    g = graph_of(lambda: [dstep() for _ in range(reps)])
    g.replay()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(steps):
        g.replay()
    e1.record()
    torch.cuda.synchronize(device)
    call_us = e0.elapsed_time(e1) * 1e3 / (steps * reps * n_layers)
    byts = decode_bytes(wd, positions)
    ach = byts / (call_us / 1e6) / 1e9
    out["decode"] = {
        "workload": wd.name, "batch": wd.batch, "position": positions[0],
        "layers_in_turn": n_layers, "us_per_layer_call": round(call_us, 3),
        "tokens_per_s_per_layer": round(wd.batch / (call_us / 1e6), 1),
        "timing": f"CUDA graph of {reps} x {n_layers} back-to-back calls (each layer its own "
                  "K/V and summaries: 17 GB working set, above L2), CUDA events around the "
                  "replays",
        "roofline": {"bound": "hbm", "achieved": round(ach, 1), "peak": pk["hbm"],
                     "unit": "GB/s", "frac": round(ach / pk["hbm"], 4),
                     "bytes_per_call": byts}}
    del layers, g
    torch.cuda.empty_cache()
    return out


# ----------------------------------------------------------------------------
# the CPU oracle (baseline and reference arm)
# ----------------------------------------------------------------------------

def oracle_sample(w, q_begin, kv_heads):
    """Oracle work of one segment restricted to `kv_heads`: summaries of the
    history and the segment, routing, forward and backward.  Returns tokens of
    full-layer work it stands for (segment tokens x share of heads)."""
    import numpy as np
    import oracle
    from hierarchical_routed_sparse_hga_b200 import synth
    G = w.group_heads
    qh = [h * G + g for h in kv_heads for g in range(G)]
    k = synth.widen(synth.keys(w, kv_heads), w.dtype)
    v = synth.widen(synth.values(w, kv_heads), w.dtype)
    q = synth.widen(synth.queries(w, q_begin, qh), w.dtype)
    do = synth.widen(synth.douts(w, q_begin, qh), w.dtype) if w.backward else None
    T = q_begin + w.seg_len
    t0 = time.perf_counter()
    gsum = np.zeros((w.batch, len(kv_heads), w.ctx_len // 8, w.head_dim))
    bsum = np.zeros((w.batch, len(kv_heads), w.ctx_len // 64, w.head_dim))
    if q_begin:
        g, b = oracle.build_summaries(k, 0, q_begin)
        gsum[:, :, :q_begin // 8], bsum[:, :, :q_begin // 64] = g, b
    oracle.segment_step(q, k, v, do, q_begin, gsum, bsum, w.topk_blocks, w.topk_groups,
                        len(kv_heads), backward=w.backward)
    dt = time.perf_counter() - t0
    return w.batch * w.seg_len * len(kv_heads) / w.n_kv_heads, dt, T


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return os.cpu_count() or 1


def cpu_baseline(w, budget_s=15.0):
    """Oracle on a bounded sample: the last segment, KV heads taken one at a time
    until about budget_s seconds of CPU work."""
    q_begin = w.segments()[-1]
    tokens, secs, heads = 0.0, 0.0, []
    for h in range(w.n_kv_heads):
        t, dt, _ = oracle_sample(w, q_begin, [h])
        tokens += t
        secs += dt
        heads.append(h)
        if secs >= budget_s:
            break
    return {"value": round(tokens / secs, 2), "unit": "tokens/s", "cores": blas_threads(),
            "kind": "oracle",
            "sample": f"{args_workload_name(w)}: segment at q_begin={q_begin} "
                      f"({'fwd+bwd' if w.backward else 'fwd'}, summaries+route+attention), "
                      f"KV heads {heads} of {w.n_kv_heads} (their {w.group_heads} query heads "
                      f"each); tokens counted as seg_len x heads/{w.n_kv_heads}; "
                      f"{secs:.1f} s of float64 NumPy"}


def args_workload_name(w):
    return w.name


def workload_config(name, w, world):
    """The workload part of the JSON line's config, the same in both arms."""
    return {"workload": name, "batch_per_gpu": w.batch, "seq_len": w.ctx_len,
            "seg_len": w.seg_len, "n_q_heads": w.n_q_heads, "n_kv_heads": w.n_kv_heads,
            "head_dim": w.head_dim, "topk_blocks": w.topk_blocks,
            "topk_groups": w.topk_groups, "backward": w.backward,
            "parallelism": f"replicas{world}",
            "l2": "GPU arm: flushed between timed steps (512 MiB write, untimed); "
                  "oracle arm: host caches"}


def run_reference(args, rank, world):
    if rank != 0:
        return
    from hierarchical_routed_sparse_hga_b200 import synth
    w = synth.workloads()[args.workload]
    q_begin = w.segments()[-1]
    for i in range(args.warmup):
        oracle_sample(w, q_begin, [i % w.n_kv_heads])
    tokens, secs = 0.0, 0.0
    for i in range(args.steps):
        t, dt, _ = oracle_sample(w, q_begin, [i % w.n_kv_heads])
        tokens += t
        secs += dt
    value = tokens / secs
    sample = (f"{w.name}: per step the oracle on the segment at q_begin={q_begin}, one KV "
              f"head (rotating) of {w.n_kv_heads}; tokens counted as seg_len/{w.n_kv_heads}")
    line = {"impl": "reference", "metric": METRIC, "value": round(value, 2), "unit": "tokens/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(secs / args.steps * 1e3, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_config(w.name, w, world),
            "launch": {"attention": "oracle (float64 NumPy on the host cores)"},
            "cpu_baseline": {"value": round(value, 2), "unit": "tokens/s",
                             "cores": blas_threads(), "kind": "oracle", "sample": sample},
            "e2e": {"value": round(value, 2), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    args = parse()
    rank, world, local = dist_env()
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    run_gpu(args, rank, world, local)


if __name__ == "__main__":
    main()
