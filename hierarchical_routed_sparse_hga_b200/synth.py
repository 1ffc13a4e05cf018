"""Seeded synthetic inputs for the HGA hot path.

This module only draws and lays out inputs; it holds none of the method's
arithmetic (no summaries, no routing, no attention).  Both the CUDA path and
the CPU oracle are fed from it.  It imports nothing else from this package.

Recipe (one reading of the workloads the HGA pages and the five workload
descriptions give; "Long-Context Fine-Tuning with Limited VRAM", method
description of two-level routing over 64-token blocks and 8-token groups):

* every (batch b, KV head h, 64-token block c) has a centroid C ~ N(0, I_d);
* K[b,h,t] = C[b,h,t//64] + 0.5 * N(0, I_d);   V ~ N(0, I_d);  dO ~ N(0, I_d);
* Q[b,h',t] = C[b,h,r] + 0.5 * N(0, I_d) with h = h' // G and r a planted
  "target" block drawn uniformly, per (b, KV head, segment, query block), from
  the history blocks before the segment (the query block's own block when the
  segment has no history).  All G heads and all 64 tokens of the query block
  share r and draw independent noise;
* scaled workloads (the Qwen3-8B-shaped ones) multiply Q and K by 1/sqrt(d),
  then apply NeoX rotate-half RoPE (base 1e6, position = global token index)
  in float64;
* values are rounded once: float64 -> float32 (round to nearest even) and,
  for bf16 workloads, float32 -> bf16 (round to nearest even).

Every tensor is drawn from its own counter-style stream,
``numpy.random.default_rng(SeedSequence([seed, tensor_id, b, head, seg]))``,
so any slice (one head, one segment) can be regenerated alone and chunked
generation of large workloads gives the same values as whole generation.

bf16 arrays are returned as ``uint16`` bit patterns; ``bf16_to_f64`` widens
them exactly.
"""

from __future__ import annotations

import dataclasses
import math

import numpy as np

BLOCK = 64
GROUP = 8
QBLOCK = 64

# tensor ids for the per-tensor streams
_T_CENTROID, _T_KNOISE, _T_V, _T_TARGET, _T_QNOISE, _T_DO, _T_DEC_TARGET, _T_DEC_Q, \
    _T_PROJ = range(9)


@dataclasses.dataclass(frozen=True)
class Workload:
    """Shape and distribution of one synthetic HGA workload."""

    name: str
    batch: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    ctx_len: int            # total tokens in the sequence (history + every segment)
    seg_len: int            # active segment length
    topk_blocks: int
    topk_groups: int
    dtype: str              # "f32" or "bf16"
    scaled: bool            # multiply Q, K by 1/sqrt(d)
    rope_base: float | None
    seed: int
    first_seg: int = 0      # segments before this one are history only (no Q)
    backward: bool = True

    @property
    def n_seg(self) -> int:
        return self.ctx_len // self.seg_len

    @property
    def group_heads(self) -> int:
        return self.n_q_heads // self.n_kv_heads

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.head_dim)

    def segments(self):
        """Global start token of every segment that carries queries."""
        return [s * self.seg_len for s in range(self.first_seg, self.n_seg)]


def workloads() -> dict:
    """The five workloads, by name.

    tiny_f32            d=64 fp32, 2048 history + one 256-token segment
    qwen3_fwd_16k       Qwen3-8B layer shape, one 2048 segment after 14336 history
    qwen3_fwdbwd_16k    same shape, 8 segments of 2048 over 16384 tokens, fwd+bwd
    qwen3_fwd_128k      same shape, 64 segments of 2048 over 131072 tokens, fwd only
    qwen3_tiered_b8_32k batch 8 x 32768 tokens, 16 segments each, fwd+bwd
    """
    q3 = dict(n_q_heads=32, n_kv_heads=8, head_dim=128, dtype="bf16", scaled=True,
              rope_base=1.0e6)
    return {
        "tiny_f32": Workload("tiny_f32", 1, 1, 1, 64, 2048 + 256, 256, 4, 16, "f32",
                             False, None, seed=0, first_seg=8),
        "qwen3_fwd_16k": Workload("qwen3_fwd_16k", 1, ctx_len=16384, seg_len=2048,
                                  topk_blocks=16, topk_groups=64, seed=1, first_seg=7,
                                  backward=False, **q3),
        "qwen3_fwdbwd_16k": Workload("qwen3_fwdbwd_16k", 1, ctx_len=16384, seg_len=2048,
                                     topk_blocks=16, topk_groups=64, seed=2, **q3),
        "qwen3_fwd_128k": Workload("qwen3_fwd_128k", 1, ctx_len=131072, seg_len=2048,
                                   topk_blocks=16, topk_groups=64, seed=3, backward=False,
                                   **q3),
        "qwen3_tiered_b8_32k": Workload("qwen3_tiered_b8_32k", 8, ctx_len=32768,
                                        seg_len=2048, topk_blocks=16, topk_groups=64,
                                        seed=4, **q3),
    }


def custom(name="custom", *, batch=1, n_q_heads=4, n_kv_heads=1, head_dim=64,
           ctx_len=512, seg_len=256, topk_blocks=2, topk_groups=8, dtype="f32",
           scaled=False, rope_base=None, seed=0, first_seg=0, backward=True) -> Workload:
    """A workload of any shape with the same distributions (tests use it)."""
    return Workload(name, batch, n_q_heads, n_kv_heads, head_dim, ctx_len, seg_len,
                    topk_blocks, topk_groups, dtype, scaled, rope_base, seed,
                    first_seg, backward)


# ----------------------------------------------------------------------------
# rounding helpers
# ----------------------------------------------------------------------------

def f32_to_bf16_bits(x32: np.ndarray) -> np.ndarray:
    """Round float32 to bf16 (nearest, ties to even); return uint16 bits."""
    u = np.ascontiguousarray(x32, dtype=np.float32).view(np.uint32)
    bias = np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))
    return ((u + bias) >> np.uint32(16)).astype(np.uint16)


def bf16_to_f32(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << np.uint32(16)).view(np.float32)


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    return bf16_to_f32(bits).astype(np.float64)


def to_storage(x64: np.ndarray, dtype: str) -> np.ndarray:
    """float64 -> float32 (RNE) -> [bf16 bits (RNE)]."""
    x32 = x64.astype(np.float32)
    return f32_to_bf16_bits(x32) if dtype == "bf16" else x32


def widen(a: np.ndarray, dtype: str) -> np.ndarray:
    """Storage array -> exact float64 values."""
    return bf16_to_f64(a) if dtype == "bf16" else a.astype(np.float64)


# ----------------------------------------------------------------------------
# streams
# ----------------------------------------------------------------------------

def _rng(w: Workload, tensor: int, *idx: int) -> np.random.Generator:
    return np.random.default_rng(np.random.SeedSequence([w.seed, tensor, *idx]))


def _rope(x: np.ndarray, pos0: int, base: float) -> np.ndarray:
    """NeoX rotate-half rotary embedding of rows x[t] at positions pos0 + t."""
    n, d = x.shape
    half = d // 2
    inv = base ** (-np.arange(half, dtype=np.float64) * 2.0 / d)
    ang = (pos0 + np.arange(n, dtype=np.float64))[:, None] * inv[None, :]
    c, s = np.cos(ang), np.sin(ang)
    x1, x2 = x[:, :half], x[:, half:]
    return np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=1)


def centroids(w: Workload, b: int, h: int) -> np.ndarray:
    """[ctx_len/64, d] float64 block centroids of one (batch, KV head)."""
    return _rng(w, _T_CENTROID, b, h).standard_normal((w.ctx_len // BLOCK, w.head_dim))


def _prep(x: np.ndarray, w: Workload, pos0: int) -> np.ndarray:
    if w.scaled:
        x = x * w.scale
    if w.rope_base is not None:
        x = _rope(x, pos0, w.rope_base)
    return x


def keys_head(w: Workload, b: int, h: int) -> np.ndarray:
    """Post-RoPE K of one (batch, KV head) over the whole context, storage dtype."""
    c = centroids(w, b, h)
    noise = _rng(w, _T_KNOISE, b, h).standard_normal((w.ctx_len, w.head_dim))
    k = np.repeat(c, BLOCK, axis=0) + 0.5 * noise
    return to_storage(_prep(k, w, 0), w.dtype)


def values_head(w: Workload, b: int, h: int) -> np.ndarray:
    v = _rng(w, _T_V, b, h).standard_normal((w.ctx_len, w.head_dim))
    return to_storage(v, w.dtype)


def targets(w: Workload, b: int, h: int, seg_begin: int) -> np.ndarray:
    """Planted target block r per query block of the segment starting at seg_begin."""
    n_qb = w.seg_len // QBLOCK
    n_hist = seg_begin // BLOCK
    if n_hist == 0:
        return seg_begin // BLOCK + np.arange(n_qb)
    rng = _rng(w, _T_TARGET, b, h, seg_begin // w.seg_len)
    return rng.integers(0, n_hist, size=n_qb)


def queries_head(w: Workload, b: int, hq: int, seg_begin: int) -> np.ndarray:
    """Post-RoPE Q of one (batch, query head) for one segment, storage dtype."""
    h = hq // w.group_heads
    c = centroids(w, b, h)
    r = targets(w, b, h, seg_begin)
    base = np.repeat(c[r], QBLOCK, axis=0)
    noise = _rng(w, _T_QNOISE, b, hq, seg_begin // w.seg_len).standard_normal(
        (w.seg_len, w.head_dim))
    return to_storage(_prep(base + 0.5 * noise, w, seg_begin), w.dtype)


def dout_head(w: Workload, b: int, hq: int, seg_begin: int) -> np.ndarray:
    rng = _rng(w, _T_DO, b, hq, seg_begin // w.seg_len)
    return to_storage(rng.standard_normal((w.seg_len, w.head_dim)), w.dtype)


def projections(w: Workload, seg_begin: int):
    """Token-major projection outputs of one segment before RoPE: q_proj
    [B, S, Hq, d], k_proj and v_proj [B, S, Hkv, d], storage dtype.  Keys and
    queries follow the recipe above (centroids, planted target blocks, 0.5
    noise, the 1/sqrt(d) scale of scaled workloads) without the rotation,
    which the upstream pass applies; drawn from their own streams."""
    S, G = w.seg_len, w.group_heads
    B, Hq, Hkv, d = w.batch, w.n_q_heads, w.n_kv_heads, w.head_dim
    qp = np.empty((B, S, Hq, d))
    kp = np.empty((B, S, Hkv, d))
    vp = np.empty((B, S, Hkv, d))
    scale = w.scale if w.scaled else 1.0
    seg = seg_begin // w.seg_len
    for b in range(B):
        for h in range(Hkv):
            c = centroids(w, b, h)
            kn = _rng(w, _T_PROJ, 0, b, h, seg).standard_normal((S, d))
            kp[b, :, h] = (np.repeat(c[seg_begin // BLOCK:(seg_begin + S) // BLOCK], BLOCK, axis=0)
                           + 0.5 * kn) * scale
            vp[b, :, h] = _rng(w, _T_PROJ, 1, b, h, seg).standard_normal((S, d))
            r = targets(w, b, h, seg_begin)
            for g in range(G):
                qn = _rng(w, _T_PROJ, 2, b, h * G + g, seg).standard_normal((S, d))
                qp[b, :, h * G + g] = (np.repeat(c[r], QBLOCK, axis=0) + 0.5 * qn) * scale
    return tuple(to_storage(t, w.dtype) for t in (qp, kp, vp))


def decode_query_head(w: Workload, b: int, hq: int, pos: int) -> np.ndarray:
    """Post-RoPE query [d] of the token at global position pos (a decode
    step): the centroid of a planted block drawn uniformly from the complete
    blocks before the token's own block (its own block when there are none),
    plus 0.5 * N(0, I_d); the planted block is shared by the G heads."""
    h = hq // w.group_heads
    n_before = pos // BLOCK
    r = (_rng(w, _T_DEC_TARGET, b, h, pos).integers(0, n_before) if n_before
         else n_before)
    noise = _rng(w, _T_DEC_Q, b, hq, pos).standard_normal(w.head_dim)
    x = centroids(w, b, h)[r] + 0.5 * noise
    return to_storage(_prep(x[None, :], w, pos)[0], w.dtype)


def decode_queries(w: Workload, positions) -> np.ndarray:
    """[B, Hq, d] decode queries, sequence b at global position positions[b]."""
    return np.stack([np.stack([decode_query_head(w, b, hq, int(positions[b]))
                               for hq in range(w.n_q_heads)]) for b in range(w.batch)])


# ----------------------------------------------------------------------------
# whole tensors (layouts of the C ABI: K, V [B,Hkv,T,d]; Q, dO [B,Hq,S,d])
# ----------------------------------------------------------------------------

def keys(w: Workload, heads=None) -> np.ndarray:
    hs = range(w.n_kv_heads) if heads is None else heads
    return np.stack([np.stack([keys_head(w, b, h) for h in hs]) for b in range(w.batch)])


def values(w: Workload, heads=None) -> np.ndarray:
    hs = range(w.n_kv_heads) if heads is None else heads
    return np.stack([np.stack([values_head(w, b, h) for h in hs]) for b in range(w.batch)])


def queries(w: Workload, seg_begin: int, q_heads=None) -> np.ndarray:
    hs = range(w.n_q_heads) if q_heads is None else q_heads
    return np.stack([np.stack([queries_head(w, b, hq, seg_begin) for hq in hs])
                     for b in range(w.batch)])


def douts(w: Workload, seg_begin: int, q_heads=None) -> np.ndarray:
    hs = range(w.n_q_heads) if q_heads is None else q_heads
    return np.stack([np.stack([dout_head(w, b, hq, seg_begin) for hq in hs])
                     for b in range(w.batch)])


# ----------------------------------------------------------------------------
# the same recipe drawn on the device with torch (large performance sweeps)
# ----------------------------------------------------------------------------

def device_inputs(w: Workload, device, backward=True):
    """K, V [B,Hkv,T,d] and per-segment Q, dO [B,Hq,S,d] drawn on `device`.

    Same distributions and layout as the NumPy streams above (centroids per
    block, 0.5 noise, planted target blocks, 1/sqrt(d) scaling and RoPE for
    scaled workloads), drawn from torch's generator seeded with w.seed: the
    values differ from the NumPy streams, so parity tests never use this; it
    exists because drawing gigabytes of inputs with NumPy takes minutes.
    """
    import torch
    dt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    g = torch.Generator(device=device)
    g.manual_seed(w.seed)
    B, Hkv, Hq, T, S, d = w.batch, w.n_kv_heads, w.n_q_heads, w.ctx_len, w.seg_len, w.head_dim
    G = w.group_heads

    def rope(x, pos0):
        if w.rope_base is None:
            return x
        half = d // 2
        inv = w.rope_base ** (-torch.arange(half, device=device, dtype=torch.float64) * 2.0 / d)
        pos = pos0 + torch.arange(x.shape[-2], device=device, dtype=torch.float64)
        ang = pos[:, None] * inv[None, :]
        c, s = torch.cos(ang).float(), torch.sin(ang).float()
        x1, x2 = x[..., :half], x[..., half:]
        return torch.cat([x1 * c - x2 * s, x2 * c + x1 * s], dim=-1)

    scale = w.scale if w.scaled else 1.0
    cent = torch.randn((B, Hkv, T // BLOCK, d), generator=g, device=device)
    k = cent.repeat_interleave(BLOCK, dim=2) + 0.5 * torch.randn((B, Hkv, T, d), generator=g,
                                                                   device=device)
    k = rope(k * scale, 0).to(dt)
    v = torch.randn((B, Hkv, T, d), generator=g, device=device).to(dt)
    qs, dos = [], []
    n_qb = S // QBLOCK
    for s0 in w.segments():
        n_hist = s0 // BLOCK
        if n_hist:
            r = torch.randint(0, n_hist, (B, Hkv, n_qb), generator=g, device=device)
        else:
            r = (s0 // BLOCK + torch.arange(n_qb, device=device)).expand(B, Hkv, n_qb)
        base = torch.gather(cent, 2, r[..., None].expand(B, Hkv, n_qb, d))
        base = base.repeat_interleave(QBLOCK, dim=2).repeat_interleave(G, dim=1)
        q = base + 0.5 * torch.randn((B, Hq, S, d), generator=g, device=device)
        qs.append(rope(q * scale, s0).to(dt).contiguous())
        if backward:
            dos.append(torch.randn((B, Hq, S, d), generator=g, device=device).to(dt))
    return k.contiguous(), v.contiguous(), qs, dos


def device_decode_inputs(w: Workload, positions, device):
    """K, V [B,Hkv,T,d] and the decode queries [B,Hq,d] of the tokens at
    `positions`, drawn on `device` with the recipe above (planted block per
    (sequence, KV head) among the complete blocks before the token's own
    block).  Like device_inputs, for performance runs only."""
    import torch
    dt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    g = torch.Generator(device=device)
    g.manual_seed(w.seed)
    B, Hkv, Hq, T, d = w.batch, w.n_kv_heads, w.n_q_heads, w.ctx_len, w.head_dim
    G = w.group_heads
    scale = w.scale if w.scaled else 1.0

    def rope(x, pos):
        if w.rope_base is None:
            return x
        half = d // 2
        inv = w.rope_base ** (-torch.arange(half, device=device, dtype=torch.float64) * 2.0 / d)
        ang = pos.to(torch.float64)[..., None] * inv
        c, s = torch.cos(ang).float(), torch.sin(ang).float()
        x1, x2 = x[..., :half], x[..., half:]
        return torch.cat([x1 * c - x2 * s, x2 * c + x1 * s], dim=-1)

    cent = torch.randn((B, Hkv, T // BLOCK, d), generator=g, device=device)
    k = torch.empty((B, Hkv, T, d), dtype=dt, device=device)
    v = torch.empty((B, Hkv, T, d), dtype=dt, device=device)
    t_idx = torch.arange(T, device=device)
    for b in range(B):                        # one sequence at a time bounds the float32 temporaries
        kb = cent[b].repeat_interleave(BLOCK, dim=1) + 0.5 * torch.randn(
            (Hkv, T, d), generator=g, device=device)
        k[b] = rope(kb * scale, t_idx[None, :].expand(Hkv, T)).to(dt)
        v[b] = torch.randn((Hkv, T, d), generator=g, device=device).to(dt)
    pos = torch.as_tensor(positions, device=device, dtype=torch.int64)
    n_before = torch.clamp(pos // BLOCK, min=1)
    r = (torch.rand((B, Hkv), generator=g, device=device) * n_before[:, None]).long()
    r = torch.where((pos // BLOCK)[:, None] > 0, r, (pos // BLOCK)[:, None].expand(B, Hkv))
    base = torch.gather(cent, 2, r[..., None, None].expand(B, Hkv, 1, d))[:, :, 0]
    q = base.repeat_interleave(G, dim=1) + 0.5 * torch.randn((B, Hq, d), generator=g,
                                                               device=device)
    q = rope(q * scale, pos[:, None].expand(B, Hq)).to(dt)
    return k, v, q.contiguous()
