"""Seeded synthetic decode workloads for the Hybrid-Block attention path.

This module only *builds inputs*: queries, paged K/V caches, page tables and
sequence lengths, with planted "needle" keys so that token selection is not
trivial.  It contains none of the attention, scoring or selection arithmetic;
the CUDA library and the CPU oracle both consume what it produces.

Input recipe (the same on every device; a seeded ``torch.Generator``):
  * Q, K, V ~ N(0, 1) in fp32, then rounded to the storage type
    (bf16 round-to-nearest-even, or E4M3 with a per-(slot, kv-head) fp32 scale
    amax/448, codes rounded to nearest-even and clamped to +-448);
  * needle keys: 3*u + N(0, 0.1^2) per element, u the unit vector of the sum of
    the full-attention query heads of the KV head's group; placed among the
    selectable positions [0, T - window), uniformly without replacement, or in
    equal bursts of consecutive positions (multi-turn tool-output shape);
  * paged caches use a seeded permutation of all pages as the page table;
    slots past the end of each sequence hold finite N(0,1) data unless
    ``pad_fill="nan"`` asks for NaNs there (robustness cases).
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional, Tuple, Union

import numpy as np
import torch

__all__ = ["WorkloadSpec", "Workload", "WORKLOADS", "generate", "raw", "slots_of"]


@dataclasses.dataclass(frozen=True)
class WorkloadSpec:
    name: str
    batch: int
    num_kv_heads: int
    group: int
    head_dim: int
    seq_len: Union[int, Tuple[int, int]]  # fixed, or (lo, hi) uniform inclusive
    kv_dtype: str  # "f32" | "bf16" | "e4m3"
    q_dtype: str  # "f32" | "bf16"
    page_size: Optional[int]  # None: contiguous cache (capacity rounded up to 64)
    sparse_layers: int
    needles: int = 0  # per (sequence, KV head)
    needle_bursts: int = 0  # 0: uniform placement; else this many equal bursts
    window: int = 128
    k_global: int = 1024

    @property
    def num_q_heads(self) -> int:
        return self.num_kv_heads * self.group

    def replace(self, **kw) -> "WorkloadSpec":
        return dataclasses.replace(self, **kw)


# The five decode workloads of the Hybrid-Block path (window 128, k_global 1024).
WORKLOADS = {
    s.name: s
    for s in [
        WorkloadSpec("tiny_fp32_t2048", 1, 1, 4, 64, 2048, "f32", "f32", None, 2, needles=8),
        WorkloadSpec("decode_b8_32k_bf16", 8, 4, 8, 128, 32768, "bf16", "bf16", None, 3, needles=64),
        WorkloadSpec("paged_b64_8k_128k_bf16", 64, 4, 8, 128, (8192, 131072), "bf16", "bf16", 64, 3,
                     needles=32),
        WorkloadSpec("ctx256k_b4_bf16_paged", 4, 4, 8, 128, 262144, "bf16", "bf16", 64, 3,
                     needles=256, needle_bursts=8),
        WorkloadSpec("ctx1m_b1_fp8_paged", 1, 4, 8, 128, 1048576, "e4m3", "bf16", 64, 3, needles=1024),
        # the compact MQA configuration: one KV head shared by all 32 query heads
        WorkloadSpec("mqa_ctx256k_b4_bf16_paged", 4, 1, 32, 128, 262144, "bf16", "bf16", 64, 3,
                     needles=256, needle_bursts=8),
        WorkloadSpec("mqa_ctx1m_b1_fp8_paged", 1, 1, 32, 128, 1048576, "e4m3", "bf16", 64, 3, needles=1024),
    ]
}

_TORCH = {"f32": torch.float32, "bf16": torch.bfloat16, "e4m3": torch.uint8}
E4M3_MAX = 448.0


@dataclasses.dataclass
class Workload:
    spec: WorkloadSpec
    q_full: torch.Tensor  # [B, Hq, d] storage dtype
    q_sparse: torch.Tensor  # [Ls, B, Hq, d]
    k: torch.Tensor  # [num_slots, Hkv, d] (uint8 codes for e4m3)
    v: torch.Tensor
    k_scale: Optional[torch.Tensor]  # [num_slots, Hkv] fp32 (e4m3 only)
    v_scale: Optional[torch.Tensor]
    seq_lens: torch.Tensor  # [B] int32
    page_table: Optional[torch.Tensor]  # [B, max_pages] int32, or None (contiguous)
    page_size: int  # page size, or per-sequence capacity when contiguous
    needle_pos: list  # per (b, kvh): sorted logical positions of the needles

    @property
    def max_pages(self) -> int:
        return 1 if self.page_table is None else self.page_table.shape[1]

    @property
    def num_slots(self) -> int:
        return self.k.shape[0]

    @property
    def t_cap(self) -> int:
        return self.page_size * self.max_pages


def _quantize_e4m3(x: torch.Tensor):
    """fp32 rows [..., d] -> (uint8 E4M3 codes, fp32 scale per row)."""
    amax = x.abs().amax(dim=-1)
    scale = torch.where(amax > 0, amax / E4M3_MAX, torch.ones_like(amax))
    y = (x / scale.unsqueeze(-1)).clamp(-E4M3_MAX, E4M3_MAX)
    return y.to(torch.float8_e4m3fn).view(torch.uint8), scale.float()


def _store(x: torch.Tensor, dtype: str):
    if dtype == "e4m3":
        return _quantize_e4m3(x)
    return x.to(_TORCH[dtype]), None


def slots_of(w: Workload, b: int, t: torch.Tensor) -> torch.Tensor:
    """Physical slots of logical positions ``t`` of sequence ``b`` (the
    address rule of the cache layout: page_table[b, t // P] * P + t % P, or
    b * capacity + t for the contiguous layout)."""
    t = t.to(torch.int64)
    if w.page_table is None:
        return b * w.page_size + t
    pt = w.page_table[b].to(torch.int64).to(t.device)
    return pt[t // w.page_size] * w.page_size + t % w.page_size


def _needle_positions(gen, n_cand: int, n: int, bursts: int, device) -> torch.Tensor:
    n = min(n, n_cand)
    if n <= 0:
        return torch.zeros(0, dtype=torch.int64)
    if bursts <= 0:
        pos = torch.randperm(n_cand, generator=gen, device=device)[:n]
        return torch.sort(pos.cpu()).values
    per = n // bursts
    if per * bursts > n_cand:
        return torch.arange(n_cand)
    starts = []
    while len(starts) < bursts:
        s = int(torch.randint(0, n_cand - per + 1, (1,), generator=gen, device=device).item())
        if all(abs(s - o) >= per for o in starts):  # overlap -> redraw
            starts.append(s)
    return torch.sort(torch.cat([torch.arange(s, s + per) for s in starts])).values


def generate(spec: WorkloadSpec, seed: int = 0, device="cpu", pad_fill: Optional[str] = None,
             seq_lens=None, chunk_slots: int = 1 << 19) -> Workload:
    """Build one seeded workload on ``device``.  ``seq_lens`` overrides the
    spec's lengths (edge cases); ``pad_fill="nan"`` writes NaN into every slot
    that no sequence position maps to."""
    device = torch.device(device)
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    B, Hkv, G, d = spec.batch, spec.num_kv_heads, spec.group, spec.head_dim
    Hq = Hkv * G
    if seq_lens is not None:
        lens = torch.as_tensor(seq_lens, dtype=torch.int32)
        assert lens.numel() == B
    elif isinstance(spec.seq_len, tuple):
        lo, hi = spec.seq_len
        lens = torch.randint(lo, hi + 1, (B,), generator=gen, device=device).to(torch.int32).cpu()
    else:
        lens = torch.full((B,), spec.seq_len, dtype=torch.int32)
    lens_l = [int(x) for x in lens]

    q_full32 = torch.randn(B, Hq, d, generator=gen, device=device)
    q_sparse32 = torch.randn(spec.sparse_layers, B, Hq, d, generator=gen, device=device)
    q_full = q_full32.to(_TORCH[spec.q_dtype])
    q_sparse = q_sparse32.to(_TORCH[spec.q_dtype])

    if spec.page_size is None:
        cap = max(64, -(-max(lens_l) // 64) * 64)
        page_size, page_table, num_slots = cap, None, B * cap
    else:
        page_size = spec.page_size
        npages = [-(-t // page_size) for t in lens_l]
        total = sum(npages)
        perm = torch.randperm(max(total, 1), generator=gen, device=device).cpu().to(torch.int32)
        max_pages = max(max(npages), 1)
        page_table = torch.zeros(B, max_pages, dtype=torch.int32)
        off = 0
        for b, n in enumerate(npages):
            page_table[b, :n] = perm[off:off + n]
            off += n
        num_slots = max(total, 1) * page_size
        page_table = page_table.to(device)

    kv_dt = spec.kv_dtype
    store_dt = _TORCH[kv_dt]
    k = torch.empty(num_slots, Hkv, d, dtype=store_dt, device=device)
    v = torch.empty(num_slots, Hkv, d, dtype=store_dt, device=device)
    k_scale = v_scale = None
    if kv_dt == "e4m3":
        k_scale = torch.empty(num_slots, Hkv, dtype=torch.float32, device=device)
        v_scale = torch.empty(num_slots, Hkv, dtype=torch.float32, device=device)
    for dst, sc in ((k, k_scale), (v, v_scale)):
        for s0 in range(0, num_slots, chunk_slots):
            s1 = min(num_slots, s0 + chunk_slots)
            x = torch.randn(s1 - s0, Hkv, d, generator=gen, device=device)
            codes, scale = _store(x, kv_dt)
            dst[s0:s1] = codes
            if sc is not None:
                sc[s0:s1] = scale
            del x

    w = Workload(spec, q_full, q_sparse, k, v, k_scale, v_scale, lens, page_table, page_size, [])

    # needles: 3*u + N(0, 0.1^2), u = direction of the group's summed full-layer query
    qg = q_full.float().view(B, Hkv, G, d).sum(dim=2)
    u = qg / qg.norm(dim=-1, keepdim=True).clamp_min(1e-30)
    for b in range(B):
        n_cand = max(0, lens_l[b] - spec.window)
        for h in range(Hkv):
            pos = _needle_positions(gen, n_cand, spec.needles, spec.needle_bursts, device)
            w.needle_pos.append(pos.tolist())
            if pos.numel() == 0:
                continue
            noise = torch.randn(pos.numel(), d, generator=gen, device=device)
            rows = 3.0 * u[b, h].unsqueeze(0) + 0.1 * noise
            codes, scale = _store(rows, kv_dt)
            sl = slots_of(w, b, pos.to(device))
            k[sl, h] = codes
            if k_scale is not None:
                k_scale[sl, h] = scale

    if pad_fill == "nan":
        used = torch.zeros(num_slots, dtype=torch.bool, device=device)
        for b in range(B):
            used[slots_of(w, b, torch.arange(lens_l[b], device=device))] = True
        nan_code = {"f32": float("nan"), "bf16": float("nan")}
        for dst in (k, v):
            if kv_dt == "e4m3":
                dst[~used] = 0x7F
            else:
                dst[~used] = nan_code[kv_dt]
    elif pad_fill is not None:
        raise ValueError(pad_fill)
    w.seq_lens = lens.to(device)
    return w


def raw(t: Optional[torch.Tensor]) -> Optional[np.ndarray]:
    """Stored bytes of a tensor as a numpy array (bf16 -> uint16 bit patterns)."""
    if t is None:
        return None
    t = t.detach().cpu().contiguous()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.numpy()
