"""Seeded synthetic inputs shared by the oracle tests, the CUDA parity tests and bench.py.

This module only draws random numbers and casts them; it holds none of the attention
arithmetic. Every tensor is drawn on the CPU from ``torch.Generator`` seeds so that the same
bytes reach the oracle and the GPU.

Recipe (values i.i.d. N(0, 1) drawn in float32, then cast to the storage dtype with
round-to-nearest-even):

* q first, in one draw of shape [B, Hq, D];
* then K: for b in batch order, for each KV head, one draw of [len_b, D] (valid rows only);
* then V in the same order. Rows at positions >= len_b hold ``pad_fill`` (0 by default; the
  bounds tests use NaN so any read past the cache length poisons the result);
* "peaked" K (long-context workload): per (b, KV head), ``peaked_rows`` row indices below len_b
  are drawn without replacement from numpy's default_rng(seed + 200) and those K rows are
  multiplied by ``peak_scale`` in float32 before the cast;
* cache lengths drawn uniformly, both ends inclusive, with numpy default_rng(seed).
* E4M3 caches (``make_fp8``) are the bf16 caches above quantized: one scale per tensor,
  scale = (largest finite |value| over the tensor) / 448 rounded to float32, codes = torch's
  round-to-nearest cast of value / scale to float8_e4m3fn (NaN padding stays NaN).

The named workloads are the six benchmark shapes of this project (decode MHA fp32, decode
MHA bf16 13B-like, decode GQA bf16 70B-like, long-context GQA, mixed chunked-prefill step, and
the 70B-like batch verifying 4 speculative tokens per sequence); tensor seed = 1000 + index,
length seed = 1100 + index (the verification step reuses the 70B-like lengths).
"""

from __future__ import annotations

from dataclasses import dataclass
from typing import Dict, List, Optional

import numpy as np
import torch

__all__ = [
    "DecodeInputs", "ChunkInputs", "uniform_lens", "make_decode_inputs", "make_chunk_inputs",
    "WORKLOADS", "workload", "to_numpy_exact", "Fp8Cache", "quantize_e4m3", "make_fp8",
]


@dataclass
class DecodeInputs:
    q: torch.Tensor            # [B, Hq, D]
    k_cache: torch.Tensor      # [B, Hkv, S_cap, D]
    v_cache: torch.Tensor      # [B, Hkv, S_cap, D]
    cache_lens: torch.Tensor   # int32 [B]
    num_splits: int = 0
    name: str = ""


@dataclass
class ChunkInputs:
    q_chunk: torch.Tensor      # [sum(chunk_lens), Hq, D]
    k_cache: torch.Tensor      # [B, Hkv, S_cap, D]
    v_cache: torch.Tensor
    prefix_lens: torch.Tensor  # int32 [B]
    chunk_lens: torch.Tensor   # int32 [B]
    name: str = ""


def uniform_lens(seed: int, batch: int, lo: int, hi: int) -> List[int]:
    """Integer lengths uniform on [lo, hi], both ends inclusive."""
    return [int(x) for x in np.random.default_rng(seed).integers(lo, hi + 1, size=batch)]


def _fill_cache(gen: torch.Generator, B: int, H: int, S_cap: int, D: int, lens: List[int],
                dtype: torch.dtype, pad_fill: float,
                peak_rows: Optional[Dict[tuple, np.ndarray]] = None,
                peak_scale: float = 8.0) -> torch.Tensor:
    cache = torch.full((B, H, S_cap, D), float(pad_fill), dtype=dtype)
    for b in range(B):
        n = max(0, min(int(lens[b]), S_cap))
        for h in range(H):
            if n == 0:
                continue
            x = torch.randn((n, D), generator=gen, dtype=torch.float32)
            if peak_rows is not None and (b, h) in peak_rows:
                idx = torch.from_numpy(peak_rows[(b, h)].astype(np.int64))
                x[idx] *= peak_scale
            cache[b, h, :n] = x.to(dtype)
    return cache


def make_decode_inputs(batch: int, q_heads: int, kv_heads: int, head_dim: int, capacity: int,
                       lens: List[int], dtype: torch.dtype, seed: int, num_splits: int = 0,
                       pad_fill: float = 0.0, peaked_rows: int = 0, peak_scale: float = 8.0,
                       name: str = "") -> DecodeInputs:
    gen = torch.Generator().manual_seed(seed)
    q = torch.randn((batch, q_heads, head_dim), generator=gen, dtype=torch.float32).to(dtype)
    peaks = None
    if peaked_rows > 0:
        rng = np.random.default_rng(seed + 200)
        peaks = {}
        for b in range(batch):
            n = max(0, min(int(lens[b]), capacity))
            for h in range(kv_heads):
                peaks[(b, h)] = rng.choice(n, size=min(peaked_rows, n), replace=False)
    k = _fill_cache(gen, batch, kv_heads, capacity, head_dim, lens, dtype, pad_fill, peaks,
                    peak_scale)
    v = _fill_cache(gen, batch, kv_heads, capacity, head_dim, lens, dtype, pad_fill)
    return DecodeInputs(q=q, k_cache=k, v_cache=v,
                        cache_lens=torch.tensor(lens, dtype=torch.int32),
                        num_splits=num_splits, name=name)


def make_chunk_inputs(prefix_lens: List[int], chunk_lens: List[int], q_heads: int,
                      kv_heads: int, head_dim: int, capacity: int, dtype: torch.dtype,
                      seed: int, pad_fill: float = 0.0, name: str = "") -> ChunkInputs:
    """Packed query chunks plus a cache holding each request's prefix and chunk K/V."""
    gen = torch.Generator().manual_seed(seed)
    total = int(sum(chunk_lens))
    q = torch.randn((total, q_heads, head_dim), generator=gen, dtype=torch.float32).to(dtype)
    lens = [int(p) + int(c) for p, c in zip(prefix_lens, chunk_lens)]
    B = len(chunk_lens)
    k = _fill_cache(gen, B, kv_heads, capacity, head_dim, lens, dtype, pad_fill)
    v = _fill_cache(gen, B, kv_heads, capacity, head_dim, lens, dtype, pad_fill)
    return ChunkInputs(q_chunk=q, k_cache=k, v_cache=v,
                       prefix_lens=torch.tensor(prefix_lens, dtype=torch.int32),
                       chunk_lens=torch.tensor(chunk_lens, dtype=torch.int32), name=name)


@dataclass
class PagedCache:
    k_pages: torch.Tensor      # [num_pages, Hkv, page_size, D]
    v_pages: torch.Tensor
    block_table: torch.Tensor  # int32 [B, pages_per_seq]; -1 past each sequence's last page


def make_paged(k_cache: torch.Tensor, v_cache: torch.Tensor, cache_lens: List[int],
               page_size: int, seed: int, spare_pages: int = 3,
               pad_fill: float = float("nan"), shuffle: bool = True) -> PagedCache:
    """Scatter a contiguous cache [B, Hkv, S_cap, D] into pages at seeded, shuffled physical
    positions (`shuffle=False`: in order, sequence after sequence, as a fresh allocator hands them
    out). Every sequence gets ceil(S_cap / page_size) table entries; the pages holding its first
    ceil(len / page_size) * page_size keys are copied, later entries are -1, and the unused
    physical pages (plus `spare_pages` extra ones) hold `pad_fill`."""
    B, hkv, cap, d = k_cache.shape
    pps = max(1, -(-cap // page_size))
    used = [-(-max(0, min(int(n), cap)) // page_size) for n in cache_lens]
    npages = sum(used) + spare_pages
    phys = (np.random.default_rng(seed).permutation(max(1, npages)) if shuffle
            else np.arange(max(1, npages)))
    kp = torch.full((max(1, npages), hkv, page_size, d), pad_fill, dtype=k_cache.dtype)
    vp = torch.full((max(1, npages), hkv, page_size, d), pad_fill, dtype=v_cache.dtype)
    table = torch.full((B, pps), -1, dtype=torch.int32)
    i = 0
    for b in range(B):
        for j in range(used[b]):
            pg = int(phys[i])
            i += 1
            table[b, j] = pg
            rows = min(page_size, cap - j * page_size)
            kp[pg, :, :rows] = k_cache[b, :, j * page_size:j * page_size + rows]
            vp[pg, :, :rows] = v_cache[b, :, j * page_size:j * page_size + rows]
    return PagedCache(k_pages=kp, v_pages=vp, block_table=table)


@dataclass
class Fp8Cache:
    k_codes: torch.Tensor      # uint8 E4M3 codes, the cache's shape
    v_codes: torch.Tensor
    k_scale: float             # the cached value of code c is e4m3(c) * scale
    v_scale: float


def _finite_amax(x: torch.Tensor) -> float:
    m = 0.0
    for i in range(x.shape[0]):   # one leading slice at a time (the caches are GBs)
        xi = x[i].float()
        xi = torch.where(torch.isfinite(xi), xi.abs(), torch.zeros((), dtype=torch.float32))
        m = max(m, float(xi.max()) if xi.numel() else 0.0)
    return m


def quantize_e4m3(x: torch.Tensor, scale: float) -> torch.Tensor:
    """uint8 E4M3 codes of x / scale: torch's round-to-nearest cast, after clamping to the
    largest finite code (448); NaN stays NaN. Done one leading slice at a time."""
    out = torch.empty(x.shape, dtype=torch.uint8)
    for i in range(x.shape[0]):
        y = torch.clamp(x[i].float() / scale, -448.0, 448.0)
        out[i] = y.to(torch.float8_e4m3fn).view(torch.uint8)
    return out


def make_fp8(k_cache: torch.Tensor, v_cache: torch.Tensor,
             k_scale: Optional[float] = None, v_scale: Optional[float] = None) -> Fp8Cache:
    """E4M3 copy of a cache (or page pool) with one scale per tensor (default: amax / 448 as a
    float32 number)."""
    ks = k_scale if k_scale is not None else float(np.float32(max(_finite_amax(k_cache), 1e-30) / 448.0))
    vs = v_scale if v_scale is not None else float(np.float32(max(_finite_amax(v_cache), 1e-30) / 448.0))
    return Fp8Cache(k_codes=quantize_e4m3(k_cache, ks), v_codes=quantize_e4m3(v_cache, vs),
                    k_scale=ks, v_scale=vs)


# ---- the five named workloads --------------------------------------------------------------

WORKLOADS = {
    1: "decode_mha_fp32_b1_h8_d64_len1024_splits4",
    2: "decode_mha_bf16_b4_h40_d128_len16384",
    3: "decode_gqa_bf16_b32_hq64_hkv8_d128_lenU1024-32768",
    4: "longctx_gqa_bf16_hq64_hkv8_d128_len32768_peaked",
    5: "mixed_chunk512_prefix15872_plus31decode_h32_d128",
    6: "verify4_gqa_bf16_b32_hq64_hkv8_d128_lenU1024-32768",
}


def workload(index: int, batch: Optional[int] = None, pad_fill: float = 0.0):
    """Build one of the six named workloads (index 1..6) at its full size."""
    seed = 1000 + index
    lseed = 1100 + index
    if index == 1:
        return make_decode_inputs(1, 8, 8, 64, 1024, [1024], torch.float32, seed,
                                  num_splits=4, pad_fill=pad_fill, name=WORKLOADS[1])
    if index == 2:
        return make_decode_inputs(4, 40, 40, 128, 16384, [16384] * 4, torch.bfloat16, seed,
                                  pad_fill=pad_fill, name=WORKLOADS[2])
    if index == 3:
        lens = uniform_lens(lseed, 32, 1024, 32768)
        b = 32 if batch is None else int(batch)   # a smaller batch keeps the first b sequences
        name = WORKLOADS[3] if b == 32 else f"{WORKLOADS[3]}_first{b}"
        return make_decode_inputs(b, 64, 8, 128, 32768, lens[:b], torch.bfloat16, seed,
                                  pad_fill=pad_fill, name=name)
    if index == 4:
        b = 1 if batch is None else int(batch)
        return make_decode_inputs(b, 64, 8, 128, 32768, [32768] * b, torch.bfloat16,
                                  seed, peaked_rows=8, peak_scale=8.0,
                                  pad_fill=pad_fill, name=f"{WORKLOADS[4]}_b{b}")
    if index == 5:
        dec = uniform_lens(lseed, 31, 512, 8192)
        prefix = [15872] + [n - 1 for n in dec]
        chunk = [512] + [1] * 31
        b = 32 if batch is None else int(batch)   # a smaller batch keeps the first b requests
        name = WORKLOADS[5] if b == 32 else f"{WORKLOADS[5]}_first{b}"
        return make_chunk_inputs(prefix[:b], chunk[:b], 32, 32, 128, 16384, torch.bfloat16,
                                 seed, pad_fill=pad_fill, name=name)
    if index == 6:
        # multi-token verification: every sequence of the 70B-like decode batch checks 4
        # speculative tokens, appended to its cache (prefix + 4 = a length of workload 3's draw)
        lens = uniform_lens(1100 + 3, 32, 1024, 32768)
        b = 32 if batch is None else int(batch)
        name = WORKLOADS[6] if b == 32 else f"{WORKLOADS[6]}_first{b}"
        return make_chunk_inputs([n - 4 for n in lens[:b]], [4] * b, 64, 8, 128, 32768,
                                 torch.bfloat16, seed, pad_fill=pad_fill, name=name)
    raise ValueError(f"unknown workload {index}")


def to_numpy_exact(t: torch.Tensor) -> np.ndarray:
    """CPU numpy view of a tensor with no value change: bf16 becomes its uint16 bit pattern."""
    t = t.detach().cpu().contiguous()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.numpy()
