"""Plain float64 CPU oracle for decode attention and chunked-prefill attention.

TEST INFRASTRUCTURE ONLY. Nothing on the product path imports this module: only the
tests, ``__graft_entry__.smoke()`` and ``bench.py`` (its CPU-baseline leg and its
``--impl reference`` arm) may call it. It shares no code with the CUDA library.

Sources (web pages, cited by title and section):

* "大语言模型长序列推理优化：ChunkedPrefill与FlashDecoding技术解析"
  (LLM long-sequence inference: ChunkedPrefill and FlashDecoding), below "ChunkedPrefill page".
  §2.1 gives chunk attention: scores = q·Kᵀ/√d_head over the cache with the chunk's own
  K/V appended first, under a causal mask. §3.1 gives decode attention as a
  softmax-weighted sum of V rows computed block by block with an online softmax.
* "大模型推理加速FlashDecoding算法原理与多GPU并行解码实战"
  (FlashDecoding algorithm and multi-GPU decoding), below "FlashDecoding page".
  Section "FlashDecoding算法原理与标准注意力机制对比" fixes the shapes
  Q [batch, heads, 1, head_dim], K/V [batch, heads, seq_len, head_dim] and the scaled
  score q·kᵀ/√head_dim; section "多GPU张量并行扩展下的FlashDecoding实现" masks keys at
  positions >= cache_lens; section "部署落地的工程细节" item 3 maps the query heads of a
  GQA group onto one KV head.

What is computed (the plain definition; FlashDecoding reaches exactly this result up to
rounding, so the oracle is the definition itself with no splitting):

    for each batch row b and query head h, with kv = h // G (G = Hq / Hkv), n = len_b:
        s_j  = (q_h · k_j) * scale            j < n,   scale = 1/sqrt(D) by default
        M    = max_j s_j
        O    = sum_j exp(s_j - M) v_j / sum_j exp(s_j - M)
        LSE  = M + ln sum_j exp(s_j - M)              (natural log of the scaled scores)

Readings where the pages are silent:

* n = 0 gives O = 0 and LSE = -inf.
* A cache length outside [0, S_cap] is clamped into that range (the CUDA side clamps too
  and raises a status flag).
* A chunk row i of request b sees keys j <= prefix_len_b + i (bottom-right causal
  alignment: the chunk's K/V already sit in the cache at [prefix, prefix + chunk_len)).

Inputs are numpy arrays: float32 / float64 values, or uint16 arrays holding the raw bits of
bf16 values. Every value is widened exactly to float64 before any arithmetic.
"""

from __future__ import annotations

import math
from typing import Iterable, Optional, Sequence, Tuple

import numpy as np

__all__ = [
    "widen",
    "decode_attention",
    "chunk_prefill_attention",
    "attention_rows",
    "gather_pages",
    "decode_attention_paged",
    "e4m3_value",
    "dequant_e4m3",
    "DequantView",
    "decode_attention_fp8",
    "decode_attention_paged_fp8",
]


def widen(x: np.ndarray) -> np.ndarray:
    """Exact float64 copy of ``x``.

    uint16 arrays are bf16 bit patterns: a bf16 number is the upper 16 bits of an IEEE
    binary32, so shifting the bits up by 16 gives the binary32 with the same value, and
    binary32 -> binary64 is exact.
    """
    x = np.asarray(x)
    if x.dtype == np.uint16:
        return (x.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)
    if x.dtype in (np.float32, np.float64):
        return x.astype(np.float64)
    raise TypeError(f"oracle: unsupported input dtype {x.dtype}")


def attention_rows(q_rows: np.ndarray, keys: np.ndarray, values: np.ndarray,
                   n_visible: Sequence[int], scale: float) -> Tuple[np.ndarray, np.ndarray]:
    """Softmax attention of several query rows over a prefix of one key/value sequence.

    q_rows [R, D] float64, keys/values [N, D] float64, n_visible[r] = number of leading keys
    row r may see. Returns (O [R, D], LSE [R]) in float64.

    The definition in the matrix form of the ChunkedPrefill page §2.1 (scores = Q·Kᵀ/√d, then a
    mask, a softmax per row and the product with V): the score matrix of all rows at once, each
    row keeping its first n_visible[r] scores; then per row the max, the exponentials, the
    normalised weighted sum of V rows and the log-sum-exp. A row with no visible key keeps
    O = 0 and LSE = -inf.
    """
    R, D = q_rows.shape
    out = np.zeros((R, D), dtype=np.float64)
    lse = np.full((R,), -np.inf, dtype=np.float64)
    n_vis = np.asarray(n_visible, dtype=np.int64).reshape(R)
    N = int(n_vis.max()) if R else 0
    if N <= 0:
        return out, lse
    s = (q_rows @ keys[:N].T) * scale                    # s[r, j] = q_r·k_j * scale
    s[np.arange(N)[None, :] >= n_vis[:, None]] = -np.inf  # keys past row r's limit: excluded
    has = n_vis > 0
    m = s[has].max(axis=1)                               # M_r = max_j s[r, j]
    e = np.exp(s[has] - m[:, None])                      # exp(s_j - M_r); 0 where excluded
    z = e.sum(axis=1)                                    # sum_j exp(s_j - M_r)
    out[has] = (e @ values[:N]) / z[:, None]             # sum_j exp(s_j - M_r) v_j / z_r
    lse[has] = m + np.log(z)                             # M_r + ln z_r
    return out, lse


def _clamp_len(n: int, cap: int) -> int:
    return max(0, min(int(n), int(cap)))


def decode_attention(q: np.ndarray, k_cache: np.ndarray, v_cache: np.ndarray,
                     cache_lens: Sequence[int], scale: Optional[float] = None,
                     rows: Optional[Iterable[Tuple[int, int]]] = None
                     ) -> Tuple[np.ndarray, np.ndarray]:
    """Decode attention (one query token per sequence) against a contiguous KV cache.

    q [B, Hq, D]; k_cache, v_cache [B, Hkv, S_cap, D]; cache_lens [B].
    Returns out [B, Hq, D] and lse [B, Hq], both float64. With ``rows`` (an iterable of
    (b, h) pairs) only those outputs are computed; the rest are NaN.

    Source: FlashDecoding page, section "FlashDecoding算法原理与标准注意力机制对比" (shapes,
    scaled scores) and section "多GPU张量并行扩展下的FlashDecoding实现" (keys at positions
    >= cache_lens are masked); GQA head mapping from section "部署落地的工程细节" item 3.
    """
    B, Hq, D = q.shape
    Bk, Hkv, S_cap, Dk = k_cache.shape
    if Bk != B or Dk != D or v_cache.shape != k_cache.shape:
        raise ValueError("oracle: shape mismatch")
    if Hq % Hkv != 0:
        raise ValueError("oracle: Hq must be a multiple of Hkv")
    G = Hq // Hkv
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    out = np.full((B, Hq, D), np.nan, dtype=np.float64)
    lse = np.full((B, Hq), np.nan, dtype=np.float64)
    if rows is None:
        rows = [(b, h) for b in range(B) for h in range(Hq)]
    # Group the requested rows by (b, kv head) so each key/value slab is widened once.
    groups = {}
    for b, h in rows:
        groups.setdefault((int(b), int(h) // G), []).append(int(h))
    for (b, kv), heads in sorted(groups.items()):
        n = _clamp_len(cache_lens[b], S_cap)
        keys = widen(k_cache[b, kv, :n])
        values = widen(v_cache[b, kv, :n])
        qr = widen(q[b, heads])
        o, l = attention_rows(qr, keys, values, [n] * len(heads), scale)
        out[b, heads] = o
        lse[b, heads] = l
    return out, lse


def chunk_prefill_attention(q_chunk: np.ndarray, k_cache: np.ndarray, v_cache: np.ndarray,
                            prefix_lens: Sequence[int], chunk_lens: Sequence[int],
                            scale: Optional[float] = None,
                            rows: Optional[Iterable[Tuple[int, int]]] = None
                            ) -> Tuple[np.ndarray, np.ndarray]:
    """Causal attention of packed query chunks against their cached prefix plus themselves.

    q_chunk [sum(chunk_lens), Hq, D], packed request by request; k_cache, v_cache
    [B, Hkv, S_cap, D] already hold each request's prefix and its chunk at
    [prefix_len_b, prefix_len_b + chunk_len_b). Row i of request b sees keys
    j <= prefix_len_b + i. Returns out [sum(chunk_lens), Hq, D] and lse [sum(chunk_lens), Hq].
    ``rows`` selects (packed row, h) pairs; the rest are NaN.

    Source: ChunkedPrefill page §2.1 (the chunk's K/V are appended to the cache, then
    scores against the whole cache under a causal mask) and its list of three requirements
    (persist each chunk's KV; a token sees only itself and earlier tokens); prefix reuse from
    "Chunked-Prefills分块预填充机制：破解大模型推理的吞吐与延迟困局" §三.2 (KV cache reuse).
    A request with chunk_len = 1 and prefix_len = len - 1 is plain decode over len keys.
    """
    total, Hq, D = q_chunk.shape
    B, Hkv, S_cap, Dk = k_cache.shape
    if Dk != D or v_cache.shape != k_cache.shape:
        raise ValueError("oracle: shape mismatch")
    if len(prefix_lens) != B or len(chunk_lens) != B:
        raise ValueError("oracle: prefix_lens / chunk_lens must have one entry per request")
    if int(sum(int(c) for c in chunk_lens)) != total:
        raise ValueError("oracle: q_chunk rows must equal sum(chunk_lens)")
    if Hq % Hkv != 0:
        raise ValueError("oracle: Hq must be a multiple of Hkv")
    G = Hq // Hkv
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    row_req = np.zeros(total, dtype=np.int64)
    row_pos = np.zeros(total, dtype=np.int64)
    off = 0
    for b in range(B):
        c = int(chunk_lens[b])
        row_req[off:off + c] = b
        row_pos[off:off + c] = np.arange(c)
        off += c
    out = np.full((total, Hq, D), np.nan, dtype=np.float64)
    lse = np.full((total, Hq), np.nan, dtype=np.float64)
    if rows is None:
        rows = [(p, h) for p in range(total) for h in range(Hq)]
    groups = {}
    for p, h in rows:
        p = int(p)
        groups.setdefault((int(row_req[p]), int(h) // G), []).append((p, int(h)))
    for (b, kv), items in sorted(groups.items()):
        limit = _clamp_len(int(prefix_lens[b]) + int(chunk_lens[b]), S_cap)
        keys = widen(k_cache[b, kv, :limit])
        values = widen(v_cache[b, kv, :limit])
        qr = np.stack([widen(q_chunk[p, h]) for p, h in items])
        # row i of the chunk sees prefix_len + i + 1 keys, clamped to the cache capacity
        n_vis = [_clamp_len(int(prefix_lens[b]) + int(row_pos[p]) + 1, S_cap) for p, _ in items]
        o, l = attention_rows(qr, keys, values, n_vis, scale)
        for r, (p, h) in enumerate(items):
            out[p, h] = o[r]
            lse[p, h] = l[r]
    return out, lse


def gather_pages(pages: np.ndarray, block_table: Sequence[Sequence[int]], lens: Sequence[int],
                 capacity: int) -> np.ndarray:
    """Contiguous cache [B, Hkv, capacity, D] from a paged one.

    pages [num_pages, Hkv, page_size, D]; token t of sequence b lives in page
    block_table[b][t // page_size] at row t % page_size. Rows at or past len_b are left zero (the
    attention below never reads them). This is the meaning of a block table in the paged-cache
    row of the hot path (the FlashDecoding page, "部署落地的工程细节", pairs FlashDecoding with a
    paged KV cache); the gather is the whole definition.
    """
    npg, hkv, psz, d = pages.shape
    B = len(lens)
    out = np.zeros((B, hkv, capacity, d), dtype=pages.dtype)
    for b in range(B):
        n = max(0, min(int(lens[b]), capacity))
        for t0 in range(0, n, psz):
            pg = int(block_table[b][t0 // psz])
            m = min(psz, n - t0)
            out[b, :, t0:t0 + m] = pages[pg, :, :m]
    return out


def decode_attention_paged(q: np.ndarray, k_pages: np.ndarray, v_pages: np.ndarray,
                           block_table: Sequence[Sequence[int]], cache_lens: Sequence[int],
                           scale: Optional[float] = None,
                           rows: Optional[Iterable[Tuple[int, int]]] = None
                           ) -> Tuple[np.ndarray, np.ndarray]:
    """Decode attention over a paged cache: the pages gathered into a contiguous cache, then
    ``decode_attention`` (the plain definition) over it."""
    psz = k_pages.shape[2]
    # a sequence holds at most (entries of its block-table row) * page_size keys; longer lengths
    # are clamped to that, as a contiguous cache clamps them to its capacity
    cap = max(1, len(block_table[0]) if len(block_table) else 1) * psz
    kc = gather_pages(k_pages, block_table, cache_lens, cap)
    vc = gather_pages(v_pages, block_table, cache_lens, cap)
    return decode_attention(q, kc, vc, cache_lens, scale=scale, rows=rows)


# ------------------------------------------------------------------------- FP8 KV cache ---
#
# The FlashDecoding page, section "与其他推理加速方案的组合使用" (combining FlashDecoding with
# other speed-ups), item "Quantization + FlashDecoding", pairs the method with an INT8/FP8 KV
# cache and has the scores computed on values dequantized to bf16. It names neither the FP8
# format nor the scale granularity. The reading taken here: the cache holds OCP E4M3 codes
# (4 exponent bits with bias 7, 3 mantissa bits, no infinities, S.1111.111 is NaN), with one
# scale for all of K and one for all of V; the cached value of a code c is e4m3(c) * scale.
# Every E4M3 value has at most 4 significant bits and an exponent inside bf16's range, so
# "dequantize to bf16" loses nothing, and the definition below is the plain attention over the
# exact values e4m3(c) * scale.


def e4m3_value(code: int) -> float:
    """Value of one E4M3 code (an integer 0..255), from the format's definition.

    sign s = bit 7, exponent field e = bits 6..3, mantissa field m = bits 2..0:
      e = 15 and m = 7   -> NaN
      e = 0              -> (-1)^s * (m / 8) * 2^(1 - 7)      (subnormal)
      otherwise          -> (-1)^s * (1 + m / 8) * 2^(e - 7)
    """
    code = int(code)
    if not 0 <= code <= 255:
        raise ValueError("oracle: an E4M3 code is one byte")
    s = -1.0 if code & 0x80 else 1.0
    e = (code >> 3) & 0xF
    m = code & 0x7
    if e == 15 and m == 7:
        return math.nan
    if e == 0:
        return s * (m / 8.0) * 2.0 ** (1 - 7)
    return s * (1.0 + m / 8.0) * 2.0 ** (e - 7)


_E4M3_TABLE = np.array([e4m3_value(c) for c in range(256)], dtype=np.float64)


def dequant_e4m3(codes: np.ndarray, scale: float) -> np.ndarray:
    """float64 values e4m3(code) * scale of a uint8 array of E4M3 codes."""
    codes = np.asarray(codes)
    if codes.dtype != np.uint8:
        raise TypeError(f"oracle: E4M3 codes must be uint8, got {codes.dtype}")
    return _E4M3_TABLE[codes] * float(scale)


class DequantView:
    """Read-only view of an array of E4M3 codes as the float64 values e4m3(c) * scale. Indexing
    it dequantizes only the selected elements, so the definition below reads a large cache one
    (sequence, KV head) slab at a time, as it reads a bf16 one."""

    def __init__(self, codes: np.ndarray, scale: float):
        self.codes = np.asarray(codes)
        if self.codes.dtype != np.uint8:
            raise TypeError(f"oracle: E4M3 codes must be uint8, got {self.codes.dtype}")
        self.scale = float(scale)
        self.shape = self.codes.shape
        self.dtype = np.dtype(np.float64)

    def __getitem__(self, idx):
        return dequant_e4m3(self.codes[idx], self.scale)


def decode_attention_fp8(q: np.ndarray, k_codes: np.ndarray, v_codes: np.ndarray,
                         k_scale: float, v_scale: float, cache_lens: Sequence[int],
                         scale: Optional[float] = None,
                         rows: Optional[Iterable[Tuple[int, int]]] = None
                         ) -> Tuple[np.ndarray, np.ndarray]:
    """Decode attention over an E4M3 cache: ``decode_attention`` (the plain definition) over the
    dequantized values, K with k_scale and V with v_scale."""
    kc = DequantView(k_codes, k_scale)
    vc = DequantView(v_codes, v_scale)
    return decode_attention(q, kc, vc, cache_lens, scale=scale, rows=rows)


def decode_attention_paged_fp8(q: np.ndarray, k_pages: np.ndarray, v_pages: np.ndarray,
                               k_scale: float, v_scale: float,
                               block_table: Sequence[Sequence[int]], cache_lens: Sequence[int],
                               scale: Optional[float] = None,
                               rows: Optional[Iterable[Tuple[int, int]]] = None
                               ) -> Tuple[np.ndarray, np.ndarray]:
    """Paged E4M3 cache: ``decode_attention_paged`` over the dequantized pages."""
    kp = DequantView(k_pages, k_scale)
    vp = DequantView(v_pages, v_scale)
    return decode_attention_paged(q, kp, vp, block_table, cache_lens, scale=scale, rows=rows)
