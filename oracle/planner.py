"""Plain-Python split planner oracle.

TEST INFRASTRUCTURE ONLY (see ``oracle/attention.py``). The CUDA library plans its split-KV
work on the host (``fd_split_plan``) and on the device; the tests require both to equal this
plan exactly, integer for integer.

Source: "大模型推理加速FlashDecoding算法原理与多GPU并行解码实战" (FlashDecoding algorithm and
multi-GPU decoding), section "Variable-Length序列动态切分策略": a greedy allocator fills
workers up to target = ceil(total tokens / workers) with pieces of at most max_chunk = 1024
tokens, never leaves a piece under min_chunk = 128 on its own, and exists so that short
sequences do not leave workers idle. Section "性能压测与瓶颈分析" adds that pieces under about
256 tokens lose to launch overhead. The ChunkedPrefill page ("大语言模型长序列推理优化：
ChunkedPrefill与FlashDecoding技术解析", §3.1) gives the tile range 256-1024 tokens, and the
Chunked-Prefills page ("Chunked-Prefills分块预填充机制：破解大模型推理的吞吐与延迟困局",
§四.1) gives the rule chunk_size = min(MAX_CHUNK_SIZE, input_length / NUM_CHUNKS).

Reading used on one GPU (the workers are the persistent CTAs, one per SM):

1. total = sum of the clamped cache lengths.
2. For each target of W = 8, 4, 2, 1 waves of items over the CTAs,
   chunk_W = clamp(ceil(total * Hkv / (W * num_ctas)), 256, 1024) tokens and
   items_W = Hkv * sum_b max(1, ceil(len_b / chunk_W)). The chunk is the chunk_W of least
   estimated makespan ceil(items_W / num_ctas) * (ceil(chunk_W / 128) + 2), ties to the larger W
   (2 = the fixed cost of a work item in 128-key tiles; the pages' allocator fills every worker
   once, which W = 1 is, and its ~256-token floor keeps pieces from getting too small for their
   overhead, which the cost term weighs).
3. n_b = max(1, ceil(len_b / chunk)) splits for sequence b.
4. Split s of sequence b is [floor(s * len_b / n_b), floor((s + 1) * len_b / n_b)): the offset
   restarts at 0 for every sequence and no token is dropped (the printed allocator never
   resets its offset between sequences and drops tokens once the workers run out).
5. With equal splits every split of a multi-split sequence has more than chunk / 2 >= 128
   tokens, so the printed "merge a piece under min_chunk into the previous one" rule never
   fires; the tests check that bound.
6. Items are ordered longest first (LPT list scheduling over the persistent CTAs): sequences
   by their longest split, descending, ties by index; within a sequence by KV head, then split.

A fixed split count (num_splits > 0) instead gives every sequence num_splits splits of
chunk_b = ceil(len_b / num_splits) tokens, split s = [min(s * chunk_b, len_b),
min((s + 1) * chunk_b, len_b)) (the FlashDecoding page's chunk_size rule); trailing splits
may be empty.

Aligned plans (``align`` = A > 1, used for a paged cache so that no key tile of A keys crosses a
page) put every split boundary on a multiple of A keys and change nothing else: with
U_b = ceil(len_b / A) units, planner split s = [min(len_b, A floor(s U_b / n_b)),
min(len_b, A floor((s + 1) U_b / n_b))), and a fixed count uses chunk_b rounded up to a multiple
of A. With A = 1 both rules are the ones above.

Chunked prefill (``chunk_plan``): a request with chunk_len = 1 is a decode row over
prefix_len + 1 keys and is planned as above (over the decode requests only). A request with a
longer chunk is cut into query tiles of 128 rows; tile t sees at most
K_t = min(prefix + min(chunk_len, 128 (t + 1)), S_cap) keys, cut on a fixed grid of
CHUNK_KV_SPLIT keys: split s = [CHUNK_KV_SPLIT s, min(CHUNK_KV_SPLIT (s + 1), K_t)) for
s < n_t = max(1, ceil(K_t / CHUNK_KV_SPLIT)). The grid is the same for every tile of a request, so
the tiles of one head read the same K/V ranges. Every row of a tile owns n_t partial slots. Tile
items run in the order (request, query head, split, tile): the tiles sharing a split's keys are
adjacent, so they run at the same time and share those keys in L2. A request with
2 <= chunk_len <= 128 / G rows and G = Hq / Hkv >= 2 (a multi-token verification step, say) is
served by head-packed tiles instead: one tile per (KV head, split) holds its rows for all G query
heads (tile row r = chunk position r // G of query head h G + r mod G), so the head index of its
items is a KV head; it has a single query tile (t = 0) and the same splits and slots.
"""

from __future__ import annotations

from dataclasses import dataclass, field
from typing import List, Sequence, Tuple

__all__ = [
    "MIN_CHUNK", "MAX_CHUNK", "WAVES", "Q_TILE", "CHUNK_KV_SPLIT",
    "DecodePlan", "decode_plan", "choose_chunk", "ChunkPlan", "chunk_plan",
]

MIN_CHUNK = 256        # launch-overhead floor, FlashDecoding page "性能压测与瓶颈分析"
MAX_CHUNK = 1024       # max_chunk of the allocator / top of the 256-1024 tile range
MIN_PIECE = 128        # min_chunk of the allocator
WAVES = 8              # largest target of items per persistent CTA
WAVE_CHOICES = (8, 4, 2, 1)
ITEM_FIXED_TILES = 2   # fixed cost of a work item, in 128-key tiles
Q_TILE = 128           # query rows per chunked-prefill tile
CHUNK_KV_SPLIT = 4096  # keys per split for a chunked-prefill query tile


def _cdiv(a: int, b: int) -> int:
    return -(-a // b)


@dataclass
class DecodePlan:
    chunk_tokens: int
    splits_per_seq: List[int]
    # (b, kv_head, split, start, end) in execution order
    items: List[Tuple[int, int, int, int, int]] = field(default_factory=list)

    @property
    def total_items(self) -> int:
        return len(self.items)

    @property
    def max_splits_per_seq(self) -> int:
        return max(self.splits_per_seq) if self.splits_per_seq else 0


def _split_bounds_equal(n_tok: int, n_split: int, align: int = 1) -> List[Tuple[int, int]]:
    units = _cdiv(n_tok, align)
    return [(min(n_tok, align * ((s * units) // n_split)),
             min(n_tok, align * (((s + 1) * units) // n_split))) for s in range(n_split)]


def _split_bounds_fixed(n_tok: int, n_split: int, align: int = 1) -> List[Tuple[int, int]]:
    c = _cdiv(n_tok, n_split) if n_tok > 0 else 0
    c = align * _cdiv(c, align)
    return [(min(s * c, n_tok), min((s + 1) * c, n_tok)) for s in range(n_split)]


def choose_chunk(lens: Sequence[int], num_kv_heads: int, num_ctas: int) -> int:
    """Step 2 of the module docstring: the chunk of the least estimated makespan."""
    total = sum(lens)
    n = max(1, num_ctas)
    best = None
    for waves in WAVE_CHOICES:
        chunk = max(MIN_CHUNK, min(MAX_CHUNK, _cdiv(total * num_kv_heads, waves * n)))
        items = num_kv_heads * sum(max(1, _cdiv(x, chunk)) for x in lens)
        cost = _cdiv(items, n) * (_cdiv(chunk, 128) + ITEM_FIXED_TILES)
        if best is None or cost < best[0]:
            best = (cost, chunk)
    return best[1]


def decode_plan(cache_lens: Sequence[int], num_kv_heads: int, cache_capacity: int,
                num_ctas: int, num_splits: int = 0, align: int = 1) -> DecodePlan:
    """Plan the split-KV work of one decode call (see the module docstring)."""
    lens = [max(0, min(int(x), int(cache_capacity))) for x in cache_lens]
    B = len(lens)
    if num_splits > 0:
        bounds = [_split_bounds_fixed(n, num_splits, align) for n in lens]
        chunk = 0
        keys = [_cdiv(n, num_splits) for n in lens]
    else:
        chunk = choose_chunk(lens, num_kv_heads, num_ctas)
        counts = [max(1, _cdiv(n, chunk)) for n in lens]
        bounds = [_split_bounds_equal(n, c, align) for n, c in zip(lens, counts)]
        keys = [_cdiv(n, c) for n, c in zip(lens, counts)]
    order = sorted(range(B), key=lambda b: (-keys[b], b))
    items = []
    for b in order:
        for h in range(num_kv_heads):
            for s, (t0, t1) in enumerate(bounds[b]):
                items.append((b, h, s, t0, t1))
    return DecodePlan(chunk_tokens=chunk, splits_per_seq=[len(x) for x in bounds], items=items)


@dataclass
class ChunkPlan:
    decode: DecodePlan                     # plan over the chunk_len == 1 requests (indexed by request)
    decode_requests: List[int]             # request index of each decode row, in request order
    # (b, q_tile, q_head, split, key_start, key_end) in execution order; for a head-packed
    # request the head is a KV head
    tile_items: List[Tuple[int, int, int, int, int, int]] = field(default_factory=list)
    row_splits: List[int] = field(default_factory=list)      # partial slots per packed row
    head_packed: List[int] = field(default_factory=list)     # requests served by head-packed tiles


def chunk_plan(prefix_lens: Sequence[int], chunk_lens: Sequence[int], num_q_heads: int,
               num_kv_heads: int, cache_capacity: int, num_ctas: int) -> ChunkPlan:
    """Plan a chunked-prefill call: decode rows via ``decode_plan``, longer chunks by tiles."""
    B = len(chunk_lens)
    dec_req = [b for b in range(B) if int(chunk_lens[b]) == 1]
    dec_lens = [int(prefix_lens[b]) + 1 for b in dec_req]
    dec = decode_plan(dec_lens, num_kv_heads, cache_capacity, num_ctas, 0)
    # express decode items by request index
    dec.items = [(dec_req[i], h, s, t0, t1) for (i, h, s, t0, t1) in dec.items]
    row_splits: List[int] = []
    tiles = []
    packed: List[int] = []
    G = num_q_heads // num_kv_heads
    for b in range(B):
        c = int(chunk_lens[b])
        if c == 1:
            row_splits.append(dec.splits_per_seq[dec_req.index(b)])
            continue
        if c <= 0:
            continue  # an empty chunk has no rows and no items
        p = int(prefix_lens[b])
        n_tiles = _cdiv(c, Q_TILE)
        k_t = [max(0, min(p + min(c, Q_TILE * (t + 1)), int(cache_capacity))) for t in range(n_tiles)]
        n_t = [max(1, _cdiv(k, CHUNK_KV_SPLIT)) for k in k_t]
        for t in range(n_tiles):
            row_splits.extend([n_t[t]] * min(Q_TILE, c - Q_TILE * t))
        head_packed = G >= 2 and 2 <= c and c * G <= Q_TILE
        if head_packed:
            packed.append(b)
        for h in range(num_kv_heads if head_packed else num_q_heads):
            for s in range(max(n_t)):
                for t in range(n_tiles):
                    if s < n_t[t]:
                        k0 = min(CHUNK_KV_SPLIT * s, k_t[t])
                        k1 = min(CHUNK_KV_SPLIT * (s + 1), k_t[t])
                        tiles.append((b, t, h, s, k0, k1))
    return ChunkPlan(decode=dec, decode_requests=dec_req, tile_items=tiles, row_splits=row_splits,
                     head_packed=packed)
