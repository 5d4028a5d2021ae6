// Split planning shared by the host planner (fd_split_plan) and the device planner kernel, plus
// the work-item formats and the workspace layout the kernels read.
//
// Source: "大模型推理加速FlashDecoding算法原理与多GPU并行解码实战" (FlashDecoding algorithm and
// multi-GPU decoding), section "Variable-Length序列动态切分策略": a greedy allocator that fills
// each worker up to ceil(total tokens / workers) with pieces of at most max_chunk = 1024 tokens
// and never leaves a piece under min_chunk = 128 alone; section "性能压测与瓶颈分析": pieces
// under ~256 tokens lose to launch overhead. On one GPU the workers are persistent CTAs; the
// plan below gives every sequence equal splits sized so that about kWaves items exist per CTA,
// restarts the offset for every sequence and drops no token.
#pragma once

#include <stddef.h>
#include <stdint.h>

#include "../../include/fd.h"

#if defined(__CUDACC__)
#define FD_HD __host__ __device__ __forceinline__
#else
#define FD_HD inline
#endif

namespace fd {

constexpr int32_t kMinChunk = 256;        // launch-overhead floor ("性能压测与瓶颈分析")
constexpr int32_t kMaxChunk = 1024;       // allocator max_chunk / top of the 256-1024 tile range
constexpr int32_t kWaves = 8;             // target work items per persistent CTA
constexpr int32_t kQTile = 128;           // chunked-prefill query rows per tile
// Keys per split of a chunked-prefill query tile. Measured on B200: 4096 against 2048 takes the
// 4-token verification workload from 457 to 435 us per call (half the partial results to write
// and merge) and leaves the mixed 512-row chunk step unchanged; 6144 and 8192 slow the chunk
// step (fewer, longer tile items balance worse over the tile kernel's CTAs).
constexpr int32_t kChunkKvSplit = 4096;
constexpr int32_t kMaxPlanBatch = 4096;   // largest batch the device planners accept (shared memory per CTA)
constexpr int32_t kFusedPlanMaxBatch = 256;  // largest batch the tensor-core split kernel plans itself
constexpr int32_t kPagedKeyAlign = 128;      // split boundaries of a paged cache: one key tile
constexpr int32_t kTcKeyAlign = 128;         // split boundaries on the tensor-core decode path

// One split of one (sequence, KV head): keys [t0, t1) of cache row b, output row `row`.
struct DecodeItem {
  int32_t row;     // output row: b for decode, the packed query row for chunked prefill
  int32_t b;       // cache batch index
  int32_t h;       // KV head
  int32_t split;   // split index within the sequence
  int32_t t0, t1;  // key range
  int32_t nsplit;  // splits of this sequence (1: write the final output directly)
  int32_t slot;    // partial slot of this split; the slots of one (row, KV head) group are
                   // consecutive: row_base[row] * Hkv + h * nsplit + split
};
static_assert(sizeof(DecodeItem) == 32, "DecodeItem is 32 bytes");

// One key split of one 128-row query tile of one head of a chunked-prefill request.
struct TileItem {
  int32_t b, h, split, nsplit;
  int32_t k0, k1;    // key range of the split
  int32_t row0;      // packed query row of the tile's first row
  int32_t pos0;      // chunk position of the tile's first row
  int32_t rows;      // valid rows in the tile (<= kQTile)
  int32_t prefix;    // prefix length: row at chunk position i sees keys <= prefix + i
  int32_t slot0;     // partial slot of (row0, split 0); row r uses slot0 + r * nsplit + split
  int32_t head_packed;  // 1: head-packed tile (h is a KV head; tile row r is chunk position r / G of
                        // query head h * G + r % G); 0: one query head h, tile row = chunk position
  int32_t pad[4];
};
static_assert(sizeof(TileItem) == 64, "TileItem is 64 bytes");

// Header at the start of every workspace.
struct WsHeader {
  uint32_t status;          // FD_FLAG_* bits, sticky until fd_poll_status
  int32_t num_dec_items;    // decode items planned by the last call
  int32_t num_tile_items;   // tile items planned by the last call
  int32_t dec_counter;      // dynamic scheduler cursor: zero between calls (the planner zeroes
                            // it; the tensor-core split kernel's last CTA zeroes it on exit)
  int32_t tile_counter;
  int32_t dec_exit;         // CTAs of the tensor-core split kernel that have finished (zero
                            // between calls)
  int32_t tile_ctas;        // chunked prefill: CTAs the tile kernel keeps (least chunk_tile_cost)
  int32_t pad[57];
};
static_assert(sizeof(WsHeader) == 256, "WsHeader is 256 bytes");

FD_HD int64_t cdiv64(int64_t a, int64_t b) { return (a + b - 1) / b; }
// ceil(a / b) for 0 <= a < 2^31 and 0 < b < 2^31 in 32-bit unsigned arithmetic (a + b - 1 < 2^32),
// the same value as cdiv64 at a fraction of a 64-bit division's instructions
FD_HD int32_t cdiv32(int32_t a, int32_t b) {
  return static_cast<int32_t>((static_cast<uint32_t>(a) + static_cast<uint32_t>(b) - 1u) /
                              static_cast<uint32_t>(b));
}
FD_HD size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

FD_HD int32_t clamp_len(int64_t len, int32_t cap) {
  return len < 0 ? 0 : (len > cap ? cap : static_cast<int32_t>(len));
}

// The chunk (split size) comes from a target number of item waves W over the CTAs:
//   chunk_W = clamp(ceil(total * Hkv / (W * nctas)), kMinChunk, kMaxChunk).
// A small call (a few long sequences, say) under W = kWaves would be cut into items of one or two
// key tiles, whose fixed cost (start, Q load, partial result, merge) then outweighs their keys;
// so the planner weighs W = 8, 4, 2, 1 and keeps the chunk of least estimated makespan
//   ceil(items_W / nctas) * (ceil(chunk_W / 128) + kItemFixedTiles),
// items_W = Hkv * sum_b max(1, ceil(len_b / chunk_W)), ties to the larger W. Large calls, whose
// chunk is kMaxChunk for every W, keep the plan of W = kWaves.
constexpr int kPlanWaveChoices = 4;
constexpr int32_t kItemFixedTiles = 2;  // fixed cost of a work item, in 128-key tiles
FD_HD int32_t plan_waves(int i) { return kWaves >> i; }  // 8, 4, 2, 1

FD_HD int32_t plan_chunk_for_waves(int64_t total, int32_t hkv, int32_t nctas, int32_t waves) {
  int64_t c = cdiv64(total * hkv, static_cast<int64_t>(waves) * (nctas > 0 ? nctas : 1));
  if (c < kMinChunk) c = kMinChunk;
  if (c > kMaxChunk) c = kMaxChunk;
  return static_cast<int32_t>(c);
}

// The chunk of least estimated makespan among the candidates chunks[i] = plan_chunk_for_waves(...,
// plan_waves(i)), given split_sums[i] = sum_b max(1, ceil(len_b / chunks[i])).
// Estimated makespan of one candidate: ceil(items / nctas) * (ceil(chunk / 128) + kItemFixedTiles).
FD_HD int64_t plan_chunk_cost(int64_t split_sum, int32_t chunk, int32_t hkv, int32_t nctas) {
  const int64_t n = nctas > 0 ? nctas : 1;
  return cdiv64(split_sum * hkv, n) * (cdiv64(chunk, 128) + kItemFixedTiles);
}

FD_HD int32_t plan_pick_chunk(const int32_t* chunks, const int64_t* split_sums, int32_t hkv,
                              int32_t nctas) {
  int32_t best = chunks[0];
  int64_t best_cost = 0;
  for (int i = 0; i < kPlanWaveChoices; ++i) {
    const int64_t cost = plan_chunk_cost(split_sums[i], chunks[i], hkv, nctas);
    if (i == 0 || cost < best_cost) {
      best = chunks[i];
      best_cost = cost;
    }
  }
  return best;
}

// Splits of a sequence: the fixed count, else max(1, ceil(len / chunk)).
FD_HD int32_t plan_num_splits(int32_t len, int32_t chunk, int32_t fixed) {
  if (fixed > 0) return fixed;
  int32_t n = len > 0 ? cdiv32(len, chunk) : 0;
  return n < 1 ? 1 : n;
}

// Key range of split s. Fixed mode: [min(s*c, len), min((s+1)*c, len)) with c = ceil(len/n)
// (the FlashDecoding page's chunk_size rule); planner mode: equal splits
// [floor(s*len/n), floor((s+1)*len/n)). With align = A > 1 (a paged cache, so that no key tile
// crosses a page) every boundary sits on a multiple of A keys: planner mode cuts the
// U = ceil(len/A) units equally, [min(len, A*floor(s*U/n)), min(len, A*floor((s+1)*U/n))), and
// fixed mode rounds c up to a multiple of A.
FD_HD void plan_split_range(int32_t len, int32_t n, int32_t s, int32_t fixed, int32_t align,
                            int32_t* t0, int32_t* t1) {
  if (fixed > 0) {
    int64_t c = cdiv64(len, n);
    if (align > 1) c = cdiv64(c, align) * align;
    int64_t a = s * c, e = (s + 1) * c;
    *t0 = static_cast<int32_t>(a < len ? a : len);
    *t1 = static_cast<int32_t>(e < len ? e : len);
  } else if (align > 1) {
    const int64_t units = cdiv64(len, align);
    const int64_t a = (static_cast<int64_t>(s) * units / n) * align;
    const int64_t e = (static_cast<int64_t>(s + 1) * units / n) * align;
    *t0 = static_cast<int32_t>(a < len ? a : len);
    *t1 = static_cast<int32_t>(e < len ? e : len);
  } else {
    const int64_t a = static_cast<int64_t>(s) * len, e = static_cast<int64_t>(s + 1) * len;
    if (e <= INT32_MAX) {  // 32-bit division when the products fit (the common case)
      *t0 = static_cast<int32_t>(a) / n;
      *t1 = static_cast<int32_t>(e) / n;
    } else {
      *t0 = static_cast<int32_t>(a / n);
      *t1 = static_cast<int32_t>(e / n);
    }
  }
}

// Longest-first ordering key of a sequence: its longest split.
FD_HD int32_t plan_sort_key(int32_t len, int32_t n) {
  return len > 0 ? cdiv32(len, n) : 0;
}

// Upper bound of the decode items of any plan of this shape (any lengths), used to size the
// workspace: sum_b n_b < B + max(kWaves * nctas / Hkv, B * S_cap / kMaxChunk).
FD_HD int64_t decode_max_items(int64_t B, int64_t hkv, int64_t cap, int32_t fixed,
                               int32_t nctas) {
  if (fixed > 0) return B * hkv * fixed;
  int64_t a = static_cast<int64_t>(kWaves) * (nctas > 0 ? nctas : 1);
  int64_t b = cdiv64(hkv * B * cap, kMaxChunk);
  return hkv * B + (a > b ? a : b);
}

// Chunked prefill: keys seen by query tile t of a chunk of c rows at prefix p (clamped to S_cap),
// and the number of kChunkKvSplit-key splits they are cut into.
FD_HD int32_t chunk_tile_keys(int32_t prefix, int32_t c, int32_t t, int32_t cap) {
  const int64_t last = static_cast<int64_t>(t + 1) * kQTile;
  const int64_t k = static_cast<int64_t>(prefix) + (last < c ? last : c);
  return k < 0 ? 0 : (k > cap ? cap : static_cast<int32_t>(k));
}
// A request of 2 <= c <= kQTile / G chunk rows with G >= 2 query heads per KV head (a
// multi-token verification step, say) is served by head-packed tiles: one 128-row tile holds its
// c rows for all G heads of a KV head, so every key tile is read and multiplied once per KV head
// rather than once per query head.
FD_HD bool chunk_packed(int32_t c, int32_t g) { return g >= 2 && c >= 2 && c * g <= kQTile; }
FD_HD int32_t chunk_tile_splits(int32_t keys) {
  const int32_t n = static_cast<int32_t>(cdiv64(keys, kChunkKvSplit));
  return n < 1 ? 1 : n;
}

// A chunked-prefill call runs its tile kernel and its decode-row split kernel side by side: the
// tile kernel keeps N of the device's nsm multiprocessors (its other CTAs leave at once) and the
// decode rows stream on the rest, taking over the tiles' multiprocessors when those finish.
// Cost model (B200 measurements): a tile CTA spends kTileKeyTileUs per 128-key tile of a
// 128-row query tile, whatever its valid rows; decode rows stream at most kDecodeSmGBs per
// multiprocessor and kHbmGBs in all. While the tiles run (phase 1) the decode rows stream at
// min(kHbmGBs, (nsm - N) kDecodeSmGBs); what is left then streams at kHbmGBs. N minimises the
// total: the time of phase 1 plus that of the rest. `key_tiles` counts the 128-key tiles of all
// tile items, `dec_bytes` the K/V bytes of the decode rows. No tiles: 0; no decode rows: nsm.
// The three constants were fitted to one B200 sweep of N = 50..95 on the mixed workload (16192 key
// tiles, 2.19 GB of decode rows), which they reproduce within 2 % for N >= 70.
constexpr float kTileKeyTileUs = 2.3f;  // µs per key tile of a 128-row query tile, per CTA
constexpr float kDecodeSmGBs = 60.f;    // tensor-core decode rows per multiprocessor, beside the tiles
constexpr float kHbmGBs = 6500.f;       // decode rows on the whole device
// Estimated time (µs) of the call when the tile kernel keeps n of the nsm multiprocessors. The
// planner keeps the n of least cost (the smallest such n on ties); with no tile items it keeps
// 0, with no decode rows all nsm.
FD_HD float chunk_tile_cost(int64_t key_tiles, float dec_bytes, int32_t nsm, int32_t n) {
  const float t1 = static_cast<float>(key_tiles) * kTileKeyTileUs / static_cast<float>(n);
  const float sm_rate = static_cast<float>(nsm - n) * kDecodeSmGBs;
  const float rate = (sm_rate < kHbmGBs ? sm_rate : kHbmGBs) * 1e3f;  // bytes per microsecond
  const float left = dec_bytes - rate * t1;
  return t1 + (left > 0.f ? left / (kHbmGBs * 1e3f) : 0.f);
}

// Upper bounds for a chunked-prefill call of T packed rows over B requests (any lengths).
FD_HD int64_t chunk_max_tile_items(int64_t B, int64_t T, int64_t hq, int64_t cap) {
  return (cdiv64(T, kQTile) + B) * cdiv64(cap > 0 ? cap : 1, kChunkKvSplit) * hq;
}
FD_HD int64_t chunk_max_slots(int64_t B, int64_t T, int64_t hkv, int64_t cap, int32_t nctas) {
  // decode rows: at most decode_max_items / Hkv splits; tile rows: ceil(S_cap / split) each
  const int64_t dec = decode_max_items(B, hkv, cap, 0, nctas) / hkv + 1;
  return (dec + T * cdiv64(cap > 0 ? cap : 1, kChunkKvSplit)) * hkv;
}

// Workspace layout (byte offsets, 256-byte aligned sections).
struct WsLayout {
  size_t dec_items, tile_items, row_nsplit, row_base, arrivals, part_o, part_lse, total;
};

// Partial slots hold the G = Hq / Hkv query heads of one KV head: [slot][G][D] fp32 outputs and
// [slot][G] base-2 LSEs, so `max_slots` counts (row, KV head, split) triples.
FD_HD WsLayout ws_layout(int64_t max_dec_items, int64_t max_tile_items, int64_t rows,
                         int64_t max_slots, int32_t hq, int32_t d, int32_t hkv = 1) {
  WsLayout L;
  size_t off = sizeof(WsHeader);
  L.dec_items = off;
  off = align_up(off + static_cast<size_t>(max_dec_items) * sizeof(DecodeItem), 256);
  L.tile_items = off;
  off = align_up(off + static_cast<size_t>(max_tile_items) * sizeof(TileItem), 256);
  L.row_nsplit = off;
  off = align_up(off + static_cast<size_t>(rows) * 4, 256);
  L.row_base = off;
  off = align_up(off + static_cast<size_t>(rows) * 4, 256);
  L.arrivals = off;
  off = align_up(off + static_cast<size_t>(rows) * hkv * 4, 256);
  const int64_t g = hq / (hkv > 0 ? hkv : 1);
  L.part_o = off;
  off = align_up(off + static_cast<size_t>(max_slots) * g * d * 4, 256);
  L.part_lse = off;
  off = align_up(off + static_cast<size_t>(max_slots) * g * 4, 256);
  L.total = off;
  return L;
}

}  // namespace fd
