// Kernel parameter blocks and launcher declarations shared inside the library.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"
#include "plan.h"

namespace fd {

// Device planner for a decode call (or the decode rows of a chunked-prefill call).
struct PlanParams {
  const int32_t* lens;      // [B] cache lengths (decode) or prefix lengths (chunk mode)
  const int32_t* chunk_lens;  // chunk mode only: [B] chunk lengths; nullptr for decode
  int32_t B, hkv, hq, cap, fixed, nctas;
  int32_t align;            // split boundaries on multiples of `align` keys (<= 1: unaligned)
  int64_t max_dec_items, max_tile_items, max_rows, max_slots;
  WsHeader* hdr;
  DecodeItem* items;
  TileItem* tiles;
  int32_t* row_nsplit;
  int32_t* row_base;
  int32_t* arrivals;        // [rows * Hkv] split-completion counters of the in-kernel merge
  int32_t total_rows;       // chunk mode: packed query rows T (= sum of chunk lengths)
  int32_t decode_merged_in_kernel;  // chunk mode: decode rows merge inside their split kernel
  int32_t tile_sms;         // chunk mode: multiprocessors the tile kernel is launched on
  int64_t kv_key_bytes;     // chunk mode: K + V bytes of one key over all KV heads
  // optional export of the decode plan (fd_split_plan_device)
  int32_t* out_splits;
  int32_t* out_items;
  int32_t out_cap;
  int32_t* out_total;
};

// Split pass of decode items (both the CUDA-core and the tensor-core kernels).
struct DecodeParams {
  const void* q;     // [rows, Hq, D]
  int64_t q_sr, q_sh;  // element strides of row and head
  const void* k;     // [B, Hkv, S_cap, D], token rows contiguous
  const void* v;
  int64_t kv_sb, kv_sh;  // element strides of batch and head (same for k and v)
  void* out;         // [rows, Hq, D]
  int64_t o_sr, o_sh;
  float* lse;        // [rows, Hq] contiguous
  int32_t hq, hkv, g, d, cap;
  int32_t q_box_rows;   // rows of one Q tensor-map box (tensor-core kernel): min(16, Hq)
  int32_t kv_box_rows;  // rows of one K/V tensor-map box (tensor-core kernel): min(128, S_cap)
  float scale_log2;  // softmax scale * log2(e)
  WsHeader* hdr;
  const DecodeItem* items;  // planner output; nullptr: the tensor-core kernel plans itself
  const int32_t* row_base;
  float* part_o;     // [slots, G, D], the slots of one (row, KV head) group consecutive
  float* part_lse;   // [slots, G] (log2 domain)
  int32_t* arrivals; // [rows, Hkv] split-completion counters of the in-kernel merge
  // in-kernel plan (items == nullptr, tensor-core kernel, B <= kFusedPlanMaxBatch): the inputs of
  // the planner and the row tables the combine kernel reads
  const int32_t* lens;
  int32_t B, fixed, plan_ctas, max_items;
  int32_t* row_nsplit_out;
  int32_t* row_base_out;
  int32_t align;     // split boundaries on multiples of `align` keys (<= 1: unaligned)
  // paged cache (block_table != nullptr): k and v are [num_pages, Hkv, page_size, D] with kv_sb
  // the page stride; token t of sequence b is row t % page_size of page
  // block_table[b * pages_per_seq + t / page_size]. page_size divides 128 or is a multiple of
  // it, and split boundaries are 128-key aligned, so a key tile never crosses a page.
  const int32_t* block_table;
  int32_t pages_per_seq, page_size, num_pages;
  // bf16 pages of < 128 keys whose KV heads are consecutive (head stride = page_size rows):
  // the K/V maps are 5-D and copy a whole page per box, each 8-row group's two 64-column halves
  // side by side (see load_small_pages); 0: the 4-D maps, one box per page and half
  int32_t pg_interleave = 0;
  // E4M3 cache (kv_fp8 != 0, tensor-core kernel): k and v hold one-byte codes; the key scale is
  // folded into scale_log2 and every output is multiplied by v_scale (1 for other caches)
  float v_scale = 1.f;
  int32_t kv_fp8 = 0;
};

__device__ __forceinline__ MergeTarget merge_target(const DecodeParams& p) {
  MergeTarget t;
  t.part_o = p.part_o;
  t.part_lse = p.part_lse;
  t.arrivals = p.arrivals;
  t.out = p.out;
  t.o_sr = p.o_sr;
  t.o_sh = p.o_sh;
  t.lse = p.lse;
  t.hq = p.hq;
  t.hkv = p.hkv;
  t.g = p.g;
  t.d = p.d;
  return t;
}

// Chunked-prefill tiles.
struct TileParams {
  const void* q;     // [T, Hq, D] packed query chunks
  int64_t q_sr, q_sh;
  void* out;
  int64_t o_sr, o_sh;
  float* lse;
  int32_t hq, hkv, g, d, cap;
  int32_t q_box_rows;   // rows of one Q tensor-map box: min(128, T)
  int32_t qp_box_rows;  // chunk rows of one head-packed Q box (G heads each): min(128 / G, T)
  int32_t quad_rows;    // head-packed requests of <= 32 / G rows are quarter items (0: none)
  int32_t qq_box_rows;  // chunk rows of one quarter-item Q box (G heads each): min(32 / G, T)
  int32_t g_recip16;    // ceil(2^16 / G): (r * g_recip16) >> 16 == r / G for 0 <= r < 128
  int32_t kv_box_rows;  // rows of one K/V tensor-map box: min(128, S_cap)
  float scale_log2;
  WsHeader* hdr;
  const TileItem* tiles;
  float* part_o;
  float* part_lse;
};

// LSE merge of the partials of rows with more than one split.
struct CombineParams {
  const int32_t* row_nsplit;
  const int32_t* row_base;
  const float* part_o;
  const float* part_lse;
  void* out;
  int64_t o_sr, o_sh;
  float* lse;
  int32_t rows, hq, hkv, g, d, dtype;
};

cudaError_t launch_plan_decode(const PlanParams& p, cudaStream_t stream);
cudaError_t launch_plan_chunk(const PlanParams& p, cudaStream_t stream);

// CUDA-core split kernel: any dtype, D in {64,128}, G <= 8.
int simt_ctas_per_sm();
cudaError_t launch_decode_simt(const DecodeParams& p, int dtype, int nctas, cudaStream_t stream);

// tcgen05 split kernel: bf16 cache with D == 128, 2 <= G <= 16; or an E4M3 cache with D == 128,
// 1 <= G <= 8 (p.kv_fp8).
cudaError_t launch_decode_tc(const DecodeParams& p, const CUtensorMap& tmap_q,
                             const CUtensorMap& tmap_k, const CUtensorMap& tmap_v, int nctas,
                             cudaStream_t stream);

// tcgen05 chunked-prefill tile kernel: bf16, D == 64 or 128. tmap_qp loads head-packed Q tiles
// (G heads x qp_box_rows rows); any Q map when no tile is head-packed.
cudaError_t launch_chunk_tc(const TileParams& p, const CUtensorMap& tmap_q,
                            const CUtensorMap& tmap_qp, const CUtensorMap& tmap_qq,
                            const CUtensorMap& tmap_k, const CUtensorMap& tmap_v, int nctas,
                            cudaStream_t stream);

// Launched with programmatic dependent launch after a split kernel (tensor-core decode path; the
// CUDA-core kernel merges its own groups in-kernel).
cudaError_t launch_combine(const CombineParams& p, cudaStream_t stream);

}  // namespace fd
