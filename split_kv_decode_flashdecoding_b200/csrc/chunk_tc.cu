// Chunked-prefill attention tiles on the 5th-generation tensor cores (tcgen05 + TMEM).
//
// A work item is one key split [k0, k1) of one 128-row query tile of one query head of a chunk
// request ("大语言模型长序列推理优化：ChunkedPrefill与FlashDecoding技术解析" §2.1: the chunk's K/V
// are already in the cache; its queries attend to the whole cache under a causal mask; the
// prefix may be a reused cache, "Chunked-Prefills分块预填充机制：破解大模型推理的吞吐与延迟困局"
// §三.2). Row r of the tile is chunk position pos0 + r and sees keys j <= prefix + pos0 + r.
// Per 128-key tile of the split:
//
//   S[128 rows x 128 keys] = Q_tile · K_tileᵀ         UMMA M=128 N=128 K=D, both K-major (TMA SW128)
//   one thread per row: mask, running max m (rescaled lazily), p = 2^(s·scale·log2e − m),
//   running sum l, P split into bf16 hi + lo (both rounded to nearest) and stored into tensor
//   memory
//   O_hi[128 x D] += P_hi · V_tile, O_lo[128 x D] += P_lo · V_tile
//                                                        UMMA M=128 N=D, A from TMEM, V MN-major
//
// with head_dim D = 64 or 128 (one instantiation each).
//
// S is double-buffered in TMEM and P is written back over the S buffer it came from (per
// 32-key chunk: 16 words of hi pairs, then 16 words of lo pairs), so P is double-buffered too.
// The hi and lo products accumulate in two accumulators that the epilogue adds: the tensor
// core's fp32 accumulation truncates, and the tiny lo terms added into the hi accumulator would
// double the truncations the output carries. The two accumulators fill the rest of tensor
// memory, so an item's first P·V product waits until the epilogue has read the previous item's
// (the softmax of the new item runs meanwhile). The reference maximum m moves only when a row's
// maximum grows by more than 2^8, so O is rescaled rarely — only then does the softmax wait for
// the previous P·V product; p <= 2^8 is exact enough in fp32 and in the hi/lo split. At the end of
// the split the epilogue writes O / l and LSE = m + log2 l: the final output when the tile has a
// single split, else a partial for the combine kernel.
//
// Head-packed tiles (a request of 2 <= c <= 128 / G rows, G >= 2: a multi-token verification
// step, "大模型推理加速FlashDecoding算法原理与多GPU并行解码实战", "与其他推理加速方案的组合使用",
// item "Speculative Decoding + FlashDecoding"): one tile holds the c rows of all G query heads of
// one KV head, tile row r being chunk position r / G of query head h G + r mod G, loaded by one
// TMA box of G heads x 128 / G rows. Each key tile is then read and multiplied once per KV head,
// not once per query head; the per-row causal limit and output address follow the mapping.
//
// Warp roles: 0-3 softmax (thread = TMEM lane = query row); 4 TMA producer of Q and K (2-stage
// K ring, the next item's Q prefetched); 5 issuer of the S products and TMEM owner; 6-9 epilogue
// (warp w reads TMEM lanes 32 (w mod 4) + [0, 32)); 10 TMA producer of V (2-stage ring); 11
// issuer of the P·V products. A tcgen05.mma holds its issuing thread for about as long as the
// tensor pipe needs for it, so the two product chains of a tile are issued by two threads. K and
// V stages are released separately: K once S has read it, V once P·V has.
#include "common.cuh"
#include "internal.h"

namespace fd {

namespace {

constexpr int kCkRows = 128;   // query rows per tile = UMMA M
constexpr int kCkKeys = 128;   // keys per key tile = N of S, K of P·V
constexpr int kCkKStages = 2;
constexpr int kCkVStages = 2;
constexpr int kCkProducer = 4;     // Q and K
constexpr int kCkMma = 5;
constexpr int kCkVProducer = 10;
constexpr int kCkPv = 11;          // issues the P·V products (warp 5 the S products)
constexpr int kCkThreads = 12 * 32;
constexpr uint32_t kCkTmemCols = 512;
constexpr uint32_t kColS0 = 0;     // S/P buffers at columns 0 and 128
constexpr uint32_t kColOHi = 256;  // O accumulator of the P_hi products (D columns); the
                                   // P_lo accumulator follows at kColOHi + D
constexpr uint32_t kCkHalf = kCkRows * 64 * 2;  // one 64-column half of a 128-row tile
constexpr float kRescaleThreshold = 8.0f;       // log2 units

// kD = head dim (64 or 128) = K of S, N of P·V; rows of Q, K and V are held in kD / 64
// 64-column halves (one 128-byte swizzle row each).
template <int kD>
struct __align__(1024) CkSmem {
  static constexpr int kHalves = kD / 64;
  __nv_bfloat16 q[2][kHalves][kCkRows * 64];           // [item parity][d half], SW128
  __nv_bfloat16 k[kCkKStages][kHalves][kCkKeys * 64];  // [stage][d half], SW128
  __nv_bfloat16 v[kCkVStages][kHalves][kCkKeys * 64];
  int32_t meta[kCkKStages];                      // valid keys of the K stage (MMA warp)
  int32_t item_slot[2][2];                       // item index (-1: stop), key tiles
  TileItem item[2];
  // hand-off to the epilogue warps, by item parity: per-row running max and sum, the item
  float mfin[2][kCkRows], lfin[2][kCkRows];
  TileItem epi[2];
  int32_t epi_stop[2];
  uint64_t kfull[kCkKStages], kempty[kCkKStages], vfull[kCkVStages], vempty[kCkVStages];
  uint64_t qfull[2], qempty[2], sfull[2];
  uint64_t sfree[2];   // S/P buffer free again: the P·V product that read its P has completed
  // P(J) ready, one barrier per tile parity: a fast warp's next arrival on pfull[J & 1] is for
  // tile J + 2, whose S needs P·V(J), which needs the whole phase of tile J
  uint64_t pfull[2];
  uint64_t pfree;      // every P·V product (the softmax waits for the previous one to rescale O)
  uint64_t ofin, oempty;            // per item: its last P·V product done / its O read
  uint64_t lready[2], lfree[2];      // by item parity
  uint64_t drain, drain_pv;
  uint32_t tmem_base;
  int abort_flag;
};
static_assert(sizeof(CkSmem<128>) + 1024 <= 227 * 1024, "chunk tile kernel shared memory");
static_assert(kColOHi + 2 * 128 <= kCkTmemCols, "chunk tile kernel tensor memory");

__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<const uint32_t*>(&h);
}

template <int kD>
__global__ void __launch_bounds__(kCkThreads, 1)
    chunk_tc_kernel(const TileParams p, const __grid_constant__ CUtensorMap tmap_q,
                    const __grid_constant__ CUtensorMap tmap_qp,
                    const __grid_constant__ CUtensorMap tmap_k,
                    const __grid_constant__ CUtensorMap tmap_v) {
  using Smem = CkSmem<kD>;
  constexpr int kHalves = Smem::kHalves;
  constexpr uint32_t kColOLo = kColOHi + kD;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  Smem& S = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;

  // The planner chose how many CTAs this kernel keeps: the decode rows of the same call run
  // beside it on the other multiprocessors, so the rest leave before taking any resource.
  pdl_wait_prerequisites();
  pdl_launch_dependents();
  if (static_cast<int>(blockIdx.x) >= *reinterpret_cast<volatile int32_t*>(&p.hdr->tile_ctas)) return;

  if (tid == 0) {
    for (int s = 0; s < kCkKStages; ++s) {
      mbar_init(&S.kfull[s], 1);
      mbar_init(&S.kempty[s], 1);
    }
    for (int s = 0; s < kCkVStages; ++s) {
      mbar_init(&S.vfull[s], 1);
      mbar_init(&S.vempty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&S.qfull[i], 1);
      mbar_init(&S.qempty[i], 1 + 4 + 1 + 1);  // S issuer, softmax warps, V producer, P·V issuer
      mbar_init(&S.sfull[i], 1);
      mbar_init(&S.sfree[i], 1);
      mbar_init(&S.pfull[i], 4);
      mbar_init(&S.lready[i], 4);
      mbar_init(&S.lfree[i], 4);
    }
    mbar_init(&S.pfree, 1);
    mbar_init(&S.ofin, 1);
    mbar_init(&S.oempty, 4);
    mbar_init(&S.drain, 1);
    mbar_init(&S.drain_pv, 1);
    S.abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kCkMma) {
    tmem_alloc(&S.tmem_base, kCkTmemCols);
    tmem_relinquish();
  }
  if (warp == kCkProducer && lane == 0) {
    prefetch_tensor_map(&tmap_q);
    prefetch_tensor_map(&tmap_qp);
    prefetch_tensor_map(&tmap_k);
    prefetch_tensor_map(&tmap_v);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = S.tmem_base;
  const WaitCtx ctx{&S.abort_flag, &p.hdr->status};
  const uint32_t kv_tx = kHalves * 128u * static_cast<uint32_t>(p.kv_box_rows);

  if (warp == kCkProducer) {
    // ======================= TMA producer of Q and K =======================
    if (lane == 0) {
      const int n_items = *reinterpret_cast<volatile int32_t*>(&p.hdr->num_tile_items);
      const uint64_t pol = l2_evict_first_policy();
      uint32_t J = 0, K = 0;
      bool ok = true;
      int idx = atomicAdd(&p.hdr->tile_counter, 1);
      TileItem it{};
      if (idx < n_items) it = p.tiles[idx];
      while (ok && idx < n_items) {
        int nidx = n_items;
        TileItem nit{};
        const int len = it.k1 - it.k0;
        const int ntile = len > 0 ? (len + kCkKeys - 1) / kCkKeys : 1;
        const int claim_j = max(0, ntile - 3), read_j = max(0, ntile - 2);
        const int ps = K & 1;
        if (!mbar_wait(&S.qempty[ps], ((K >> 1) & 1u) ^ 1u, ctx)) { ok = false; break; }
        S.item_slot[ps][0] = idx;
        S.item_slot[ps][1] = ntile;
        S.item[ps] = it;
        if (it.head_packed) {
          // G heads x qp_box_rows chunk rows, rows ordered (chunk row, head)
          mbar_arrive_expect_tx(&S.qfull[ps], kHalves * 128u * static_cast<uint32_t>(p.g * p.qp_box_rows));
#pragma unroll
          for (int hf = 0; hf < kHalves; ++hf)
            tma_load_3d(S.q[ps][hf], &tmap_qp, &S.qfull[ps], 64 * hf, it.h * p.g, it.row0);
        } else {
          mbar_arrive_expect_tx(&S.qfull[ps], kHalves * 128u * static_cast<uint32_t>(p.q_box_rows));
#pragma unroll
          for (int hf = 0; hf < kHalves; ++hf)
            tma_load_3d(S.q[ps][hf], &tmap_q, &S.qfull[ps], 64 * hf, it.h, it.row0);
        }
        const int hkv = it.head_packed ? it.h : it.h / p.g;
        for (int j = 0; j < ntile; ++j, ++J) {
          if (j == claim_j) nidx = atomicAdd(&p.hdr->tile_counter, 1);
          const int st = J % kCkKStages;
          if (!mbar_wait(&S.kempty[st], ((J / kCkKStages) & 1u) ^ 1u, ctx)) { ok = false; break; }
          const int t = it.k0 + j * kCkKeys;
          const int valid = max(0, min(kCkKeys, it.k1 - t));
          S.meta[st] = valid;
          if (valid > 0) {
            mbar_arrive_expect_tx(&S.kfull[st], kv_tx);
#pragma unroll
            for (int hf = 0; hf < kHalves; ++hf)
              tma_load_4d_stream(S.k[st][hf], &tmap_k, &S.kfull[st], 64 * hf, t, hkv, it.b, pol);
          } else {
            mbar_arrive(&S.kfull[st]);
          }
          if (j == read_j && nidx < n_items) nit = p.tiles[nidx];
        }
        ++K;
        idx = nidx;
        it = nit;
      }
      if (ok) {
        const int ps = K & 1;
        if (mbar_wait(&S.qempty[ps], ((K >> 1) & 1u) ^ 1u, ctx)) {
          S.item_slot[ps][0] = -1;
          S.item_slot[ps][1] = 0;
          mbar_arrive(&S.qfull[ps]);
        }
      }
      if (S.abort_flag) {
        for (uint32_t back = 1; back <= kCkKStages && back <= J; ++back) {
          const uint32_t jj = J - back;
          mbar_drain(&S.kfull[jj % kCkKStages], (jj / kCkKStages) & 1u);
        }
      }
    }
    __syncwarp();
  } else if (warp == kCkVProducer) {
    // ======================= TMA producer of V =======================
    if (lane == 0) {
      const uint64_t pol = l2_evict_first_policy();
      uint32_t J = 0, K = 0;
      bool ok = true;
      while (ok) {
        const int ps = K & 1;
        if (!mbar_wait(&S.qfull[ps], (K >> 1) & 1u, ctx)) { ok = false; break; }
        const int idx = S.item_slot[ps][0];
        const int ntile = S.item_slot[ps][1];
        const TileItem it = S.item[ps];
        mbar_arrive(&S.qempty[ps]);
        if (idx < 0) break;
        const int hkv = it.head_packed ? it.h : it.h / p.g;
        for (int j = 0; j < ntile; ++j, ++J) {
          const int st = J % kCkVStages;
          if (!mbar_wait(&S.vempty[st], ((J / kCkVStages) & 1u) ^ 1u, ctx)) { ok = false; break; }
          const int t = it.k0 + j * kCkKeys;
          const int valid = max(0, min(kCkKeys, it.k1 - t));
          if (valid > 0) {
            mbar_arrive_expect_tx(&S.vfull[st], kv_tx);
#pragma unroll
            for (int hf = 0; hf < kHalves; ++hf)
              tma_load_4d_stream(S.v[st][hf], &tmap_v, &S.vfull[st], 64 * hf, t, hkv, it.b, pol);
          } else {
            mbar_arrive(&S.vfull[st]);
          }
        }
        ++K;
      }
      if (S.abort_flag) {
        for (uint32_t back = 1; back <= kCkVStages && back <= J; ++back) {
          const uint32_t jj = J - back;
          mbar_drain(&S.vfull[jj % kCkVStages], (jj / kCkVStages) & 1u);
        }
      }
    }
    __syncwarp();
  } else if (warp == kCkMma) {
    // ======================= S issuer =======================
    if (lane == 0) {
      const uint32_t idesc_s = idesc_bf16_f32(kCkRows, kCkKeys, false, false);
      uint32_t J = 0, K = 0;
      bool ok = true;
      while (ok) {
        const int ps = K & 1;
        if (!mbar_wait(&S.qfull[ps], (K >> 1) & 1u, ctx)) { ok = false; break; }
        const int idx = S.item_slot[ps][0];
        const int ntile = S.item_slot[ps][1];
        if (idx < 0) break;
        const uint32_t q0 = smem_u32(S.q[ps][0]);
        const uint32_t q1 = smem_u32(S.q[ps][kHalves - 1]);
        for (int j = 0; j < ntile; ++j, ++J) {
          const int st = J % kCkKStages;
          const int sb = J & 1;
          if (!mbar_wait(&S.kfull[st], (J / kCkKStages) & 1u, ctx)) { ok = false; break; }
          // the S/P buffer is free once the P·V product of tile J - 2 has read its P
          if (!mbar_wait(&S.sfree[sb], ((J >> 1) & 1u) ^ 1u, ctx)) { ok = false; break; }
          tc_fence_after();
          const int valid = S.meta[st];
          if (valid > 0) {
            const uint32_t k0 = smem_u32(S.k[st][0]);
            const uint32_t k1 = smem_u32(S.k[st][kHalves - 1]);
#pragma unroll
            for (int kk = 0; kk < kD / 16; ++kk) {
              const uint32_t qa = (kk < 4 ? q0 : q1) + (kk & 3) * 32;
              const uint32_t ka = (kk < 4 ? k0 : k1) + (kk & 3) * 32;
              umma_bf16_ss(tmem + kColS0 + sb * 128, smem_desc(qa, 16, 1024, kLayoutSW128),
                           smem_desc(ka, 16, 1024, kLayoutSW128), idesc_s, kk > 0 ? 1u : 0u);
            }
          }
          umma_commit(&S.sfull[sb]);
          umma_commit(&S.kempty[st]);
          if (j == ntile - 1) umma_commit(&S.qempty[ps]);
        }
        if (!ok) break;
        ++K;
      }
      umma_commit(&S.drain);
      mbar_drain(&S.drain, 0);
    }
    __syncwarp();
  } else if (warp == kCkPv) {
    // ======================= P·V issuer =======================
    // Follows the items the Q/K producer publishes; each tile's keys come from the item.
    if (lane == 0) {
      const uint32_t idesc_o = idesc_bf16_f32(kCkRows, kD, false, true);
      uint32_t J = 0, K = 0;
      bool ok = true;
      while (ok) {
        const int ps = K & 1;
        if (!mbar_wait(&S.qfull[ps], (K >> 1) & 1u, ctx)) { ok = false; break; }
        const int idx = S.item_slot[ps][0];
        const int ntile = S.item_slot[ps][1];
        const TileItem it = S.item[ps];
        mbar_arrive(&S.qempty[ps]);
        if (idx < 0) break;
        for (int j = 0; j < ntile; ++j, ++J) {
          const int vs = J % kCkVStages;
          const int valid = max(0, min(kCkKeys, it.k1 - (it.k0 + j * kCkKeys)));
          if (!mbar_wait(&S.vfull[vs], (J / kCkVStages) & 1u, ctx)) { ok = false; break; }
          if (!mbar_wait(&S.pfull[J & 1], (J >> 1) & 1u, ctx)) { ok = false; break; }
          // the item's first products overwrite the accumulators the previous item used
          if (j == 0 && !mbar_wait(&S.oempty, (K & 1u) ^ 1u, ctx)) { ok = false; break; }
          tc_fence_after();
          const int nk = (valid + 15) / 16;
          const uint32_t vaddr = smem_u32(S.v[vs][0]);
          const uint32_t pcol = kColS0 + (J & 1) * 128;  // P of this tile, over its S buffer
          for (int part = 0; part < 2; ++part) {
            const uint32_t ocol = part ? kColOLo : kColOHi;
            for (int kk = 0; kk < nk; ++kk) {
              const uint64_t bd = smem_desc(vaddr + kk * 2048, kCkHalf, 1024, kLayoutSW128);
              const uint32_t acol = pcol + 32 * (kk >> 1) + 16 * part + 8 * (kk & 1);
              umma_bf16_ts(tmem + ocol, tmem + acol, bd, idesc_o, (j > 0 || kk > 0) ? 1u : 0u);
            }
          }
          umma_commit(&S.pfree);
          umma_commit(&S.sfree[J & 1]);
          umma_commit(&S.vempty[vs]);
          if (j == ntile - 1) umma_commit(&S.ofin);
        }
        if (!ok) break;
        ++K;
      }
      umma_commit(&S.drain_pv);
      mbar_drain(&S.drain_pv, 0);
    }
    __syncwarp();
  } else if (warp < 4) {
    // ======================= softmax (thread = query row) =======================
    // The four warps never meet at a named barrier (rows are independent), so a warp whose wait
    // timed out may leave on its own.
    const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
    const int r = tid;
    uint32_t J = 0, K = 0;
    bool ok = true;
    while (ok) {
      const int ps = K & 1;
      if (!mbar_wait(&S.qfull[ps], (K >> 1) & 1u, ctx)) break;
      const int idx = S.item_slot[ps][0];
      const int ntile = S.item_slot[ps][1];
      const TileItem it = S.item[ps];
      __syncwarp();
      if (lane == 0) mbar_arrive(&S.qempty[ps]);
      const uint32_t ob = K & 1;
      if (idx < 0) {
        // tell the epilogue warps to stop
        if (mbar_wait(&S.lfree[ob], ((K >> 1) & 1u) ^ 1u, ctx)) {
          if (lane == 0) S.epi_stop[ob] = 1;
          __syncwarp();
          if (lane == 0) mbar_arrive(&S.lready[ob]);
        }
        break;
      }
      // The item's descriptor goes to the epilogue warps now (their hand-off slot of this parity
      // is free once they have read the item two back), so it need not stay in registers across
      // the key tiles; the per-row max and sum follow at the end.
      if (!mbar_wait(&S.lfree[ob], ((K >> 1) & 1u) ^ 1u, ctx)) break;
      if (tid == 0) {
        S.epi[ob] = it;
        S.epi_stop[ob] = 0;
      }
      // chunk position of this tile row (head-packed: row r is position r / G of head r mod G)
      // and the last key it sees (below every key when the row lies outside the chunk)
      const int pos = it.head_packed ? (r * p.g_recip16) >> 16 : r;
      const int limit = pos < it.rows ? it.prefix + it.pos0 + pos : -1;
      float m = -INFINITY, l = 0.f;
      for (int j = 0; j < ntile; ++j, ++J) {
        const int sb = J & 1;
        if (!mbar_wait(&S.sfull[sb], (J >> 1) & 1u, ctx)) { ok = false; break; }
        tc_fence_after();
        // this key tile, from the item descriptor (the K stage may already hold a later tile)
        const int kt0 = it.k0 + j * kCkKeys;
        const int valid = max(0, min(kCkKeys, it.k1 - kt0));
        // keys [0, nvis) of the tile are visible to this row: inside the split, at or before the
        // row's causal limit, and the row inside the chunk
        const int nvis = max(0, min(valid, limit - kt0 + 1));
        const bool full = __all_sync(0xffffffffu, nvis == kCkKeys);
        const uint32_t sp = tmem + lane_base + kColS0 + sb * 128;  // this tile's S, then its P
        // pass 1: the row's maximum over its visible keys (scale > 0, so it is applied after);
        // four independent maxima keep the dependency chains short
        float tmax = -INFINITY;
        if (valid > 0) {
          float mx[4];
#pragma unroll
          for (int a = 0; a < 4; ++a) mx[a] = -INFINITY;
#pragma unroll 1
          for (int h = 0; h < kCkKeys; h += 64) {
            uint32_t raw[64];
            tmem_ld32(sp + h, *reinterpret_cast<uint32_t(*)[32]>(raw));
            tmem_ld32(sp + h + 32, *reinterpret_cast<uint32_t(*)[32]>(raw + 32));
            tmem_wait_ld();
            if (full) {
#pragma unroll
              for (int i = 0; i < 64; ++i) mx[i & 3] = fmaxf(mx[i & 3], __uint_as_float(raw[i]));
            } else {
#pragma unroll
              for (int i = 0; i < 64; ++i)
                if (h + i < nvis) mx[i & 3] = fmaxf(mx[i & 3], __uint_as_float(raw[i]));
            }
          }
          tmax = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3]));
          tmax *= p.scale_log2;
        }
        const float mn = fmaxf(m, tmax);
        const bool move = mn > m + kRescaleThreshold || (m == -INFINITY && mn != -INFINITY);
        const float mref = move ? mn : m;
        const float alpha = move ? (m == -INFINITY ? 0.f : fast_exp2(m - mn)) : 1.f;
        if (j > 0 && __any_sync(0xffffffffu, move)) {
          // O changes only after the previous product has added into it
          if (!mbar_wait(&S.pfree, (J - 1) & 1u, ctx)) { ok = false; break; }
          tc_fence_after();
          const uint32_t oc = tmem + lane_base + kColOHi;  // O_hi, then O_lo right after it
#pragma unroll 1
          for (int c = 0; c < 2 * kD; c += 32) {
            uint32_t o[32];
            tmem_ld32(oc + c, o);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
            tmem_st32(oc + c, o);
          }
        }
        // pass 2, 64 keys at a time: p = 2^(s·scale − m), split into bf16 hi + lo and written over
        // the tile's own S columns (a 32-key chunk's words cover only columns already read). hi is
        // p rounded to the nearest bf16 and lo the exact fp32 remainder p − hi, rounded the same
        // way, so |p − hi − lo| <= 2^-17 p, without bias. mref = −inf only when no key is visible,
        // and then every x below is −inf already.
        const float negm = mref == -INFINITY ? 0.f : -mref;
        float rsum[4];  // four independent partial sums of p
#pragma unroll
        for (int a = 0; a < 4; ++a) rsum[a] = 0.f;
#pragma unroll 1
        for (int h = 0; h < kCkKeys; h += 64) {
          uint32_t raw[64];
          if (valid > 0) {
            tmem_ld32(sp + h, *reinterpret_cast<uint32_t(*)[32]>(raw));
            tmem_ld32(sp + h + 32, *reinterpret_cast<uint32_t(*)[32]>(raw + 32));
            tmem_wait_ld();
          }
#pragma unroll
          for (int c = 0; c < 64; c += 32) {
            uint32_t w[32];
#pragma unroll
            for (int i = 0; i < 32; i += 2) {
              const int k0 = h + c + i;
              float x0 = fmaf(__uint_as_float(raw[c + i]), p.scale_log2, negm);
              float x1 = fmaf(__uint_as_float(raw[c + i + 1]), p.scale_log2, negm);
              if (!full) {
                x0 = k0 < nvis ? x0 : -INFINITY;
                x1 = k0 + 1 < nvis ? x1 : -INFINITY;
              }
              const float p0 = fast_exp2(x0), p1 = fast_exp2(x1);
              rsum[(i >> 1) & 3] += p0 + p1;
              const __nv_bfloat162 hi = __floats2bfloat162_rn(p0, p1);
              const float2 hf = __bfloat1622float2(hi);
              w[i / 2] = *reinterpret_cast<const uint32_t*>(&hi);
              w[16 + i / 2] = pack_bf16x2(p0 - hf.x, p1 - hf.y);
            }
            tmem_st32(sp + h + c, w);
          }
        }
        const float rs = (rsum[0] + rsum[1]) + (rsum[2] + rsum[3]);
        l = fmaf(l, alpha, rs);
        m = mref;
        if ((valid & 15) != 0) {
          // zero V rows [valid, next multiple of 16): they may lie past the request's keys
          const int vs = J % kCkVStages;
          if (!mbar_wait(&S.vfull[vs], (J / kCkVStages) & 1u, ctx)) { ok = false; break; }
          const int r0 = valid, r1 = (valid + 15) & ~15;
          for (int c = tid; c < (r1 - r0) * 8 * kHalves; c += 128) {
            const int row = r0 + c / (8 * kHalves);
            *reinterpret_cast<uint4*>(reinterpret_cast<unsigned char*>(S.v[vs][(c / 8) % kHalves]) +
                                      row * 128 + (c & 7) * 16) = make_uint4(0u, 0u, 0u, 0u);
          }
          fence_proxy_async_smem();
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&S.pfull[sb]);
      }
      if (!ok) break;
      // ---- hand the rows' running max and sum to the epilogue warps ----
      S.mfin[ob][r] = m;
      S.lfin[ob][r] = l;
      __syncwarp();
      if (lane == 0) mbar_arrive(&S.lready[ob]);
      ++K;
    }
  } else {
    // ======================= epilogue: O / l and the LSE of every row =======================
    const int quad = warp & 3;
    const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
    const int r = quad * 32 + lane;
    for (uint32_t K = 0;; ++K) {
      const uint32_t ob = K & 1;
      if (!mbar_wait(&S.lready[ob], (K >> 1) & 1u, ctx)) break;
      if (S.epi_stop[ob]) break;
      const TileItem it = S.epi[ob];
      const float m = S.mfin[ob][r];
      const float l = S.lfin[ob][r];
      __syncwarp();
      if (lane == 0) mbar_arrive(&S.lfree[ob]);
      if (!mbar_wait(&S.ofin, K & 1u, ctx)) break;
      tc_fence_after();
      const int pos = it.head_packed ? (r * p.g_recip16) >> 16 : r;  // chunk position of the row
      const bool row_ok = pos < it.rows;
      const bool direct = it.nsplit == 1;
      const float inv = l > 0.f ? 1.f / l : 0.f;
      const float lse2 = l > 0.f ? m + log2f(l) : -INFINITY;
      // a row that saw no key has O = 0 (its accumulator may never have been written)
      const bool seen = l > 0.f;
      const int head = it.head_packed ? it.h * p.g + (r - pos * p.g) : it.h;  // query head
      const int hkv = head / p.g, g = head - hkv * p.g;
      const int64_t row = static_cast<int64_t>(it.row0) + pos;
      const int64_t slot = static_cast<int64_t>(it.slot0) +
                           (static_cast<int64_t>(pos) * p.hkv + hkv) * it.nsplit + it.split;
      __nv_bfloat16* out = static_cast<__nv_bfloat16*>(p.out) + row * p.o_sr +
                           static_cast<int64_t>(head) * p.o_sh;
      float* dst = p.part_o + (slot * p.g + g) * kD;
      // O = O_hi + O_lo, 32 columns at a time
#pragma unroll 1
      for (int c = 0; c < kD; c += 32) {
        uint32_t o[32], lo[32];
        tmem_ld32(tmem + lane_base + kColOHi + c, o);
        tmem_ld32(tmem + lane_base + kColOLo + c, lo);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; ++i)
          o[i] = seen ? __float_as_uint(__uint_as_float(o[i]) + __uint_as_float(lo[i])) : 0u;
        if (row_ok) {
          if (direct) {
#pragma unroll
            for (int i = 0; i < 32; i += 8) {
              uint4 v;
              v.x = pack_bf16x2(__uint_as_float(o[i + 0]) * inv, __uint_as_float(o[i + 1]) * inv);
              v.y = pack_bf16x2(__uint_as_float(o[i + 2]) * inv, __uint_as_float(o[i + 3]) * inv);
              v.z = pack_bf16x2(__uint_as_float(o[i + 4]) * inv, __uint_as_float(o[i + 5]) * inv);
              v.w = pack_bf16x2(__uint_as_float(o[i + 6]) * inv, __uint_as_float(o[i + 7]) * inv);
              *reinterpret_cast<uint4*>(out + c + i) = v;
            }
          } else {
#pragma unroll
            for (int i = 0; i < 32; i += 4)
              *reinterpret_cast<float4*>(dst + c + i) =
                  make_float4(__uint_as_float(o[i]) * inv, __uint_as_float(o[i + 1]) * inv,
                              __uint_as_float(o[i + 2]) * inv, __uint_as_float(o[i + 3]) * inv);
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&S.oempty);  // both accumulators read: the next item may start
      if (row_ok) {
        if (direct) p.lse[row * p.hq + head] = lse2 * kLn2;
        else p.part_lse[slot * p.g + g] = lse2;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kCkMma) tmem_dealloc(tmem, kCkTmemCols);
}

template <int kD>
cudaError_t launch_chunk_tc_t(const TileParams& p, const CUtensorMap& tq, const CUtensorMap& tqp,
                              const CUtensorMap& tk, const CUtensorMap& tv, int nctas,
                              cudaStream_t stream) {
  const size_t smem = sizeof(CkSmem<kD>) + 1024;
  cudaError_t e = cudaFuncSetAttribute(chunk_tc_kernel<kD>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(nctas);
  cfg.blockDim = dim3(kCkThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, chunk_tc_kernel<kD>, p, tq, tqp, tk, tv);
}

}  // namespace

cudaError_t launch_chunk_tc(const TileParams& p, const CUtensorMap& tq, const CUtensorMap& tqp,
                            const CUtensorMap& tk, const CUtensorMap& tv, int nctas,
                            cudaStream_t stream) {
  if (p.d == 128) return launch_chunk_tc_t<128>(p, tq, tqp, tk, tv, nctas, stream);
  if (p.d == 64) return launch_chunk_tc_t<64>(p, tq, tqp, tk, tv, nctas, stream);
  return cudaErrorInvalidValue;
}

}  // namespace fd
