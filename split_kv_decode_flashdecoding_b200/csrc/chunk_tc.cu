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
//   two threads per row, 64 keys each: mask, running max m (rescaled lazily; the pair swaps
//   its tile maxima), p = 2^(s·scale·log2e − m), running sums of p, P split into bf16 hi + lo
//   (both rounded to nearest) and stored into tensor memory
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
// A request of c <= 32 / G rows (a few speculative tokens) is a quarter item: its c G rows are
// loaded once into each 32-lane quarter of the tile, every copy's softmax takes a quarter of the
// keys (the other quarters' P words are zero), and the epilogue adds the four partial products.
// The softmax of a tile then runs on all four schedulers instead of one quarter's.
//
// Warp roles: 0-3 and 12-15 softmax (warps w and w + 12 share TMEM lanes 32 w + [0, 32), one
// query row per lane, and take keys [0, 64) and [64, 128) of each tile); 4 TMA producer of Q and
// K (2-stage K ring, the next item's Q prefetched); 5 issuer of the S products and TMEM owner;
// 6-9 epilogue (warp w reads TMEM lanes 32 (w mod 4) + [0, 32)); 10 TMA producer of V (2-stage
// ring); 11 issuer of the P·V products. The softmax is the longest step of a tile (an exp2, two
// roundings and a subtraction per key on one thread), so two warps per lane quarter halve it.
// A tcgen05.mma holds its issuing thread for about as long as the tensor pipe needs for it, so
// the two product chains of a tile are issued by two threads. K and V stages are released
// separately: K once S has read it, V once P·V has.
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
constexpr int kCkSoft2 = 12;       // warps 12-15: the second key half of the softmax
constexpr int kCkThreads = 16 * 32;
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
  // each softmax warp's scaled tile maxima, [parity][2 quarter + half][lane]: per-head and
  // larger head-packed tiles swap them within a lane quarter (xpair[parity][quarter], two
  // arrivals), quarter items among all eight warps (xall[parity], eight arrivals); each kind
  // counts its own tiles for the parity
  float tmx_pair[2][8][32], tmx_all[2][8][32];
  uint64_t xpair[2][4], xall[2];
  // quarter items: the four lane quarters' partial O (32 columns at a time) meet here, and
  // lane quarter 0 adds them (redfull: the four partials written; redfree: added)
  float red[4][32][33];
  uint64_t redfull, redfree;
  // hand-off to the epilogue warps, by item parity: per-row running max, each key half's running
  // sum, the item
  float mfin[2][kCkRows], lfin[2][2][kCkRows];
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

// Maximum of the visible keys among W consecutive S values of a row (key kbeg + i is visible
// when < nvis; full: all are); four independent maxima keep the dependency chains short.
template <int W>
__device__ __forceinline__ float masked_max(const uint32_t* raw, bool full, int kbeg, int nvis) {
  float mx[4];
#pragma unroll
  for (int a = 0; a < 4; ++a) mx[a] = -INFINITY;
  if (full) {
#pragma unroll
    for (int i = 0; i < W; ++i) mx[i & 3] = fmaxf(mx[i & 3], __uint_as_float(raw[i]));
  } else {
#pragma unroll
    for (int i = 0; i < W; ++i)
      if (kbeg + i < nvis) mx[i & 3] = fmaxf(mx[i & 3], __uint_as_float(raw[i]));
  }
  return fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3]));
}

// p = 2^(s·scale − m) for W consecutive S values of a row (invisible keys give 0), as bf16 pairs:
// whi[i] holds the nearest bf16 of keys 2i and 2i + 1, wlo[i] that of their fp32 remainders.
// Returns the fp32 sum of the p.
template <int W>
__device__ __forceinline__ float exp_split(const uint32_t* raw, bool full, int kbeg, int nvis,
                                           float scale, float negm, uint32_t (&whi)[W / 2],
                                           uint32_t (&wlo)[W / 2]) {
  float rsum[4];  // four independent partial sums of p
#pragma unroll
  for (int a = 0; a < 4; ++a) rsum[a] = 0.f;
#pragma unroll
  for (int i = 0; i < W; i += 2) {
    float x0 = fmaf(__uint_as_float(raw[i]), scale, negm);
    float x1 = fmaf(__uint_as_float(raw[i + 1]), scale, negm);
    if (!full) {
      x0 = kbeg + i < nvis ? x0 : -INFINITY;
      x1 = kbeg + i + 1 < nvis ? x1 : -INFINITY;
    }
    const float p0 = fast_exp2(x0), p1 = fast_exp2(x1);
    rsum[(i >> 1) & 3] += p0 + p1;
    const __nv_bfloat162 hi = __floats2bfloat162_rn(p0, p1);
    const float2 hf = __bfloat1622float2(hi);
    whi[i / 2] = *reinterpret_cast<const uint32_t*>(&hi);
    wlo[i / 2] = pack_bf16x2(p0 - hf.x, p1 - hf.y);
  }
  return (rsum[0] + rsum[1]) + (rsum[2] + rsum[3]);
}

template <int kD>
__global__ void __launch_bounds__(kCkThreads, 1)
    chunk_tc_kernel(const TileParams p, const __grid_constant__ CUtensorMap tmap_q,
                    const __grid_constant__ CUtensorMap tmap_qp,
                    const __grid_constant__ CUtensorMap tmap_qq,
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
      mbar_init(&S.qempty[i], 1 + 8 + 1 + 1);  // S issuer, softmax warps, V producer, P·V issuer
      mbar_init(&S.sfull[i], 1);
      mbar_init(&S.sfree[i], 1);
      mbar_init(&S.pfull[i], 8);
      mbar_init(&S.lready[i], 8);
      mbar_init(&S.lfree[i], 4);
      for (int q = 0; q < 4; ++q) mbar_init(&S.xpair[i][q], 2);
      mbar_init(&S.xall[i], 8);
    }
    mbar_init(&S.pfree, 1);
    mbar_init(&S.ofin, 1);
    mbar_init(&S.oempty, 4);
    mbar_init(&S.redfull, 4);
    mbar_init(&S.redfree, 1);
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
    prefetch_tensor_map(&tmap_qq);
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
        if (it.head_packed && it.rows <= p.quad_rows) {
          // a quarter item: the request's rows of G heads (at most 32 tile rows, ordered (chunk
          // row, head)) once in each lane quarter
          mbar_arrive_expect_tx(&S.qfull[ps], 4u * kHalves * 128u * static_cast<uint32_t>(p.g * p.qq_box_rows));
#pragma unroll
          for (int hf = 0; hf < kHalves; ++hf)
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4)
              tma_load_3d(S.q[ps][hf] + q4 * 32 * 64, &tmap_qq, &S.qfull[ps], 64 * hf, it.h * p.g, it.row0);
        } else if (it.head_packed) {
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
            // descriptors of the two 64-column halves; a 16-column step is 32 bytes, i.e. 2 in the
            // start-address field
            const uint64_t qd[2] = {smem_desc(q0, 16, 1024, kLayoutSW128), smem_desc(q1, 16, 1024, kLayoutSW128)};
            const uint64_t kd[2] = {smem_desc(smem_u32(S.k[st][0]), 16, 1024, kLayoutSW128),
                                    smem_desc(smem_u32(S.k[st][kHalves - 1]), 16, 1024, kLayoutSW128)};
#pragma unroll
            for (int kk = 0; kk < kD / 16; ++kk)
              umma_bf16_ss(tmem + kColS0 + sb * 128, qd[kk >> 2] + static_cast<uint64_t>((kk & 3) * 2),
                           kd[kk >> 2] + static_cast<uint64_t>((kk & 3) * 2), idesc_s, kk > 0 ? 1u : 0u);
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
          // V's descriptor for the first 16 keys; key step kk starts 2048 bytes further, i.e.
          // kk * 128 in the descriptor's start-address field (shared addresses stay below
          // 2^18 bytes, so the 14-bit field never carries)
          const uint64_t bd0 = smem_desc(smem_u32(S.v[vs][0]), kCkHalf, 1024, kLayoutSW128);
          const uint32_t pa = tmem + kColS0 + (J & 1) * 128;  // P of this tile, over its S buffer
          const uint32_t acc = j > 0 ? 1u : 0u;
          if (nk == kCkKeys / 16) {
            // a full tile: every address is a constant offset, so the thread issues little but
            // the products themselves
#pragma unroll
            for (int part = 0; part < 2; ++part)
#pragma unroll
              for (int kk = 0; kk < kCkKeys / 16; ++kk)
                umma_bf16_ts(tmem + (part ? kColOLo : kColOHi), pa + 32 * (kk >> 1) + 16 * part + 8 * (kk & 1),
                             bd0 + static_cast<uint64_t>(kk * 128), idesc_o, kk > 0 ? 1u : acc);
          } else {
            for (int part = 0; part < 2; ++part) {
              const uint32_t ocol = part ? kColOLo : kColOHi;
              for (int kk = 0; kk < nk; ++kk)
                umma_bf16_ts(tmem + ocol, pa + 32 * (kk >> 1) + 16 * part + 8 * (kk & 1),
                             bd0 + static_cast<uint64_t>(kk * 128), idesc_o, kk > 0 ? 1u : acc);
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
  } else if (warp < 4 || warp >= kCkSoft2) {
    // ======================= softmax (thread = TMEM lane, warp = keys of the tile) =======================
    // Warps meet only at a bounded mbarrier wait (the tile-maximum exchange), never at a named
    // barrier, so a warp whose wait timed out may leave on its own: the others' next waits time
    // out too.
    const int quad = warp & 3;
    const int half = warp >= kCkSoft2 ? 1 : 0;
    const int wslot = 2 * quad + half;
    const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
    const int r = quad * 32 + lane;     // TMEM lane = tile row
    const int stid = half * 128 + r;    // 0..255 over the eight softmax warps
    uint32_t J = 0, K = 0;
    uint32_t Jp = 0, Ja = 0;  // tiles of each exchange kind so far
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
      // the key tiles; the per-row max and sums follow at the end.
      if (!mbar_wait(&S.lfree[ob], ((K >> 1) & 1u) ^ 1u, ctx)) break;
      if (tid == 0) {
        S.epi[ob] = it;
        S.epi_stop[ob] = 0;
      }
      // Tile rows. A quarter item (a head-packed request of c <= 32 / G rows) holds its c G rows
      // in every lane quarter (row r is slot r mod 32: chunk position slot / G of head
      // slot mod G), and each of the eight warps takes 16 keys of a tile: quarter q and half h
      // take keys 32 q + 16 h + [0, 16), so a row's 128 keys are spread over eight warps on four
      // schedulers. Other head-packed tiles hold position r / G of head r mod G, per-head tiles
      // position r; there each half takes 64 keys.
      const bool quarter_item = it.head_packed && it.rows <= p.quad_rows;
      const int prow = quarter_item ? lane : r;
      const int pos = it.head_packed ? (prow * p.g_recip16) >> 16 : r;
      const int limit = pos < it.rows ? it.prefix + it.pos0 + pos : -1;
      // A warp whose 32 rows all lie outside the chunk (the last lane quarter of a head-packed
      // tile of 9 rows x 8 heads, say) has no output: it leaves its rows' P as the S bits it
      // finds, so those rows of O hold garbage that the epilogue never stores, and the next
      // item's first products overwrite.
      const bool dead = __all_sync(0xffffffffu, pos >= it.rows);
      const int kbeg = quarter_item ? 32 * quad + 16 * half : 64 * half;
      float m = -INFINITY, l = 0.f;  // l: the sum over this warp's keys
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
        // pass 1: the maximum over this warp's visible keys (scale > 0, so it is applied after);
        // a quarter item keeps its 16 values for pass 2, the 64-key halves go 32 keys at a time
        // in rolled loops (the eight roles' code shares the instruction cache)
        uint32_t raw16[16];
        float hmax = -INFINITY;
        if (valid > 0 && !dead) {
          if (quarter_item) {
            tmem_ld16(sp + kbeg, raw16);
            tmem_wait_ld();
            hmax = masked_max<16>(raw16, full, kbeg, nvis);
          } else {
#pragma unroll 1
            for (int c = 0; c < 64; c += 32) {
              uint32_t raw[32];
              tmem_ld32(sp + kbeg + c, raw);
              tmem_wait_ld();
              hmax = fmaxf(hmax, masked_max<32>(raw, full, kbeg + c, nvis));
            }
          }
          hmax *= p.scale_log2;
        }
        // the row's tile maximum: every warp posts its own, then reads those of the warps that
        // share its row (the other half of its quarter; in a quarter item all eight)
        float tmax;
        if (quarter_item) {
          float (&x)[8][32] = S.tmx_all[Ja & 1];
          x[wslot][lane] = hmax;
          __syncwarp();
          if (lane == 0) mbar_arrive(&S.xall[Ja & 1]);
          if (!mbar_wait(&S.xall[Ja & 1], (Ja >> 1) & 1u, ctx)) { ok = false; break; }
          tmax = x[0][lane];
#pragma unroll
          for (int w = 1; w < 8; ++w) tmax = fmaxf(tmax, x[w][lane]);
          ++Ja;
        } else {
          float (&x)[8][32] = S.tmx_pair[Jp & 1];
          x[wslot][lane] = hmax;
          __syncwarp();
          if (lane == 0) mbar_arrive(&S.xpair[Jp & 1][quad]);
          if (!mbar_wait(&S.xpair[Jp & 1][quad], (Jp >> 1) & 1u, ctx)) { ok = false; break; }
          tmax = fmaxf(x[2 * quad][lane], x[2 * quad + 1][lane]);
          ++Jp;
        }
        // every warp of a row reaches the same decisions from the same numbers
        const float mn = fmaxf(m, tmax);
        const bool move = mn > m + kRescaleThreshold || (m == -INFINITY && mn != -INFINITY);
        const float mref = move ? mn : m;
        const float alpha = move ? (m == -INFINITY ? 0.f : fast_exp2(m - mn)) : 1.f;
        if (j > 0 && __any_sync(0xffffffffu, move)) {
          // O changes only after the previous product has added into it; half 0 rescales O_hi,
          // half 1 O_lo (each lane quarter its own rows, or its own copy of them)
          if (!mbar_wait(&S.pfree, (J - 1) & 1u, ctx)) { ok = false; break; }
          tc_fence_after();
          const uint32_t oc = tmem + lane_base + kColOHi + half * kD;
#pragma unroll 1
          for (int c = 0; c < kD; c += 32) {
            uint32_t o[32];
            tmem_ld32(oc + c, o);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
            tmem_st32(oc + c, o);
          }
        }
        // pass 2: p = 2^(s·scale − m) over this warp's keys, split into bf16 hi + lo and written
        // over the tile's own S columns (each 32-key chunk: 16 words of hi pairs, then 16 of lo
        // pairs; a warp writes only columns it or its half-partner has read). hi is p rounded to
        // the nearest bf16 and lo the exact fp32 remainder p − hi, rounded the same way, so
        // |p − hi − lo| <= 2^-17 p, without bias. mref = −inf only when no key is visible, and
        // then every x is −inf already. A quarter item's row copy also zeroes the P words of the
        // keys other quarters take, so the four copies' products are partial sums.
        const float negm = mref == -INFINITY ? 0.f : -mref;
        float rs = 0.f;
        if (!dead) {
          if (quarter_item) {
            uint32_t whi[8], wlo[8];
            rs = exp_split<16>(raw16, full, kbeg, nvis, p.scale_log2, negm, whi, wlo);
            const uint32_t chunk = sp + 32 * quad;
            tmem_st8(chunk + 8 * half, whi);
            tmem_st8(chunk + 16 + 8 * half, wlo);
            uint32_t z[32];
#pragma unroll
            for (int i = 0; i < 32; ++i) z[i] = 0u;
            if (half == 0) {
              tmem_st32(sp + 32 * ((quad + 1) & 3), z);
              tmem_st32(sp + 32 * ((quad + 2) & 3), z);
            } else {
              tmem_st32(sp + 32 * ((quad + 3) & 3), z);
            }
          } else {
#pragma unroll 1
            for (int c = 0; c < 64; c += 32) {
              uint32_t raw[32], w[32];
              if (valid > 0) {
                tmem_ld32(sp + kbeg + c, raw);
                tmem_wait_ld();
              }
              rs += exp_split<32>(raw, full, kbeg + c, nvis, p.scale_log2, negm,
                                  *reinterpret_cast<uint32_t(*)[16]>(w),
                                  *reinterpret_cast<uint32_t(*)[16]>(w + 16));
              tmem_st32(sp + kbeg + c, w);
            }
          }
        }
        l = fmaf(l, alpha, rs);
        m = mref;
        if ((valid & 15) != 0) {
          // zero V rows [valid, next multiple of 16): they may lie past the request's keys
          const int vs = J % kCkVStages;
          if (!mbar_wait(&S.vfull[vs], (J / kCkVStages) & 1u, ctx)) { ok = false; break; }
          const int r0 = valid, r1 = (valid + 15) & ~15;
          for (int c = stid; c < (r1 - r0) * 8 * kHalves; c += 256) {
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
      // ---- hand the rows' running max and this warp's sum to the epilogue warps ----
      if (half == 0) S.mfin[ob][r] = m;
      S.lfin[ob][half][r] = l;
      __syncwarp();
      if (lane == 0) mbar_arrive(&S.lready[ob]);
      ++K;
    }
  } else {
    // ======================= epilogue: O / l and the LSE of every row =======================
    const int quad = warp & 3;
    const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
    const int r = quad * 32 + lane;
    uint32_t E = 0;  // reduction steps of quarter items so far (the same count in all four warps)
    bool ok = true;
    for (uint32_t K = 0; ok; ++K) {
      const uint32_t ob = K & 1;
      if (!mbar_wait(&S.lready[ob], (K >> 1) & 1u, ctx)) break;
      if (S.epi_stop[ob]) break;
      const TileItem it = S.epi[ob];
      const bool quarter_item = it.head_packed && it.rows <= p.quad_rows;
      // a quarter item's row (slot = lane) has a running sum in each of the eight softmax warps
      const float m = S.mfin[ob][r];
      float l = S.lfin[ob][0][r] + S.lfin[ob][1][r];
      if (quarter_item)
#pragma unroll
        for (int q = 1; q < 4; ++q)
          l += S.lfin[ob][0][((quad + q) & 3) * 32 + lane] + S.lfin[ob][1][((quad + q) & 3) * 32 + lane];
      __syncwarp();
      if (lane == 0) mbar_arrive(&S.lfree[ob]);
      if (!mbar_wait(&S.ofin, K & 1u, ctx)) break;
      tc_fence_after();
      // chunk position and query head of the row (the tile-row layouts of the softmax warps);
      // a quarter item's output is written by lane quarter 0, from the sum of the four copies
      const int prow = quarter_item ? lane : r;
      const int pos = it.head_packed ? (prow * p.g_recip16) >> 16 : r;
      const bool row_ok = pos < it.rows && (!quarter_item || quad == 0);
      const bool direct = it.nsplit == 1;
      const float inv = l > 0.f ? 1.f / l : 0.f;
      const float lse2 = l > 0.f ? m + log2f(l) : -INFINITY;
      // a row that saw no key has O = 0 (its accumulator may never have been written)
      const bool seen = l > 0.f;
      const int head = it.head_packed ? it.h * p.g + (prow - pos * p.g) : it.h;  // query head
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
        for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) + __uint_as_float(lo[i]));
        if (quarter_item) {
          // the four lane quarters' partial sums meet in shared memory (the buffer is free once
          // quarter 0 has added the previous step's)
          if (!mbar_wait(&S.redfree, (E & 1u) ^ 1u, ctx)) { ok = false; break; }
#pragma unroll
          for (int i = 0; i < 32; ++i) S.red[quad][lane][i] = __uint_as_float(o[i]);
          __syncwarp();
          if (lane == 0) mbar_arrive(&S.redfull);
          if (quad == 0) {
            if (!mbar_wait(&S.redfull, E & 1u, ctx)) { ok = false; break; }
#pragma unroll
            for (int i = 0; i < 32; ++i)
              o[i] = __float_as_uint((S.red[0][lane][i] + S.red[1][lane][i]) +
                                     (S.red[2][lane][i] + S.red[3][lane][i]));
            __syncwarp();
            if (lane == 0) mbar_arrive(&S.redfree);
          }
          ++E;
        }
        if (row_ok) {
          if (!seen)
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = 0u;
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
      if (!ok) break;
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
                              const CUtensorMap& tqq, const CUtensorMap& tk, const CUtensorMap& tv,
                              int nctas, cudaStream_t stream) {
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
  return cudaLaunchKernelEx(&cfg, chunk_tc_kernel<kD>, p, tq, tqp, tqq, tk, tv);
}

}  // namespace

cudaError_t launch_chunk_tc(const TileParams& p, const CUtensorMap& tq, const CUtensorMap& tqp,
                            const CUtensorMap& tqq, const CUtensorMap& tk, const CUtensorMap& tv,
                            int nctas, cudaStream_t stream) {
  if (p.d == 128) return launch_chunk_tc_t<128>(p, tq, tqp, tqq, tk, tv, nctas, stream);
  if (p.d == 64) return launch_chunk_tc_t<64>(p, tq, tqp, tqq, tk, tv, nctas, stream);
  return cudaErrorInvalidValue;
}

}  // namespace fd
