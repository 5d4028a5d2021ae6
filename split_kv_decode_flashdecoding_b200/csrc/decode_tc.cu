// Split-KV decode kernel for GQA groups on the 5th-generation tensor cores (tcgen05 + TMEM).
//
// A work item is one split [t0, t1) of one (sequence, KV head); the CTA serves all G query heads
// of that KV head, so every K/V byte is read once ("大模型推理加速FlashDecoding算法原理与多GPU并行
// 解码实战", "部署落地的工程细节" item 3). Per 128-key tile:
//
//   Sᵀ[128 keys x 16]   = K_tile[128 x 128] · Q_groupᵀ           UMMA M=128 N=16, K-major A/B
//   p = 2^(s*scale*log2e - m')  per key lane, split into bf16 hi + lo parts (P ≈ P_hi + P_lo)
//   Oᵀ[128 d x 2·GPAD] = V_tileᵀ · [P_hi | P_lo]ᵀ                UMMA M=128 N=2·GPAD, MN-major A/B
//
// Sᵀ lives in tensor memory, double-buffered; the softmax warps read it with tcgen05.ld and keep
// the running max m and the running sums l (per key lane) in registers. O accumulates in tensor
// memory across the item's tiles (one accumulator per item parity) and is rescaled by 2^(m - m')
// only when the running max grows by more than 2^8, the online softmax of
// "大语言模型长序列推理优化：ChunkedPrefill与FlashDecoding技术解析" §3.1 with a lazy correction.
// Splitting P into two bf16 terms keeps ~16 bits of each weight in the P·V product at no visible
// cost: the tensor pipe is far from busy in this memory-bound loop, and N must be a multiple of
// 16 anyway.
//
// Warp roles: 0-3 softmax (one thread per key lane); 4 TMA producer of Q and K; 5 issuer of the
// Sᵀ products and TMEM owner; 6-9 epilogue (one thread per d lane: O / l, partial or final
// output); 10 TMA producer of V; 11 issuer of the P·V products. A product of these shapes (N of
// 16) costs its issuing thread about as long as the tensor pipe needs for it, so the two chains
// of 8 products per tile are issued by two threads side by side. K/V tiles arrive by 4-D TMA with 128-byte swizzle into a 3-stage ring whose K
// and V halves are refilled independently; keys past the sequence end inside the last tile are
// masked to p = 0 and their V rows are zeroed in shared memory before the P·V product, so stale
// or poisoned cache rows never leak. The epilogue of an item overlaps the next item's tiles.
//
// E4M3 cache (FlashDecoding page, "与其他推理加速方案的组合使用", item "Quantization +
// FlashDecoding": scores on dequantized values). The Sᵀ product runs on the codes themselves
// (tcgen05 kind::f8f6f4, K-step 32): the TMA brings a tile's K codes into shared memory with the
// 128-byte swizzle and they are the product's A operand as they are. Q goes in as two E4M3 terms
// per head, q = 2^e (c1 + c2): c1 = E4M3(q / 2^e), c2 = E4M3(q / 2^e - c1), e chosen so the head's
// largest |q| / 2^e lies in [128, 256); a bf16 value's 8 significant bits fit in the two 4-bit
// terms, so the split is exact but for values under 2^-9 of the head's scale. Columns 0-7 of Sᵀ
// are K·c1ᵀ, columns 8-15 K·c2ᵀ; the softmax adds them and applies 2^e. Four warps make the Q
// terms per item, four more expand V in place to f16 (one hardware conversion per pair of codes;
// every E4M3 value is exact in f16), and the P·V product runs on f16 operands, P split into f16
// hi + lo. The key scale is folded into the score scale and the value scale into the output;
// everything else is the bf16 kernel.
#include "common.cuh"
#include "internal.h"

namespace fd {

namespace {

constexpr int kTcKeys = 128;           // keys per tile = UMMA M of the Sᵀ product
constexpr int kTcD = 128;              // head dim = UMMA M of the Oᵀ product
constexpr int kTcStages = 3;
constexpr int kProducerWarp = 4;     // Q and K
constexpr int kMmaWarp = 5;
constexpr int kVProducerWarp = 10;
constexpr int kPvWarp = 11;             // issues the P·V products (warp 5 the Sᵀ products)
constexpr int kTcThreads = 12 * 32;
constexpr int kConvWarp0 = 12;          // E4M3 cache: warps 12-15 split Q, 16-19 expand V
constexpr int kF8Threads = 20 * 32;
constexpr int kSoftmaxThreads = 128;
constexpr uint32_t kTmemCols = 128;
constexpr uint32_t kHalfBytes = kTcKeys * 64 * 2;   // one 64-column half of a K or V tile

constexpr int kMaxPageBoxes = 128 / 8;  // pages of one key tile (pages of >= 8 keys)
constexpr int kPidSlots = 8;             // page-id ring of the paged producers
constexpr int kPidAhead = 4;             // pages < 128 keys: ids copied this many tiles ahead

// kF8 (E4M3 cache): a K stage holds only the tile's codes (128 rows of 128 bytes, the size of one
// bf16 half), since the expanded K lives in tensor memory; a V stage holds the codes in its upper
// half and is expanded in place.
template <int GPAD, bool kF8 = false>
struct __align__(1024) TcSmem {
  static constexpr int kNO = 2 * GPAD;           // Oᵀ columns: hi then lo
  static constexpr int kPGroups = kNO / 8;       // 8-column core-matrix groups of Pᵀ
  static constexpr int kStages = kTcStages;  // K stages
  // V stages: an E4M3 tile's V path is longer (copy, expansion to f16, then P·V) and its stages
  // are refilled only once that product has completed, so it keeps one stage more
  static constexpr int kVStages = kF8 ? kTcStages + 1 : kTcStages;
  static constexpr int kKSlabs = kF8 ? 1 : 2;
  __nv_bfloat16 k[kStages][kKSlabs][kTcKeys * 64];  // [stage][d half][row*64 + col], SW128
  __nv_bfloat16 v[kVStages][2][kTcKeys * 64];
  __nv_bfloat16 q[2][2][16 * 64];                // [item parity][d half], SW128
  // E4M3 cache: Q as two E4M3 terms per head (rows 0-7 c1, rows 8-15 c2; 128 codes per row,
  // SW128), by item parity, and each head's scale 2^e
  unsigned char q8[kF8 ? 2 : 1][kF8 ? 16 * 128 : 16];
  float qscale[2][GPAD];
  __nv_bfloat16 p[2][kPGroups * kTcKeys * 8];    // [tile parity], MN-major core matrices
  float wmax[2][4][GPAD];
  // hand-off to the epilogue warps, by item parity
  float lred[2][4][GPAD];                        // per softmax warp: sum of its key lanes' l
  float mfin[2][GPAD];                           // final running max
  int32_t epi[2][4];                             // row (-1: stop), KV head, splits, slot
  int32_t meta[kStages][2];                      // per stage: tile start, valid keys (MMA warp)
  int32_t vmeta[kVStages];                        // E4M3: valid keys of the stage's V tile
  // in-kernel plan: lengths, split counts, rank order, partial-slot bases (row order) and item
  // offsets (rank order); both scans also store their total after the last entry (B + 1)
  int32_t plan_len[kFusedPlanMaxBatch], plan_n[kFusedPlanMaxBatch];
  int32_t plan_order[kFusedPlanMaxBatch], plan_rbase[kFusedPlanMaxBatch + 1];
  int32_t plan_ioff[kFusedPlanMaxBatch + 1];
  long long plan_red[kF8Threads / 32];
  long long plan_red4[kF8Threads / 32][kPlanWaveChoices];  // split sums per wave choice
  int32_t plan_clamped;
  int32_t item_slot[2][2];                       // item index (-1: stop), tiles
  DecodeItem item[2];                            // the item's descriptor (by item parity)
  // K and V of a stage are released separately: K once the Sᵀ product has read it, V once the
  // P·V product has, so the next K copy starts while the current tile is still in softmax.
  uint64_t kfull[kStages], vfull[kVStages], kempty[kStages], vempty[kVStages];
  uint64_t qfull[2], qempty[2], sfull[2], sempty[2], pfull[2], pempty[2];
  uint64_t ofull[2];   // by tile parity: that tile's P·V product has completed
  uint64_t ofin[2];    // by item parity: the item's last P·V product has completed
  uint64_t oempty[2];  // by item parity: the epilogue has read that item's O accumulator
  uint64_t lready[2], lfree[2];  // by item parity: hand-off written / read
  // E4M3 cache: the TMA completes vraw (V codes in the upper half of the stage); vfull then
  // means "expanded to f16" and is completed by the four expanding warps. q8full: the item's Q
  // terms are ready (the four Q warps).
  uint64_t vraw[kVStages];
  uint64_t q8full[2];
  // paged cache: physical page ids of tile J in slot J mod kPidSlots, written by the Q/K producer
  // (pages < 128 keys: copied asynchronously kPidAhead tiles ahead by its 32 lanes) and released
  // by the V producer (pidempty)
  int32_t pid[kPidSlots][kMaxPageBoxes];
  uint64_t pidfull[kPidSlots], pidempty[kPidSlots];
  uint64_t drain, drain_pv;
  uint32_t tmem_base;
  int abort_flag;
};

// Pages of < 128 keys (8, 16, 32 or 64): the 128-key tile that starts at key t (a multiple of
// 128 in a paged plan) and holds `valid` keys spans the n pages first .. first + n - 1 of the
// sequence's block-table row that hold some of its valid keys.
struct SmallPages {
  int first, n;
};
__device__ __forceinline__ SmallPages small_pages(int t, int valid, int page_shift) {
  SmallPages sp;
  sp.first = t >> page_shift;
  sp.n = valid <= 0 ? 0 : ((valid - 1) >> page_shift) + 1;
  return sp;
}

// Whole warp: start the asynchronous copy of a tile's page ids from the block table into `dst`,
// lane i copying entry i (entries past the sequence's row are not copied; readers take them as
// -1), then let `bar` count this lane's copies (every lane arrives: the barrier expects 32).
__device__ __forceinline__ void prefetch_small_pages(int32_t* dst, uint64_t* bar,
                                                     const DecodeParams& p, int b,
                                                     const SmallPages& sp, int lane) {
  if (lane < sp.n && sp.first + lane < p.pages_per_seq)
    cp_async_4(dst + lane, p.block_table + static_cast<int64_t>(b) * p.pages_per_seq + sp.first + lane);
  cp_async_mbar_arrive(bar);
}

// Page id of the tile starting at key t of sequence b when pages hold >= 128 keys (-1 past the
// sequence's table row).
__device__ __forceinline__ int32_t tile_page_id(const DecodeParams& p, int b, int t) {
  const int first = t / p.page_size;
  return first < p.pages_per_seq ? p.block_table[static_cast<int64_t>(b) * p.pages_per_seq + first]
                                 : -1;
}

// tma_load_4d_stream over a 5-D map (one page of a paged cache in the interleaved layout of
// load_small_pages).
__device__ __forceinline__ void tma_load_5d_stream(void* dst, const CUtensorMap* map,
                                                   uint64_t* bar, int32_t c0, int32_t c1,
                                                   int32_t c2, int32_t c3, int32_t c4,
                                                   uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.5d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      ".L2::cache_hint [%0], [%1, {%3, %4, %5, %6, %7}], [%2], %8;" ::"r"(smem_u32(dst)),
      "l"(map), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(c4), "l"(policy)
      : "memory");
}

// Whole warp: issue the K or V loads of one 128-key tile over pages of < 128 keys, page ids
// from `ids` (a slot of the ring), one box per lane:
// - an E4M3 cache: lane i < n copies page i's whole 128-byte rows;
// - bf16 with p.pg_interleave: lane i < n copies page i whole through the 5-D map, into the
//   interleaved tile layout (8-row group r of the tile at r * 2048 bytes, its first 64-column
//   half there and its second 1024 bytes further: both halves are 1024-byte swizzle atoms, so
//   the products read them with a group stride of 2048);
// - bf16 otherwise: lane i < n copies page i's first 64-column half into dst0 (the two-slab
//   layout, each half's rows 128 bytes apart) and lane n + i its second half into dst1.
// A box costs the copy engine about the same whatever its size, so one box per page halves the
// issue work of 16-key pages. A page that holds some of the tile's `valid` keys but whose index
// lies outside the pool raises FD_FLAG_BAD_PAGE; its copy still runs and reads zeros (a TMA
// coordinate outside the tensor). The caller has announced small_pages_bytes() on `bar`.
template <bool kF8>
__device__ __forceinline__ void load_small_pages(__nv_bfloat16* dst0, __nv_bfloat16* dst1,
                                                 const CUtensorMap* map, uint64_t* bar,
                                                 const SmallPages& sp, const int32_t* ids,
                                                 const DecodeParams& p, int h, int valid,
                                                 uint64_t pol, int lane) {
  const int rows = p.page_size;
  const bool whole = kF8 || p.pg_interleave != 0;  // one box per page
  const int boxes = whole ? sp.n : 2 * sp.n;
  bool bad = false;
  if (lane < boxes) {
    const int half = whole ? 0 : (lane >= sp.n ? 1 : 0);
    const int i = lane - half * sp.n;
    const int32_t id = sp.first + i < p.pages_per_seq ? ids[i] : -1;
    bad = i * rows < valid && (id < 0 || id >= p.num_pages);
    if constexpr (kF8) {
      tma_load_4d_stream(reinterpret_cast<unsigned char*>(dst0) + i * rows * 128, map, bar, 0, 0,
                         h, id, pol);
    } else {
      if (whole)  // page i = 8-row groups i * rows / 8 ..: 256 bytes (128 elements) per row
        tma_load_5d_stream(dst0 + i * rows * 128, map, bar, 0, 0, 0, h * (rows >> 3), id, pol);
      else
        tma_load_4d_stream((half ? dst1 : dst0) + i * rows * 64, map, bar, half * 64, 0, h, id, pol);
    }
  }
  if (__any_sync(0xffffffffu, bad) && lane == 0) atomicOr(&p.hdr->status, FD_FLAG_BAD_PAGE);
}

// Bytes load_small_pages delivers (both halves; E4M3: one byte per element).
template <bool kF8>
__device__ __forceinline__ uint32_t small_pages_bytes(const SmallPages& sp, const DecodeParams& p) {
  return (kF8 ? 1u : 2u) * 128u * static_cast<uint32_t>(p.page_size * sp.n);
}

// Whole warp: every lane waits for the phase itself (so each lane sees what the phase guards);
// true only if every lane's wait succeeded.
__device__ __forceinline__ bool warp_mbar_wait(uint64_t* bar, uint32_t parity, const WaitCtx& ctx) {
  const bool ok = mbar_wait(bar, parity, ctx);
  return __all_sync(0xffffffffu, ok);
}

// The loads of one 128-key tile that lies inside one page of >= 128 keys, from row `row0`.
template <bool kF8>
__device__ __forceinline__ void load_tile_page1(__nv_bfloat16* dst0, __nv_bfloat16* dst1,
                                                const CUtensorMap* map, uint64_t* bar, int32_t id,
                                                int row0, const DecodeParams& p, int h,
                                                uint64_t pol) {
  if (id < 0 || id >= p.num_pages) atomicOr(&p.hdr->status, FD_FLAG_BAD_PAGE);
  if constexpr (kF8) {
    tma_load_4d_stream(dst0, map, bar, 0, row0, h, id, pol);
  } else {
    tma_load_4d_stream(dst0, map, bar, 0, row0, h, id, pol);
    tma_load_4d_stream(dst1, map, bar, 64, row0, h, id, pol);
  }
}

// Four E4M3 codes (the bytes of w, the first in the low byte) as two f16 pairs, exactly, by the
// hardware conversion of a pair of codes.
__device__ __forceinline__ void e4m3x4_to_f16(uint32_t w, uint32_t& lo, uint32_t& hi) {
  asm("{\n\t.reg .b16 a, b;\n\t"
      "mov.b32 {a, b}, %2;\n\t"
      "cvt.rn.f16x2.e4m3x2 %0, a;\n\t"
      "cvt.rn.f16x2.e4m3x2 %1, b;\n\t}"
      : "=r"(lo), "=r"(hi)
      : "r"(w));
}

// In-place expansion of one V tile of an E4M3 cache by 128 threads (ct = 0..127). The TMA put
// the 128 rows of 128 codes (128-byte swizzle) into the upper 64-column half of the stage; the
// f16 rows go to both halves in the layout of a 16-bit tile, rows >= valid as zeros. Thread ct
// expands the 16-byte chunk c = ct % 8 of rows 16 i + ct / 8 (i = 0..7); the upper half of bf16
// row r takes exactly the bytes of code row r, every row is expanded by the warp that loads it,
// and a warp loads the codes of a group of rows before it stores any of them, so no code is
// overwritten before it is read.
__device__ __forceinline__ void expand_v_tile(__nv_bfloat16 (&buf)[2][kTcKeys * 64], int ct,
                                              int valid) {
  unsigned char* h0 = reinterpret_cast<unsigned char*>(buf[0]);
  unsigned char* h1 = reinterpret_cast<unsigned char*>(buf[1]);
  const int c = ct & 7, r0 = ct >> 3, x = r0 & 7;  // (16 i + r0) & 7 == x for every i
  unsigned char* half = c >= 4 ? h1 : h0;
  const int sa = ((2 * (c & 3)) ^ x) << 4;  // swizzled slot of elements 16c .. 16c+7
  const int sb = sa ^ 16;                   // and of 16c+8 .. 16c+15
  // two groups of four rows per thread; a group's stores touch only rows the warp loaded in it
#pragma unroll 1
  for (int g = 0; g < 2; ++g) {
    uint4 w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
      w[i] = *reinterpret_cast<const uint4*>(h1 + (16 * (4 * g + i) + r0) * 128 + ((c ^ x) << 4));
    __syncwarp();
    const bool full = valid >= kTcKeys;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int r = 16 * (4 * g + i) + r0;
      uint4 a, b;
      e4m3x4_to_f16(w[i].x, a.x, a.y);
      e4m3x4_to_f16(w[i].y, a.z, a.w);
      e4m3x4_to_f16(w[i].z, b.x, b.y);
      e4m3x4_to_f16(w[i].w, b.z, b.w);
      if (!full && r >= valid) a = b = make_uint4(0u, 0u, 0u, 0u);
      *reinterpret_cast<uint4*>(half + r * 128 + sa) = a;
      *reinterpret_cast<uint4*>(half + r * 128 + sb) = b;
    }
  }
}

// dynamic shared memory per CTA, plus the 1024 bytes of alignment slack the kernel may use
static_assert(sizeof(TcSmem<8>) + 1024 <= 227 * 1024, "tensor-core decode smem (G <= 8)");
static_assert(sizeof(TcSmem<16>) + 1024 <= 227 * 1024, "tensor-core decode smem (G <= 16)");
static_assert(sizeof(TcSmem<8, true>) + 1024 <= 227 * 1024, "tensor-core decode smem (E4M3)");

// Exclusive prefix sum over i < n (n <= 32 * 8 here) by one warp: out[i] = sum_{j<i} val(j),
// out[n] = the total (out holds n + 1 entries).
template <typename F>
__device__ __forceinline__ void warp_exclusive_scan(int n, F val, int32_t* out) {
  const int lane = threadIdx.x & 31;
  const int per = (n + 31) / 32;
  const int lo = lane * per;
  int32_t local = 0;
  for (int i = 0; i < per; ++i)
    if (lo + i < n) local += val(lo + i);
  int32_t incl = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int32_t y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  int32_t run = incl - local;
  for (int i = 0; i < per; ++i)
    if (lo + i < n) {
      out[lo + i] = run;
      run += val(lo + i);
    }
  if (lane == 31) out[n] = incl;
}

// log2 of the growth of the running maximum that forces a rescale. Below it the weights
// 2^(x - m) of a tile stay under 2^8, which fp32 sums and the bf16 hi/lo split of P carry
// without loss, so most tiles skip the exact cross-warp maximum and leave O untouched.
constexpr float kRescaleThreshold = 8.f;

// Cache layouts, one kernel instantiation each (the producers' loops stay small).
enum PageMode : int { kContiguous = 0, kBigPages = 1, kSmallPages = 2 };

template <int GPAD, int kMode, bool kF8>
__global__ void __launch_bounds__(kF8 ? kF8Threads : kTcThreads, 1)
    decode_tc_kernel(const DecodeParams p, const __grid_constant__ CUtensorMap tmap_q,
                     const __grid_constant__ CUtensorMap tmap_k,
                     const __grid_constant__ CUtensorMap tmap_v) {
  using Smem = TcSmem<GPAD, kF8>;
  constexpr int kNO = Smem::kNO;
  constexpr int kStages = Smem::kStages;
  constexpr int kVStages = Smem::kVStages;
  constexpr int kThreads = kF8 ? kF8Threads : kTcThreads;
  constexpr uint32_t kColO = 32;  // Sᵀ buffers at columns [0, 32), O accumulators after them
  constexpr uint32_t kCols = kTmemCols;
  static_assert(kColO + 2 * kNO <= kCols, "tensor memory of the decode kernel");
  static_assert(!kF8 || GPAD == 8, "the E4M3 kernel serves groups of <= 8 heads");
  constexpr uint32_t kRowBytes = kF8 ? 128u : 256u;  // bytes of one cached K or V row
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  // dynamic shared memory is only guaranteed 16-byte aligned: round up to 1024 for SW128
  Smem& S = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;

  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&S.kfull[s], 1);
      mbar_init(&S.kempty[s], 1);
    }
    for (int s = 0; s < kVStages; ++s) {
      mbar_init(&S.vfull[s], kF8 ? 4 : 1);
      mbar_init(&S.vempty[s], 1);
      mbar_init(&S.vraw[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&S.qfull[i], 1);
      // Sᵀ issuer, softmax warps, V producer, P·V issuer (and the four Q warps of an E4M3 cache)
      mbar_init(&S.qempty[i], kF8 ? 1 + 4 + 1 + 1 + 4 : 1 + 4 + 1 + 1);
      mbar_init(&S.q8full[i], 4);
      mbar_init(&S.sfull[i], 1);
      mbar_init(&S.sempty[i], 4);
      mbar_init(&S.pfull[i], 4);
      mbar_init(&S.pempty[i], 1);
      mbar_init(&S.ofull[i], 1);
      mbar_init(&S.ofin[i], 1);
      mbar_init(&S.oempty[i], 4);
      mbar_init(&S.lready[i], 4);
      mbar_init(&S.lfree[i], 4);
    }
    for (int i = 0; i < kPidSlots; ++i) {
      mbar_init(&S.pidfull[i], kMode == kSmallPages ? 32 : 1);
      mbar_init(&S.pidempty[i], 1);
    }
    mbar_init(&S.drain, 1);
    mbar_init(&S.drain_pv, 1);
    S.abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(&S.tmem_base, kCols);
    tmem_relinquish();
  }
  if (warp == kProducerWarp && lane == 0) {
    prefetch_tensor_map(&tmap_q);
    prefetch_tensor_map(&tmap_k);
    prefetch_tensor_map(&tmap_v);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = S.tmem_base;
  const WaitCtx ctx{&S.abort_flag, &p.hdr->status};
  const bool fused = p.items == nullptr;
  constexpr bool paged = kMode != kContiguous;
  if (fused) {
    // ---- the split plan, computed by every CTA in shared memory (the planner's arithmetic):
    // clamped lengths and their sum, the chunk size, split counts, longest-first ranks, item
    // offsets in rank order and partial-slot bases in row order. Only the lengths are read from
    // global memory; they are an input of this call, so this may run before the wait below.
    const int B = p.B;
    long long local = 0;
    bool clamped = false;
    for (int b = tid; b < B; b += kThreads) {
      const int32_t raw = p.lens[b];
      const int32_t L = clamp_len(raw, p.cap);
      clamped |= L != raw;
      S.plan_len[b] = L;
      local += L;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) local += __shfl_xor_sync(0xffffffffu, local, o);
    clamped = __any_sync(0xffffffffu, clamped);
    if (lane == 0) S.plan_red[warp] = local;
    if (tid == 0) S.plan_clamped = 0;
    __syncthreads();
    if (lane == 0 && clamped) S.plan_clamped = 1;
    long long total = 0;
#pragma unroll
    for (int w = 0; w < kThreads / 32; ++w) total += S.plan_red[w];
    int32_t chunk = 0;
    if (p.fixed <= 0) {  // the same for every thread
      int32_t chunks[kPlanWaveChoices];
      long long cnt[kPlanWaveChoices];
#pragma unroll
      for (int i = 0; i < kPlanWaveChoices; ++i) {
        chunks[i] = plan_chunk_for_waves(total, p.hkv, p.plan_ctas, plan_waves(i));
        cnt[i] = 0;
      }
      for (int b = tid; b < B; b += kThreads)
#pragma unroll
        for (int i = 0; i < kPlanWaveChoices; ++i) cnt[i] += plan_num_splits(S.plan_len[b], chunks[i], 0);
#pragma unroll
      for (int i = 0; i < kPlanWaveChoices; ++i) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) cnt[i] += __shfl_xor_sync(0xffffffffu, cnt[i], o);
        if (lane == 0) S.plan_red4[warp][i] = cnt[i];
      }
      __syncthreads();
      int64_t sums[kPlanWaveChoices];
#pragma unroll
      for (int i = 0; i < kPlanWaveChoices; ++i) {
        sums[i] = 0;
#pragma unroll
        for (int w = 0; w < kThreads / 32; ++w) sums[i] += S.plan_red4[w][i];
      }
      chunk = plan_pick_chunk(chunks, sums, p.hkv, p.plan_ctas);
    }
    for (int b = tid; b < B; b += kThreads) {
      const int32_t n = plan_num_splits(S.plan_len[b], chunk, p.fixed);
      S.plan_n[b] = n;
      S.plan_ioff[b] = plan_sort_key(S.plan_len[b], n);  // sort keys until the scan below
    }
    __syncthreads();
    // longest first: rank = sequences with a larger key, or an equal key and a smaller index
    for (int b = tid; b < B; b += kThreads) {
      const int32_t kb = S.plan_ioff[b];
      int r = 0;
      for (int j = 0; j < B; ++j) {
        const int32_t kj = S.plan_ioff[j];
        r += (kj > kb || (kj == kb && j < b)) ? 1 : 0;
      }
      S.plan_order[r] = b;
    }
    __syncthreads();
    if (warp == 0)
      warp_exclusive_scan(B, [&](int r) { return S.plan_n[S.plan_order[r]] * p.hkv; }, S.plan_ioff);
    else if (warp == 1)
      warp_exclusive_scan(B, [&](int b) { return S.plan_n[b]; }, S.plan_rbase);
    __syncthreads();
  }
  // Everything above overlapped the kernel before this one (programmatic dependent launch);
  // workspace and outputs are touched only below. The combine kernel may launch now: it waits
  // for this grid the same way.
  pdl_wait_prerequisites();
  pdl_launch_dependents();
  const int32_t fused_items = fused ? S.plan_ioff[p.B] : 0;
  const bool fused_overflow = fused && fused_items > p.max_items;
  if (fused && blockIdx.x == 0) {
    // the combine kernel's row tables, and the status flags the planner would raise
    for (int b = tid; b < p.B; b += kThreads) {
      p.row_nsplit_out[b] = S.plan_n[b];
      p.row_base_out[b] = S.plan_rbase[b];
    }
    if (tid == 0 && S.plan_clamped) atomicOr(&p.hdr->status, FD_FLAG_LEN_CLAMPED);
    if (tid == 0 && fused_overflow) atomicOr(&p.hdr->status, FD_FLAG_PLAN_OVERFLOW);
  }
  // item idx of the in-kernel plan: sequence of rank r (largest r with ioff[r] <= idx), then
  // KV head and split, exactly as the planner lays items out
  auto fused_item = [&](int idx) {
    int lo = 0, hi = p.B;
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (S.plan_ioff[mid] <= idx) lo = mid; else hi = mid;
    }
    const int b = S.plan_order[lo];
    const int n = S.plan_n[b];
    const int local = idx - S.plan_ioff[lo];
    const int h = local / n, s = local - h * n;
    DecodeItem it;
    it.row = b;
    it.b = b;
    it.h = h;
    it.split = s;
    plan_split_range(S.plan_len[b], n, s, p.fixed, p.align, &it.t0, &it.t1);
    it.nsplit = n;
    it.slot = S.plan_rbase[b] * p.hkv + h * n + s;
    return it;
  };

  if (warp == kProducerWarp && kMode == kSmallPages) {
    // ============ TMA producer of Q and K, pages of < 128 keys (whole warp) ============
    // A tile spans up to 16 pages here, so its page ids and page copies go one per lane: the
    // warp spends a few instructions per tile whatever the page count, where one thread would
    // spend one short dependent sequence per page. The item schedule is the one below.
    const int pshift = __ffs(p.page_size) - 1;  // page sizes 8, 16, 32, 64
    const int n_items = fused ? (fused_overflow ? 0 : fused_items)
                              : *reinterpret_cast<volatile int32_t*>(&p.hdr->num_dec_items);
    const uint64_t pol = l2_evict_first_policy();
    auto claim = [&]() {
      int v = 0;
      if (lane == 0) v = atomicAdd(&p.hdr->dec_counter, 1);
      return __shfl_sync(0xffffffffu, v, 0);
    };
    uint32_t J = 0, K = 0, pf = 0;
    bool ok = true;
    int idx = claim();
    DecodeItem it{};
    if (idx < n_items) it = fused ? fused_item(idx) : p.items[idx];
    while (ok && idx < n_items) {
      int nidx = n_items;
      DecodeItem nit{};
      bool have_next = false;
      const int len = it.t1 - it.t0;
      const int ntile = len > 0 ? (len + kTcKeys - 1) / kTcKeys : 1;
      const int ps = K & 1;
      if (!warp_mbar_wait(&S.qempty[ps], ((K >> 1) & 1u) ^ 1u, ctx)) { ok = false; break; }
      if (lane == 0) {
        S.item_slot[ps][0] = idx;
        S.item_slot[ps][1] = ntile;
        S.item[ps] = it;
        mbar_arrive_expect_tx(&S.qfull[ps], 2u * 128u * static_cast<uint32_t>(p.q_box_rows));
        tma_load_3d(S.q[ps][0], &tmap_q, &S.qfull[ps], 0, it.h * p.g, it.row);
        tma_load_3d(S.q[ps][1], &tmap_q, &S.qfull[ps], 64, it.h * p.g, it.row);
      }
      const int claim_j = max(0, ntile - 3), read_j = max(0, ntile - 2);
      for (int j = 0; j < ntile; ++j, ++J) {
        if (j == claim_j) nidx = claim();
        if (j == read_j && nidx < n_items) {
          nit = fused ? fused_item(nidx) : p.items[nidx];
          have_next = true;
        }
        // page ids of the tiles up to J + kPidAhead that are known (this item's and, once read,
        // the next item's)
        while (pf <= J + kPidAhead) {
          const int ahead = j + static_cast<int>(pf - J);
          int xb, xt, xend;  // sequence, first key and key end of tile pf
          if (ahead < ntile) {
            xb = it.b;
            xt = it.t0 + ahead * kTcKeys;
            xend = it.t1;
          } else {
            const int nl = nit.t1 - nit.t0;
            if (!have_next || ahead - ntile >= (nl > 0 ? (nl + kTcKeys - 1) / kTcKeys : 1)) break;
            xb = nit.b;
            xt = nit.t0 + (ahead - ntile) * kTcKeys;
            xend = nit.t1;
          }
          const int slot = pf % kPidSlots;
          // the V producer has released the slot's previous tile
          if (!warp_mbar_wait(&S.pidempty[slot], ((pf / kPidSlots) & 1u) ^ 1u, ctx)) { ok = false; break; }
          prefetch_small_pages(S.pid[slot], &S.pidfull[slot], p, xb,
                               small_pages(xt, min(kTcKeys, xend - xt), pshift), lane);
          ++pf;
        }
        if (!ok) break;
        const int st = J % kStages;
        const int t = it.t0 + j * kTcKeys;
        const int valid = max(0, min(kTcKeys, it.t1 - t));
        if (!warp_mbar_wait(&S.kempty[st], ((J / kStages) & 1u) ^ 1u, ctx)) { ok = false; break; }
        if (!warp_mbar_wait(&S.pidfull[J % kPidSlots], (J / kPidSlots) & 1u, ctx)) { ok = false; break; }
        const SmallPages sp = small_pages(t, valid, pshift);
        uint64_t* kbar = &S.kfull[st];  // the copy completes kfull (E4M3: the codes as they are)
        if (lane == 0) {
          S.meta[st][0] = t;
          S.meta[st][1] = valid;
          if (valid > 0) mbar_arrive_expect_tx(kbar, small_pages_bytes<kF8>(sp, p));
          else mbar_arrive(kbar);
        }
        __syncwarp();
        if (valid > 0)
          load_small_pages<kF8>(S.k[st][0], S.k[st][Smem::kKSlabs - 1], &tmap_k, kbar, sp,
                                S.pid[J % kPidSlots], p, it.h, valid, pol, lane);
      }
      ++K;
      idx = nidx;
      it = nit;
    }
    if (ok && warp_mbar_wait(&S.qempty[K & 1], ((K >> 1) & 1u) ^ 1u, ctx) && lane == 0) {
      S.item_slot[K & 1][0] = -1;
      S.item_slot[K & 1][1] = 0;
      mbar_arrive(&S.qfull[K & 1]);
    }
    asm volatile("cp.async.wait_all;" ::: "memory");
    if (S.abort_flag && lane == 0) {
      // let copies already issued land before shared memory is released
      for (uint32_t back = 1; back <= kStages && back <= J; ++back) {
        const uint32_t jj = J - back;
        mbar_drain(&S.kfull[jj % kStages], (jj / kStages) & 1u);
      }
    }
    __syncwarp();
  } else if (kMode != kSmallPages && warp == kProducerWarp) {
    // ============ TMA producer of Q and K (contiguous cache, or pages of >= 128 keys) ============
    if (lane == 0) {
      const int n_items = fused ? (fused_overflow ? 0 : fused_items)
                                : *reinterpret_cast<volatile int32_t*>(&p.hdr->num_dec_items);
      const uint64_t pol = l2_evict_first_policy();
      uint32_t J = 0, K = 0;
      bool ok = true;
      // The next item is claimed (atomic on the work cursor) when three tiles of the current one
      // remain and its descriptor is read one tile later, so both round trips overlap the ring's
      // lookahead: under full HBM load a dependent global access takes microseconds, and the
      // ring would drain waiting for it at every item boundary. Claiming no earlier keeps the
      // tail short (a CTA never sits on an item it cannot start soon).
      int idx = atomicAdd(&p.hdr->dec_counter, 1);
      DecodeItem it{};
      if (idx < n_items) it = fused ? fused_item(idx) : p.items[idx];
      // pages of >= 128 keys: the one id of the next tile is loaded into a register one tile
      // ahead and handed to the V producer through the ring
      int32_t id_pre = -1;
      bool have_pre = false;
      while (ok && idx < n_items) {
        int nidx = n_items;
        DecodeItem nit{};
        bool have_next = false;
        const int len = it.t1 - it.t0;
        const int ntile = len > 0 ? (len + kTcKeys - 1) / kTcKeys : 1;
        const int ps = K & 1;
        if (!mbar_wait(&S.qempty[ps], ((K >> 1) & 1u) ^ 1u, ctx)) { ok = false; break; }
        S.item_slot[ps][0] = idx;
        S.item_slot[ps][1] = ntile;
        S.item[ps] = it;
        mbar_arrive_expect_tx(&S.qfull[ps], 2u * 128u * static_cast<uint32_t>(p.q_box_rows));
        tma_load_3d(S.q[ps][0], &tmap_q, &S.qfull[ps], 0, it.h * p.g, it.row);
        tma_load_3d(S.q[ps][1], &tmap_q, &S.qfull[ps], 64, it.h * p.g, it.row);
        const int claim_j = max(0, ntile - 3), read_j = max(0, ntile - 2);
        for (int j = 0; j < ntile; ++j, ++J) {
          if (j == claim_j) nidx = atomicAdd(&p.hdr->dec_counter, 1);
          if constexpr (paged) {
            // the page-id load below needs the next item before this tile's copies
            if (j == read_j && nidx < n_items) {
              nit = fused ? fused_item(nidx) : p.items[nidx];
              have_next = true;
            }
          }
          const int st = J % kStages;
          const uint32_t free_parity = ((J / kStages) & 1u) ^ 1u;
          const int t = it.t0 + j * kTcKeys;
          const int valid = max(0, min(kTcKeys, it.t1 - t));
          int32_t id_big = -1;
          if constexpr (paged) {
            // this tile's page (loaded an iteration ago); start loading the next tile's
            id_big = have_pre ? id_pre : tile_page_id(p, it.b, t);
            have_pre = true;
            if (j + 1 < ntile) id_pre = tile_page_id(p, it.b, t + kTcKeys);
            else if (have_next) id_pre = tile_page_id(p, nit.b, nit.t0);
            else have_pre = false;
          }
          if (!mbar_wait(&S.kempty[st], free_parity, ctx)) { ok = false; break; }
          if constexpr (paged) {
            // hand the id to the V producer: the slot's previous tile has been released
            const int slot = J % kPidSlots;
            if (!mbar_wait(&S.pidempty[slot], ((J / kPidSlots) & 1u) ^ 1u, ctx)) { ok = false; break; }
            S.pid[slot][0] = id_big;
            mbar_arrive(&S.pidfull[slot]);
          }
          S.meta[st][0] = t;
          S.meta[st][1] = valid;
          uint64_t* kbar = &S.kfull[st];  // the copy completes kfull (E4M3: the codes as they are)
          if (valid > 0) {
            if constexpr (paged) {
              mbar_arrive_expect_tx(kbar, kRowBytes * kTcKeys);
              load_tile_page1<kF8>(S.k[st][0], S.k[st][Smem::kKSlabs - 1], &tmap_k, kbar, id_big,
                                   t % p.page_size, p, it.h, pol);
            } else {
              mbar_arrive_expect_tx(kbar, kRowBytes * static_cast<uint32_t>(p.kv_box_rows));
              tma_load_4d_stream(S.k[st][0], &tmap_k, kbar, 0, t, it.h, it.b, pol);
              if constexpr (!kF8)
                tma_load_4d_stream(S.k[st][Smem::kKSlabs - 1], &tmap_k, kbar, 64, t, it.h, it.b, pol);
            }
          } else {
            mbar_arrive(kbar);
          }
          if constexpr (!paged) {
            if (j == read_j && nidx < n_items) nit = fused ? fused_item(nidx) : p.items[nidx];
          }
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
        // let copies already issued land before shared memory is released
        for (uint32_t back = 1; back <= kStages && back <= J; ++back) {
          const uint32_t jj = J - back;
          mbar_drain(&S.kfull[jj % kStages], (jj / kStages) & 1u);
        }
      }
    }
    __syncwarp();
  } else if (warp == kVProducerWarp && kMode == kSmallPages) {
    // ============ TMA producer of V, pages of < 128 keys (whole warp, as the K producer) ============
    const int pshift = __ffs(p.page_size) - 1;
    const uint64_t pol = l2_evict_first_policy();
    uint32_t J = 0, K = 0;
    bool ok = true;
    while (ok) {
      const int ps = K & 1;
      if (!warp_mbar_wait(&S.qfull[ps], (K >> 1) & 1u, ctx)) { ok = false; break; }
      const int idx = S.item_slot[ps][0];
      const int ntile = S.item_slot[ps][1];
      const DecodeItem it = S.item[ps];
      __syncwarp();
      if (lane == 0) mbar_arrive(&S.qempty[ps]);
      if (idx < 0) break;
      for (int j = 0; j < ntile; ++j, ++J) {
        const int st = J % kVStages;
        const int t = it.t0 + j * kTcKeys;
        const int valid = max(0, min(kTcKeys, it.t1 - t));
        if (!warp_mbar_wait(&S.vempty[st], ((J / kVStages) & 1u) ^ 1u, ctx)) { ok = false; break; }
        if (!warp_mbar_wait(&S.pidfull[J % kPidSlots], (J / kPidSlots) & 1u, ctx)) { ok = false; break; }
        const SmallPages sp = small_pages(t, valid, pshift);
        uint64_t* vbar = kF8 ? &S.vraw[st] : &S.vfull[st];
        if (lane == 0) {
          if constexpr (kF8) S.vmeta[st] = valid;
          if (valid > 0) mbar_arrive_expect_tx(vbar, small_pages_bytes<kF8>(sp, p));
          else mbar_arrive(vbar);
        }
        __syncwarp();
        if (valid > 0)
          load_small_pages<kF8>(S.v[st][kF8 ? 1 : 0], S.v[st][1], &tmap_v, vbar, sp,
                                S.pid[J % kPidSlots], p, it.h, valid, pol, lane);
        __syncwarp();  // every lane has read its page id: the slot is free
        if (lane == 0) mbar_arrive(&S.pidempty[J % kPidSlots]);
      }
      ++K;
    }
    if (lane == 0) {
      if constexpr (kF8) {
        // stop marker for the V expanding warps (a stage without a tile)
        const int st = J % kVStages;
        if (ok && mbar_wait(&S.vempty[st], ((J / kVStages) & 1u) ^ 1u, ctx)) {
          S.vmeta[st] = -1;
          mbar_arrive(&S.vraw[st]);
        }
      }
      if (S.abort_flag) {
        for (uint32_t back = 1; back <= kVStages && back <= J; ++back) {
          const uint32_t jj = J - back;
          mbar_drain(kF8 ? &S.vraw[jj % kVStages] : &S.vfull[jj % kVStages], (jj / kVStages) & 1u);
        }
      }
    }
    __syncwarp();
  } else if (kMode != kSmallPages && warp == kVProducerWarp) {
    // ======================= TMA producer of V =======================
    // Follows the items the Q/K producer publishes; a V stage is refilled once the P·V product
    // of its previous tile has completed, independently of the K half.
    if (lane == 0) {
      const uint64_t pol = l2_evict_first_policy();
      const uint32_t tx = kRowBytes * static_cast<uint32_t>(p.kv_box_rows);
      uint32_t J = 0, K = 0;
      bool ok = true;
      while (ok) {
        const int ps = K & 1;
        if (!mbar_wait(&S.qfull[ps], (K >> 1) & 1u, ctx)) { ok = false; break; }
        const int idx = S.item_slot[ps][0];
        const int ntile = S.item_slot[ps][1];
        const DecodeItem it = S.item[ps];
        mbar_arrive(&S.qempty[ps]);
        if (idx < 0) break;
        for (int j = 0; j < ntile; ++j, ++J) {
          const int st = J % kVStages;
          const int t = it.t0 + j * kTcKeys;
          const int valid = max(0, min(kTcKeys, it.t1 - t));
          if (!mbar_wait(&S.vempty[st], ((J / kVStages) & 1u) ^ 1u, ctx)) { ok = false; break; }
          if constexpr (paged) {
            if (!mbar_wait(&S.pidfull[J % kPidSlots], (J / kPidSlots) & 1u, ctx)) { ok = false; break; }
          }
          uint64_t* vbar = kF8 ? &S.vraw[st] : &S.vfull[st];
          if constexpr (kF8) S.vmeta[st] = valid;
          if (valid > 0) {
            if constexpr (paged) {
              mbar_arrive_expect_tx(vbar, kRowBytes * kTcKeys);
              load_tile_page1<kF8>(S.v[st][kF8 ? 1 : 0], S.v[st][1], &tmap_v, vbar,
                                   S.pid[J % kPidSlots][0], t % p.page_size, p, it.h, pol);
            } else {
              mbar_arrive_expect_tx(vbar, tx);
              if constexpr (kF8) {
                tma_load_4d_stream(S.v[st][1], &tmap_v, vbar, 0, t, it.h, it.b, pol);
              } else {
                tma_load_4d_stream(S.v[st][0], &tmap_v, vbar, 0, t, it.h, it.b, pol);
                tma_load_4d_stream(S.v[st][1], &tmap_v, vbar, 64, t, it.h, it.b, pol);
              }
            }
          } else {
            mbar_arrive(vbar);
          }
          if constexpr (paged) mbar_arrive(&S.pidempty[J % kPidSlots]);  // ids read: slot free
        }
        ++K;
      }
      if constexpr (kF8) {
        // stop marker for the V expanding warps (a stage without a tile)
        const int st = J % kVStages;
        if (ok && mbar_wait(&S.vempty[st], ((J / kVStages) & 1u) ^ 1u, ctx)) {
          S.vmeta[st] = -1;
          mbar_arrive(&S.vraw[st]);
        }
      }
      if (S.abort_flag) {
        for (uint32_t back = 1; back <= kVStages && back <= J; ++back) {
          const uint32_t jj = J - back;
          mbar_drain(kF8 ? &S.vraw[jj % kVStages] : &S.vfull[jj % kVStages], (jj / kVStages) & 1u);
        }
      }
    }
    __syncwarp();
  } else if (warp == kMmaWarp) {
    // ======================= Sᵀ issuer =======================
    if (lane == 0) {
      const uint32_t idesc_s = kF8 ? idesc_e4m3_f32(kTcKeys, 16) : idesc_bf16_f32(kTcKeys, 16, false, false);
      uint32_t J = 0, K = 0;
      bool ok = true;
      while (ok) {
        const int ps = K & 1;
        if (!mbar_wait(&S.qfull[ps], (K >> 1) & 1u, ctx)) { ok = false; break; }
        const int idx = S.item_slot[ps][0];
        const int ntile = S.item_slot[ps][1];
        if (idx < 0) break;
        const uint32_t qaddr0 = smem_u32(S.q[ps][0]);
        const uint32_t qaddr1 = smem_u32(S.q[ps][1]);
        // E4M3 cache: the item's Q terms, from the Q warps
        if (kF8 && !mbar_wait(&S.q8full[ps], (K >> 1) & 1u, ctx)) { ok = false; break; }
        for (int j = 0; j < ntile; ++j, ++J) {
          const int st = J % kStages;
          const int sb = J & 1;
          if (!mbar_wait(&S.kfull[st], (J / kStages) & 1u, ctx)) { ok = false; break; }
          if (!mbar_wait(&S.sempty[sb], ((J >> 1) & 1u) ^ 1u, ctx)) { ok = false; break; }
          tc_fence_after();
          const int valid = S.meta[st][1];
          if (valid > 0) {
            if constexpr (kF8 && kMode == kContiguous) {
              // A = the tile's K codes, B = the Q terms: 32 codes (32 bytes) of D per product.
              // The descriptors are built once per tile (a 32-byte step is 2 in the start-address
              // field; shared addresses stay below 2^18 bytes, so it never carries).
              const uint64_t kd = smem_desc(smem_u32(S.k[st][0]), 16, 1024, kLayoutSW128);
              const uint64_t qd = smem_desc(smem_u32(S.q8[ps]), 16, 1024, kLayoutSW128);
#pragma unroll
              for (int kk = 0; kk < kTcD / 32; ++kk)
                umma_f8_ss(tmem + sb * 16, kd + static_cast<uint64_t>(kk * 2),
                           qd + static_cast<uint64_t>(kk * 2), idesc_s, kk > 0 ? 1u : 0u);
            } else if constexpr (kF8) {
              const uint32_t ka = smem_u32(S.k[st][0]);
              const uint32_t qa = smem_u32(S.q8[ps]);
#pragma unroll
              for (int kk = 0; kk < kTcD / 32; ++kk)
                umma_f8_ss(tmem + sb * 16, smem_desc(ka + kk * 32, 16, 1024, kLayoutSW128),
                           smem_desc(qa + kk * 32, 16, 1024, kLayoutSW128), idesc_s, kk > 0 ? 1u : 0u);
            } else if constexpr (kMode == kSmallPages) {
              // descriptors built once per tile, as above; the interleaved layout has the second
              // half 1024 bytes after the first and 8-row groups 2048 bytes apart
              const uint32_t kil = p.pg_interleave ? 1u : 0u;
              const uint32_t kbase = smem_u32(S.k[st][0]);
              const uint64_t kd[2] = {smem_desc(kbase, 16, 1024u << kil, kLayoutSW128),
                                      smem_desc(kil ? kbase + 1024u : smem_u32(S.k[st][Smem::kKSlabs - 1]), 16,
                                                1024u << kil, kLayoutSW128)};
              const uint64_t qd[2] = {smem_desc(qaddr0, 16, 1024, kLayoutSW128),
                                      smem_desc(qaddr1, 16, 1024, kLayoutSW128)};
#pragma unroll
              for (int kk = 0; kk < kTcD / 16; ++kk)
                umma_bf16_ss(tmem + sb * 16, kd[kk >> 2] + static_cast<uint64_t>((kk & 3) * 2),
                             qd[kk >> 2] + static_cast<uint64_t>((kk & 3) * 2), idesc_s, kk > 0 ? 1u : 0u);
            } else {
              const uint32_t k0 = smem_u32(S.k[st][0]);
              const uint32_t k1 = smem_u32(S.k[st][Smem::kKSlabs - 1]);
#pragma unroll
              for (int kk = 0; kk < kTcD / 16; ++kk) {
                const uint32_t ka = (kk < 4 ? k0 : k1) + (kk & 3) * 32;
                const uint32_t qa = (kk < 4 ? qaddr0 : qaddr1) + (kk & 3) * 32;
                umma_bf16_ss(tmem + sb * 16, smem_desc(ka, 16, 1024, kLayoutSW128),
                             smem_desc(qa, 16, 1024, kLayoutSW128), idesc_s, kk > 0 ? 1u : 0u);
              }
            }
          }
          umma_commit(&S.sfull[sb]);
          umma_commit(&S.kempty[st]);
          if (j == ntile - 1) umma_commit(&S.qempty[ps]);
        }
        if (!ok) break;
        ++K;
      }
      // every MMA this thread issued has completed once `drain` flips
      umma_commit(&S.drain);
      mbar_drain(&S.drain, 0);
    }
    __syncwarp();
  } else if (warp == kPvWarp) {
    // ======================= P·V issuer =======================
    // Follows the items the Q/K producer publishes. O of an item accumulates in the item
    // parity's columns; its first product overwrites them once the epilogue has read the item
    // two back.
    if (lane == 0) {
      const uint32_t idesc_o = kF8 ? idesc_f16_f32(kTcD, kNO, true, true)
                                   : idesc_bf16_f32(kTcD, kNO, true, true);
      uint32_t J = 0, K = 0;
      bool ok = true;
      while (ok) {
        const int ps = K & 1;
        if (!mbar_wait(&S.qfull[ps], (K >> 1) & 1u, ctx)) { ok = false; break; }
        const int idx = S.item_slot[ps][0];
        const int ntile = S.item_slot[ps][1];
        const DecodeItem it = S.item[ps];
        mbar_arrive(&S.qempty[ps]);
        if (idx < 0) break;
        const int ob = K & 1;
        for (int j = 0; j < ntile; ++j, ++J) {
          const int st = J % kVStages;
          const int pb = J & 1;
          const int valid = max(0, min(kTcKeys, it.t1 - (it.t0 + j * kTcKeys)));
          if (!mbar_wait(&S.vfull[st], (J / kVStages) & 1u, ctx)) { ok = false; break; }
          if (!mbar_wait(&S.pfull[pb], (J >> 1) & 1u, ctx)) { ok = false; break; }
          if (j == 0 && !mbar_wait(&S.oempty[ob], ((K >> 1) & 1u) ^ 1u, ctx)) { ok = false; break; }
          tc_fence_after();
          const int nk = (valid + 15) / 16;
          const uint32_t vaddr = smem_u32(S.v[st][0]);
          const uint32_t paddr = smem_u32(S.p[pb]);
          if constexpr ((kF8 && kMode == kContiguous) || (!kF8 && kMode == kSmallPages)) {
            // Descriptors built once per tile (16 keys a step: 2048 bytes of V, 128 in the
            // start-address field, and 256 of P, 16), and for a contiguous E4M3 cache a full
            // tile's products unrolled. Measured A/B at the 70B-like shape: E4M3 268 -> 258 us,
            // 16-key pages 411 -> 399 us; the contiguous bf16 kernel did not change and the
            // 128-key-page E4M3 kernel slowed (363 -> 389 us), so those keep the plain loop.
            // V of 16-key pages in the interleaved layout: halves 1024 bytes apart (LBO), 8-key
            // groups 2048 (SBO), so 16 keys a step are 4096 bytes (256 in the field)
            const uint32_t vil = (kMode == kSmallPages && p.pg_interleave) ? 1u : 0u;
            const uint64_t ad0 = smem_desc(vaddr, vil ? 1024u : kHalfBytes, 1024u << vil, kLayoutSW128);
            const uint64_t bd0 = smem_desc(paddr, 128, 2048, kLayoutNone);
            const uint32_t dcol = tmem + kColO + ob * kNO;
            const uint32_t acc = j > 0 ? 1u : 0u;
            const uint32_t vstep = 128u << vil;
            if (kF8 && kMode == kContiguous && nk == kTcKeys / 16) {
#pragma unroll
              for (int kk = 0; kk < kTcKeys / 16; ++kk)
                umma_bf16_ss(dcol, ad0 + static_cast<uint64_t>(kk * 128), bd0 + static_cast<uint64_t>(kk * 16),
                             idesc_o, kk > 0 ? 1u : acc);
            } else {
              for (int kk = 0; kk < nk; ++kk)
                umma_bf16_ss(dcol, ad0 + static_cast<uint64_t>(kk * vstep), bd0 + static_cast<uint64_t>(kk * 16),
                             idesc_o, kk > 0 ? 1u : acc);
            }
          } else {
            for (int kk = 0; kk < nk; ++kk) {
              const uint64_t ad = smem_desc(vaddr + kk * 2048, kHalfBytes, 1024, kLayoutSW128);
              const uint64_t bd = smem_desc(paddr + kk * 256, 128, 2048, kLayoutNone);
              umma_bf16_ss(tmem + kColO + ob * kNO, ad, bd, idesc_o, (j == 0 && kk == 0) ? 0u : 1u);
            }
          }
          umma_commit(&S.ofull[pb]);
          if (j == ntile - 1) umma_commit(&S.ofin[ob]);
          umma_commit(&S.pempty[pb]);
          umma_commit(&S.vempty[st]);
        }
        if (!ok) break;
        ++K;
      }
      umma_commit(&S.drain_pv);
      mbar_drain(&S.drain_pv, 0);
    }
    __syncwarp();
  } else if (warp < 4) {
    // ======================= softmax and O correction =======================
    // A timed-out wait never makes one of these warps leave on its own: the others would wait
    // for it at a named barrier, which has no time limit. Each warp notes the failure in `ok`,
    // skips the work that depended on the wait and keeps meeting the barriers; the barriers
    // themselves vote on the failure, so all four warps leave at the same point.
    const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
    float m[GPAD], lp[GPAD];
    uint32_t J = 0, K = 0;
    bool ok = true;
    // O of the current item (thread = d lane): columns [0, GPAD) the P_hi part, [GPAD, 2 GPAD)
    // the P_lo part
    auto load_o = [&](uint32_t ob, uint32_t (&r)[kNO]) {
      if constexpr (kNO == 16) tmem_ld16(tmem + lane_base + kColO + ob * kNO, r);
      else tmem_ld32(tmem + lane_base + kColO + ob * kNO, r);
      tmem_wait_ld();
    };
    for (;;) {
      const int ps = K & 1;
      ok = ok && mbar_wait(&S.qfull[ps], (K >> 1) & 1u, ctx);
      if (named_bar_or(1, kSoftmaxThreads, !ok)) break;
      const int idx = S.item_slot[ps][0];
      const int ntile = S.item_slot[ps][1];
      const DecodeItem it = S.item[ps];
      // E4M3 cache: each head's score factor 2^e * scale (read before the Q slot is released)
      float qs[GPAD];
      if constexpr (kF8) {
        if (idx >= 0) ok = ok && mbar_wait(&S.q8full[ps], (K >> 1) & 1u, ctx);
        if (named_bar_or(1, kSoftmaxThreads, !ok)) break;
#pragma unroll
        for (int g = 0; g < GPAD; ++g) qs[g] = S.qscale[ps][g] * p.scale_log2;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&S.qempty[ps]);
      const uint32_t ob = K & 1;
      if (idx < 0) {
        // tell the epilogue warps to stop
        if (mbar_wait(&S.lfree[ob], ((K >> 1) & 1u) ^ 1u, ctx)) {
          if (tid == 0) S.epi[ob][0] = -1;
          __syncwarp();
          if (lane == 0) mbar_arrive(&S.lready[ob]);
        }
        break;
      }
#pragma unroll
      for (int g = 0; g < GPAD; ++g) { m[g] = -INFINITY; lp[g] = 0.f; }
      bool abort_item = false;
      for (int j = 0; j < ntile; ++j, ++J) {
        const int st = J % kVStages;
        const int sb = J & 1;
        ok = ok && mbar_wait(&S.sfull[sb], (J >> 1) & 1u, ctx);
        tc_fence_after();
        // Keys of this tile, from the item descriptor. (Not from the stage's kfull barrier: K is
        // released as soon as Sᵀ has read it, so kfull may already be a phase further on.)
        const int valid = max(0, min(kTcKeys, it.t1 - (it.t0 + j * kTcKeys)));
        uint32_t sr[16];
        if (ok && valid > 0) {
          tmem_ld16(tmem + lane_base + sb * 16, sr);
          tmem_wait_ld();
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0 && ok) mbar_arrive(&S.sempty[sb]);

        const bool in = ok && tid < valid;
        float x[GPAD];
        bool grow = false;
#pragma unroll
        for (int g = 0; g < GPAD; ++g) {
          if constexpr (kF8)  // the two Q terms' columns, then the head's factor
            x[g] = (in && g < p.g) ? (__uint_as_float(sr[g]) + __uint_as_float(sr[8 + g])) * qs[g] : -INFINITY;
          else
            x[g] = (in && g < p.g) ? __uint_as_float(sr[g]) * p.scale_log2 : -INFINITY;
          grow |= x[g] > m[g] + kRescaleThreshold;
        }
        // One barrier per tile, which also tells every thread whether any key of the tile lies
        // more than the threshold above the running maximum (always so on an item's first tile)
        // or whether a wait has failed.
        if (named_bar_or(1, kSoftmaxThreads, grow || !ok)) {
          // exact new maximum over the 128 keys, per query head
#pragma unroll
          for (int g = 0; g < GPAD; ++g) {
            const float wm = warp_max_f32(x[g]);
            if (lane == 0) S.wmax[sb][warp][g] = wm;
          }
          if (named_bar_or(1, kSoftmaxThreads, !ok)) { abort_item = true; break; }
          float alpha[GPAD];
#pragma unroll
          for (int g = 0; g < GPAD; ++g) {
            const float tmx = fmaxf(fmaxf(S.wmax[sb][0][g], S.wmax[sb][1][g]),
                                    fmaxf(S.wmax[sb][2][g], S.wmax[sb][3][g]));
            const float mn = fmaxf(m[g], tmx);
            alpha[g] = (m[g] == -INFINITY) ? 0.f : fast_exp2(m[g] - mn);
            lp[g] *= alpha[g];
            m[g] = mn;
          }
          if (j > 0) {
            // O holds the item's earlier tiles: wait for the last of their products, scale it
            const uint32_t jp = J - 1;
            ok = ok && mbar_wait(&S.ofull[jp & 1], (jp >> 1) & 1u, ctx);
            tc_fence_after();
            if (ok) {
              uint32_t o[kNO];
              load_o(ob, o);
#pragma unroll
              for (int g = 0; g < GPAD; ++g) {
                o[g] = __float_as_uint(__uint_as_float(o[g]) * alpha[g]);
                o[GPAD + g] = __float_as_uint(__uint_as_float(o[GPAD + g]) * alpha[g]);
              }
              if constexpr (kNO == 16) tmem_st16(tmem + lane_base + kColO + ob * kNO, o);
              else tmem_st32(tmem + lane_base + kColO + ob * kNO, o);
              tmem_wait_st();
            }
          }
        }
        float pr[GPAD];
#pragma unroll
        for (int g = 0; g < GPAD; ++g) {
          pr[g] = (m[g] == -INFINITY) ? 0.f : fast_exp2(x[g] - m[g]);
          lp[g] += pr[g];
        }
        // P_hi / P_lo for this key lane (f16 in the E4M3 instantiation, whose V is f16)
        uint32_t hw[GPAD / 2], lw[GPAD / 2];
#pragma unroll
        for (int g = 0; g < GPAD; g += 2) {
          if constexpr (kF8) {
            const __half2 h2 = __floats2half2_rn(pr[g], pr[g + 1]);
            const float2 hf = __half22float2(h2);
            const __half2 l2 = __floats2half2_rn(pr[g] - hf.x, pr[g + 1] - hf.y);
            hw[g / 2] = *reinterpret_cast<const uint32_t*>(&h2);
            lw[g / 2] = *reinterpret_cast<const uint32_t*>(&l2);
          } else {
            const __nv_bfloat162 h2 = __floats2bfloat162_rn(pr[g], pr[g + 1]);
            const float2 hf = __bfloat1622float2(h2);
            const __nv_bfloat162 l2 = __floats2bfloat162_rn(pr[g] - hf.x, pr[g + 1] - hf.y);
            hw[g / 2] = *reinterpret_cast<const uint32_t*>(&h2);
            lw[g / 2] = *reinterpret_cast<const uint32_t*>(&l2);
          }
        }
        ok = ok && mbar_wait(&S.pempty[sb], ((J >> 1) & 1u) ^ 1u, ctx);
        if (!kF8 && (valid & 15) != 0) {
          // zero V rows [valid, next multiple of 16): they may lie past the sequence end (the
          // expanding warps of an E4M3 cache write those rows as zeros themselves)
          ok = ok && mbar_wait(&S.vfull[st], (J / kVStages) & 1u, ctx);
          const int r0 = valid, r1 = (valid + 15) & ~15;
          const int nchunks = (r1 - r0) * 2 * 8;
          const bool vil = kMode == kSmallPages && p.pg_interleave;
          for (int c = tid; ok && c < nchunks; c += kSoftmaxThreads) {
            const int row = r0 + c / 16;
            const int half = (c / 8) & 1;
            const int ch = c & 7;
            // byte offset of the row's half from the stage start (interleaved: see load_small_pages)
            const int off = vil ? (row >> 3) * 2048 + half * 1024 + (row & 7) * 128
                                : half * static_cast<int>(kHalfBytes) + row * 128;
            *reinterpret_cast<uint4*>(reinterpret_cast<unsigned char*>(S.v[st][0]) + off + ch * 16) =
                make_uint4(0u, 0u, 0u, 0u);
          }
        }
        if (ok) {
          unsigned char* pb = reinterpret_cast<unsigned char*>(S.p[sb]);
#pragma unroll
          for (int grp = 0; grp < GPAD / 8; ++grp) {
            *reinterpret_cast<uint4*>(pb + grp * 2048 + tid * 16) =
                make_uint4(hw[grp * 4 + 0], hw[grp * 4 + 1], hw[grp * 4 + 2], hw[grp * 4 + 3]);
            *reinterpret_cast<uint4*>(pb + (GPAD / 8 + grp) * 2048 + tid * 16) =
                make_uint4(lw[grp * 4 + 0], lw[grp * 4 + 1], lw[grp * 4 + 2], lw[grp * 4 + 3]);
          }
        }
        fence_proxy_async_smem();
        tc_fence_before();  // orders a rescale's tcgen05.st before the P·V product
        __syncwarp();
        if (lane == 0 && ok) mbar_arrive(&S.pfull[sb]);
      }
      if (abort_item) break;

      // ---- hand the item to the epilogue warps: per-warp sums of l, the running max ----
      ok = ok && mbar_wait(&S.lfree[ob], ((K >> 1) & 1u) ^ 1u, ctx);
#pragma unroll
      for (int g = 0; g < GPAD; ++g) {
        const float sum = warp_sum_f32(lp[g]);
        if (lane == 0 && ok) S.lred[ob][warp][g] = sum;
      }
      if (tid == 0 && ok) {
#pragma unroll
        for (int g = 0; g < GPAD; ++g) S.mfin[ob][g] = m[g];
        S.epi[ob][0] = it.row;
        S.epi[ob][1] = it.h;
        S.epi[ob][2] = it.nsplit;
        S.epi[ob][3] = it.slot;
      }
      __syncwarp();
      if (lane == 0 && ok) mbar_arrive(&S.lready[ob]);
      ++K;
    }
  } else if (warp >= kConvWarp0) {
    if constexpr (kF8) {
      // ================ E4M3 cache: Q terms (warps 12-15), V expansion (16-19) ================
      if (warp < kConvWarp0 + 4) {
        // Per item, Q (bf16, SW128, 16 head rows) becomes two E4M3 terms per head for the Sᵀ
        // product: thread ct handles 8 consecutive d of head ct / 16. Rows 0-7 of q8 take c1, rows
        // 8-15 c2, in the 128-byte swizzle of a K-major operand of one-byte elements.
        const int ct = tid - kConvWarp0 * 32;
        const int hd = ct >> 4;
        const int d0 = (ct & 15) * 8;
        for (uint32_t K = 0;; ++K) {
          const int ps = K & 1;
          if (!mbar_wait(&S.qfull[ps], (K >> 1) & 1u, ctx)) break;
          const int idx = S.item_slot[ps][0];
          if (idx < 0) {
            __syncwarp();
            if (lane == 0) mbar_arrive(&S.qempty[ps]);
            break;
          }
          const unsigned char* qrow = reinterpret_cast<const unsigned char*>(S.q[ps][d0 >> 6]) + hd * 128;
          const uint4 raw = *reinterpret_cast<const uint4*>(qrow + ((((d0 & 63) >> 3) ^ (hd & 7)) << 4));
          float x[8];
          {
            const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              x[2 * i] = __uint_as_float(w[i] << 16);
              x[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
            }
          }
          float mx = 0.f;
#pragma unroll
          for (int i = 0; i < 8; ++i) mx = fmaxf(mx, fabsf(x[i]));
#pragma unroll
          for (int o = 8; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
          // e with the head's largest |q| / 2^e in [128, 256) (a power of two: the scaling is
          // exact); an all-zero head (or one below 2^-100) gets e = 0 and zero terms
          int e = 0;
          if (mx >= 0x1p-100f) e = static_cast<int>((__float_as_uint(mx) >> 23) & 0xffu) - 127 - 7;
          const float inv = __uint_as_float(static_cast<uint32_t>(127 - e) << 23);  // 2^-e
          uint32_t c1w[2], c2w[2];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const float a = x[2 * i] * inv, b = x[2 * i + 1] * inv;
            uint16_t c1, c2;
            uint32_t h1;
            // c1 = E4M3(a, b) (a in the low byte), back to f16 pairs, residual, c2 = E4M3(residual)
            asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(c1) : "f"(b), "f"(a));
            asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h1) : "h"(c1));
            __half2 h2;
            memcpy(&h2, &h1, 4);
            const float2 f = __half22float2(h2);
            asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(c2) : "f"(b - f.y), "f"(a - f.x));
            const uint32_t sh = (i & 1) * 16;
            if ((i & 1) == 0) {
              c1w[i >> 1] = 0u;
              c2w[i >> 1] = 0u;
            }
            c1w[i >> 1] |= static_cast<uint32_t>(c1) << sh;
            c2w[i >> 1] |= static_cast<uint32_t>(c2) << sh;
          }
          // 8 codes at d0 of rows hd (c1) and 8 + hd (c2): half of the 16-byte chunk d0 / 16
          const int r1 = hd, r2 = 8 + hd;
          unsigned char* q8 = S.q8[ps];
          *reinterpret_cast<uint2*>(q8 + r1 * 128 + ((((d0 >> 4) ^ (r1 & 7)) << 4) | (d0 & 15))) =
              make_uint2(c1w[0], c1w[1]);
          *reinterpret_cast<uint2*>(q8 + r2 * 128 + ((((d0 >> 4) ^ (r2 & 7)) << 4) | (d0 & 15))) =
              make_uint2(c2w[0], c2w[1]);
          if ((ct & 15) == 0) S.qscale[ps][hd] = __uint_as_float(static_cast<uint32_t>(127 + e) << 23);
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            mbar_arrive(&S.q8full[ps]);
            mbar_arrive(&S.qempty[ps]);
          }
        }
      } else {
        const int ct = tid - (kConvWarp0 + 4) * 32;
        for (uint32_t J = 0;; ++J) {
          const int st = J % kVStages;
          if (!mbar_wait(&S.vraw[st], (J / kVStages) & 1u, ctx)) break;
          const int valid = S.vmeta[st];
          if (valid < 0) break;
          expand_v_tile(S.v[st], ct, valid);
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) mbar_arrive(&S.vfull[st]);
        }
      }
    }
  } else {
    // ======================= epilogue: O = (O_hi + O_lo) / l =======================
    // Runs while the softmax warps already work on the next item; its O accumulator is the other
    // item parity's, so the two never touch the same columns.
    const int quad = warp & 3;
    const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
    const int d = quad * 32 + lane;
    for (uint32_t K = 0;; ++K) {
      const uint32_t ob = K & 1;
      if (!mbar_wait(&S.lready[ob], (K >> 1) & 1u, ctx)) break;
      const int row = S.epi[ob][0];
      if (row < 0) break;
      const int h = S.epi[ob][1];
      const bool direct = S.epi[ob][2] == 1;
      const int64_t slot = direct ? 0 : static_cast<int64_t>(S.epi[ob][3]);
      float mf[GPAD], l[GPAD];
#pragma unroll
      for (int g = 0; g < GPAD; ++g) {
        mf[g] = S.mfin[ob][g];
        l[g] = S.lred[ob][0][g] + S.lred[ob][1][g] + S.lred[ob][2][g] + S.lred[ob][3][g];
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&S.lfree[ob]);
      if (!mbar_wait(&S.ofin[ob], (K >> 1) & 1u, ctx)) break;
      tc_fence_after();
      uint32_t o[kNO];
      if constexpr (kNO == 16) tmem_ld16(tmem + lane_base + kColO + ob * kNO, o);
      else tmem_ld32(tmem + lane_base + kColO + ob * kNO, o);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&S.oempty[ob]);
#pragma unroll
      for (int g = 0; g < GPAD; ++g) {
        if (g < p.g) {
          const float acc = __uint_as_float(o[g]) + __uint_as_float(o[GPAD + g]);
          const float ov = l[g] > 0.f ? acc / l[g] * p.v_scale : 0.f;
          const float lse2 = l[g] > 0.f ? mf[g] + log2f(l[g]) : -INFINITY;
          const int hq = h * p.g + g;
          if (direct) {
            __nv_bfloat16* out = static_cast<__nv_bfloat16*>(p.out) +
                                 static_cast<int64_t>(row) * p.o_sr + static_cast<int64_t>(hq) * p.o_sh;
            out[d] = __float2bfloat16_rn(ov);
            if (d == 0) p.lse[static_cast<int64_t>(row) * p.hq + hq] = lse2 * kLn2;
          } else {
            p.part_o[(slot * p.g + g) * kTcD + d] = ov;
            if (d == 0) p.part_lse[slot * p.g + g] = lse2;
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kMmaWarp) tmem_dealloc(tmem, kCols);
  if (tid == 0) release_work_cursor(&p.hdr->dec_counter, &p.hdr->dec_exit);
}

template <int GPAD, int kMode, bool kF8 = false>
cudaError_t launch_tc_t(const DecodeParams& p, const CUtensorMap& tq, const CUtensorMap& tk,
                        const CUtensorMap& tv, int nctas, cudaStream_t stream) {
  const size_t smem = sizeof(TcSmem<GPAD, kF8>) + 1024;
  cudaError_t e = cudaFuncSetAttribute(decode_tc_kernel<GPAD, kMode, kF8>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(nctas);
  cfg.blockDim = dim3(kF8 ? kF8Threads : kTcThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, decode_tc_kernel<GPAD, kMode, kF8>, p, tq, tk, tv);
}

}  // namespace

cudaError_t launch_decode_tc(const DecodeParams& p, const CUtensorMap& tmap_q,
                             const CUtensorMap& tmap_k, const CUtensorMap& tmap_v, int nctas,
                             cudaStream_t stream) {
  const int mode = p.block_table == nullptr ? kContiguous
                   : (p.page_size >= kTcKeys ? kBigPages : kSmallPages);
  if (p.kv_fp8) {
    if (p.g > 8) return cudaErrorInvalidValue;
    if (mode == kContiguous) return launch_tc_t<8, kContiguous, true>(p, tmap_q, tmap_k, tmap_v, nctas, stream);
    if (mode == kBigPages) return launch_tc_t<8, kBigPages, true>(p, tmap_q, tmap_k, tmap_v, nctas, stream);
    return launch_tc_t<8, kSmallPages, true>(p, tmap_q, tmap_k, tmap_v, nctas, stream);
  }
  if (p.g <= 8) {
    if (mode == kContiguous) return launch_tc_t<8, kContiguous>(p, tmap_q, tmap_k, tmap_v, nctas, stream);
    if (mode == kBigPages) return launch_tc_t<8, kBigPages>(p, tmap_q, tmap_k, tmap_v, nctas, stream);
    return launch_tc_t<8, kSmallPages>(p, tmap_q, tmap_k, tmap_v, nctas, stream);
  }
  if (mode == kContiguous) return launch_tc_t<16, kContiguous>(p, tmap_q, tmap_k, tmap_v, nctas, stream);
  if (mode == kBigPages) return launch_tc_t<16, kBigPages>(p, tmap_q, tmap_k, tmap_v, nctas, stream);
  return launch_tc_t<16, kSmallPages>(p, tmap_q, tmap_k, tmap_v, nctas, stream);
}

}  // namespace fd
