// Chunked-prefill attention tiles on the 5th-generation tensor cores (tcgen05 + TMEM).
//
// A work item is one key split [k0, k1) of one 128-row query tile of one query head of a chunk
// request ("大语言模型长序列推理优化：ChunkedPrefill与FlashDecoding技术解析" §2.1: the chunk's K/V
// are already in the cache; its queries attend to the whole cache under a causal mask; the
// prefix may be a reused cache, "Chunked-Prefills分块预填充机制：破解大模型推理的吞吐与延迟困局"
// §三.2). Row r of the tile is chunk position pos0 + r and sees keys j <= prefix + pos0 + r.
// Per 128-key tile of the split:
//
//   S[128 rows x 128 keys] = Q_tile · K_tileᵀ         UMMA M=128 N=128, both K-major (TMA SW128)
//   one thread per row: mask, running max m (rescaled lazily), p = 2^(s·scale·log2e − m),
//   running sum l, P split into bf16 hi + lo and stored into tensor memory
//   O[128 x 128] += P_hi · V_tile + P_lo · V_tile      UMMA M=128 N=128, A from TMEM, V MN-major
//
// S is double-buffered in TMEM and P is written back over the S buffer it came from (per
// 32-key chunk: 16 words of hi pairs, then 16 words of lo pairs, so a chunk's writes only cover
// columns already read), so P is double-buffered too; O has one buffer. The reference maximum m
// moves only when a row's maximum grows by more than 2^8, so O (in TMEM) is rescaled rarely —
// only then does the softmax wait for the previous P·V product; p <= 2^8 is exact enough in
// fp32 and in the hi/lo split.
// At the end of the split the row's O / l and LSE = m + log2 l are written: the final output
// when the tile has a single split, else a partial for the combine kernel.
//
// Warp roles as in the decode kernel: 0-3 softmax / epilogue (thread = TMEM lane = query row),
// 4 TMA producer (K/V tiles through a 2-stage ring, the next item's Q prefetched), 5 MMA issuer.
#include "common.cuh"
#include "internal.h"

namespace fd {

namespace {

constexpr int kCkRows = 128;   // query rows per tile = UMMA M
constexpr int kCkKeys = 128;   // keys per key tile = N of S, K of P·V
constexpr int kCkD = 128;      // head dim = K of S, N of P·V
constexpr int kCkStages = 2;
constexpr int kCkThreads = 192;
constexpr int kCkProducer = 4;
constexpr int kCkMma = 5;
constexpr int kCkSoftmax = 128;
constexpr uint32_t kCkTmemCols = 512;
constexpr uint32_t kColS0 = 0, kColO = 256;   // S/P buffers at 0 and 128, O at 256
constexpr uint32_t kCkHalf = kCkRows * 64 * 2;              // one 64-column half of a 128-row tile
constexpr float kRescaleThreshold = 8.0f;                   // log2 units

struct __align__(1024) CkSmem {
  __nv_bfloat16 q[2][2][kCkRows * 64];          // [item parity][d half], SW128
  __nv_bfloat16 k[kCkStages][2][kCkKeys * 64];  // [stage][d half], SW128
  __nv_bfloat16 v[kCkStages][2][kCkKeys * 64];
  int32_t meta[kCkStages][2];                   // key tile start, valid keys
  int32_t item_slot[2][2];                      // item index (-1: stop), key tiles
  TileItem item[2];
  uint64_t kfull[kCkStages], vfull[kCkStages], empty[kCkStages];
  uint64_t qfull[2], qempty[2], sfull[2], sempty[2];
  // P(J) ready, one barrier per tile parity: with a single barrier of four warp arrivals a fast
  // warp could arrive for tile J+1 before a slow one arrived for tile J and complete the phase
  // early; on pfull[J & 1] its next arrival needs S(J+2), which needs P·V(J), which needs the
  // whole phase of tile J.
  uint64_t pfull[2];
  uint64_t pfree, ofin, oempty, drain;
  uint32_t tmem_base;
  int abort_flag;
};

__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<const uint32_t*>(&h);
}

__global__ void __launch_bounds__(kCkThreads, 1)
    chunk_tc_kernel(const TileParams p, const __grid_constant__ CUtensorMap tmap_q,
                    const __grid_constant__ CUtensorMap tmap_k,
                    const __grid_constant__ CUtensorMap tmap_v) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  CkSmem& S = *reinterpret_cast<CkSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;

  if (tid == 0) {
    for (int s = 0; s < kCkStages; ++s) {
      mbar_init(&S.kfull[s], 1);
      mbar_init(&S.vfull[s], 1);
      mbar_init(&S.empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&S.qfull[i], 1);
      mbar_init(&S.qempty[i], 1 + 4);
      mbar_init(&S.sfull[i], 1);
      mbar_init(&S.sempty[i], 1);
    }
    mbar_init(&S.pfull[0], 4);
    mbar_init(&S.pfull[1], 4);
    mbar_init(&S.pfree, 1);
    mbar_init(&S.ofin, 1);
    mbar_init(&S.oempty, 4);
    mbar_init(&S.drain, 1);
    S.abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kCkMma) {
    tmem_alloc(&S.tmem_base, kCkTmemCols);
    tmem_relinquish();
  }
  if (warp == kCkProducer && lane == 0) {
    prefetch_tensor_map(&tmap_q);
    prefetch_tensor_map(&tmap_k);
    prefetch_tensor_map(&tmap_v);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = S.tmem_base;
  const WaitCtx ctx{&S.abort_flag, &p.hdr->status};
  pdl_wait_prerequisites();
  pdl_launch_dependents();

  if (warp == kCkProducer) {
    // ======================= TMA producer =======================
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
        mbar_arrive_expect_tx(&S.qfull[ps], 2u * 128u * static_cast<uint32_t>(p.q_box_rows));
        tma_load_3d(S.q[ps][0], &tmap_q, &S.qfull[ps], 0, it.h, it.row0);
        tma_load_3d(S.q[ps][1], &tmap_q, &S.qfull[ps], 64, it.h, it.row0);
        const int hkv = it.h / p.g;
        for (int j = 0; j < ntile; ++j, ++J) {
          if (j == claim_j) nidx = atomicAdd(&p.hdr->tile_counter, 1);
          const int st = J % kCkStages;
          if (!mbar_wait(&S.empty[st], ((J / kCkStages) & 1u) ^ 1u, ctx)) { ok = false; break; }
          const int t = it.k0 + j * kCkKeys;
          const int valid = max(0, min(kCkKeys, it.k1 - t));
          S.meta[st][0] = t;
          S.meta[st][1] = valid;
          if (valid > 0) {
            const uint32_t tx = 2u * 128u * static_cast<uint32_t>(p.kv_box_rows);
            mbar_arrive_expect_tx(&S.kfull[st], tx);
            tma_load_4d_stream(S.k[st][0], &tmap_k, &S.kfull[st], 0, t, hkv, it.b, pol);
            tma_load_4d_stream(S.k[st][1], &tmap_k, &S.kfull[st], 64, t, hkv, it.b, pol);
            mbar_arrive_expect_tx(&S.vfull[st], tx);
            tma_load_4d_stream(S.v[st][0], &tmap_v, &S.vfull[st], 0, t, hkv, it.b, pol);
            tma_load_4d_stream(S.v[st][1], &tmap_v, &S.vfull[st], 64, t, hkv, it.b, pol);
          } else {
            mbar_arrive(&S.kfull[st]);
            mbar_arrive(&S.vfull[st]);
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
        for (uint32_t back = 1; back <= kCkStages && back <= J; ++back) {
          const uint32_t jj = J - back;
          mbar_drain(&S.kfull[jj % kCkStages], (jj / kCkStages) & 1u);
          mbar_drain(&S.vfull[jj % kCkStages], (jj / kCkStages) & 1u);
        }
      }
    }
    __syncwarp();
  } else if (warp == kCkMma) {
    // ======================= MMA issuer =======================
    if (lane == 0) {
      const uint32_t idesc_s = idesc_bf16_f32(kCkRows, kCkKeys, false, false);
      const uint32_t idesc_o = idesc_bf16_f32(kCkRows, kCkD, false, true);
      uint32_t J = 0, K = 0;
      bool ok = true;
      bool have_prev = false;
      int prev_st = 0, prev_valid = 0;
      bool prev_first = false, prev_last = false;
      uint32_t prev_J = 0, prev_K = 0;
      auto issue_pv = [&](int st, int valid, uint32_t jt, bool first, bool last, uint32_t kt) -> bool {
        if (!mbar_wait(&S.vfull[st], (jt / kCkStages) & 1u, ctx)) return false;
        if (!mbar_wait(&S.pfull[jt & 1], (jt >> 1) & 1u, ctx)) return false;
        // the item's first product overwrites O: the previous item's O must have been read
        if (first && kt > 0 && !mbar_wait(&S.oempty, (kt - 1) & 1u, ctx)) return false;
        tc_fence_after();
        const int nk = (valid + 15) / 16;
        const uint32_t vaddr = smem_u32(S.v[st][0]);
        const uint32_t pcol = kColS0 + (jt & 1) * 128;  // P of this tile, over its S buffer
        bool acc = !first;
        for (int part = 0; part < 2; ++part) {
          for (int kk = 0; kk < nk; ++kk) {
            const uint64_t bd = smem_desc(vaddr + kk * 2048, kCkHalf, 1024, kLayoutSW128);
            const uint32_t acol = pcol + 32 * (kk >> 1) + 16 * part + 8 * (kk & 1);
            umma_bf16_ts(tmem + kColO, tmem + acol, bd, idesc_o, acc ? 1u : 0u);
            acc = true;
          }
        }
        umma_commit(&S.pfree);
        umma_commit(&S.sempty[jt & 1]);
        umma_commit(&S.empty[st]);
        if (last) umma_commit(&S.ofin);
        return true;
      };
      while (ok) {
        const int ps = K & 1;
        if (!mbar_wait(&S.qfull[ps], (K >> 1) & 1u, ctx)) { ok = false; break; }
        const int idx = S.item_slot[ps][0];
        const int ntile = S.item_slot[ps][1];
        if (idx < 0) break;
        const uint32_t q0 = smem_u32(S.q[ps][0]);
        const uint32_t q1 = smem_u32(S.q[ps][1]);
        for (int j = 0; j < ntile; ++j, ++J) {
          const int st = J % kCkStages;
          const int sb = J & 1;
          if (!mbar_wait(&S.kfull[st], (J / kCkStages) & 1u, ctx)) { ok = false; break; }
          if (!mbar_wait(&S.sempty[sb], ((J >> 1) & 1u) ^ 1u, ctx)) { ok = false; break; }
          tc_fence_after();
          const int valid = S.meta[st][1];
          if (valid > 0) {
            const uint32_t k0 = smem_u32(S.k[st][0]);
            const uint32_t k1 = smem_u32(S.k[st][1]);
#pragma unroll
            for (int kk = 0; kk < kCkD / 16; ++kk) {
              const uint32_t qa = (kk < 4 ? q0 : q1) + (kk & 3) * 32;
              const uint32_t ka = (kk < 4 ? k0 : k1) + (kk & 3) * 32;
              umma_bf16_ss(tmem + kColS0 + sb * 128, smem_desc(qa, 16, 1024, kLayoutSW128),
                           smem_desc(ka, 16, 1024, kLayoutSW128), idesc_s, kk > 0 ? 1u : 0u);
            }
          }
          umma_commit(&S.sfull[sb]);
          if (j == ntile - 1) umma_commit(&S.qempty[ps]);
          if (have_prev && !issue_pv(prev_st, prev_valid, prev_J, prev_first, prev_last, prev_K)) {
            ok = false;
            break;
          }
          have_prev = true;
          prev_st = st;
          prev_valid = valid;
          prev_J = J;
          prev_first = j == 0;
          prev_last = j == ntile - 1;
          prev_K = K;
        }
        if (!ok) break;
        ++K;
      }
      if (ok && have_prev) ok = issue_pv(prev_st, prev_valid, prev_J, prev_first, prev_last, prev_K);
      umma_commit(&S.drain);
      mbar_drain(&S.drain, 0);
    }
    __syncwarp();
  } else {
    // ======================= softmax / epilogue (thread = query row) =======================
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
      if (idx < 0) break;
      const bool row_ok = r < it.rows;
      const int limit = it.prefix + it.pos0 + r;  // last visible key of this row
      float m = -INFINITY, l = 0.f;
      for (int j = 0; j < ntile; ++j, ++J) {
        const int st = J % kCkStages;
        const int sb = J & 1;
        if (!mbar_wait(&S.sfull[sb], (J >> 1) & 1u, ctx)) { ok = false; break; }
        if (!mbar_wait(&S.kfull[st], (J / kCkStages) & 1u, ctx)) { ok = false; break; }
        tc_fence_after();
        const int kt0 = S.meta[st][0];
        const int valid = S.meta[st][1];
        const uint32_t sp = tmem + lane_base + kColS0 + sb * 128;  // this tile's S, then its P
        // keys [0, nvis) of the tile are visible to this row: inside the split, at or before the
        // row's causal limit, and the row inside the chunk
        const int nvis = row_ok ? max(0, min(valid, limit - kt0 + 1)) : 0;
        // pass 1: the row's maximum over the visible keys
        float tmax = -INFINITY;
        if (valid > 0) {
#pragma unroll
          for (int c = 0; c < kCkKeys; c += 32) {
            uint32_t raw[32];
            tmem_ld32(sp + c, raw);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i)
              if (c + i < nvis) tmax = fmaxf(tmax, __uint_as_float(raw[i]) * p.scale_log2);
          }
        }
        const float mn = fmaxf(m, tmax);
        const bool move = mn > m + kRescaleThreshold || (m == -INFINITY && mn != -INFINITY);
        const float mref = move ? mn : m;
        const float alpha = move ? (m == -INFINITY ? 0.f : fast_exp2(m - mn)) : 1.f;
        if (j > 0 && __any_sync(0xffffffffu, move)) {
          // O changes only after the previous product has added into it
          if (!mbar_wait(&S.pfree, (J - 1) & 1u, ctx)) { ok = false; break; }
          tc_fence_after();
#pragma unroll
          for (int c = 0; c < kCkD; c += 32) {
            uint32_t o[32];
            tmem_ld32(tmem + lane_base + kColO + c, o);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
            tmem_st32(tmem + lane_base + kColO + c, o);
          }
        }
        if ((valid & 15) != 0) {
          // zero V rows [valid, next multiple of 16): they may lie past the request's keys
          if (!mbar_wait(&S.vfull[st], (J / kCkStages) & 1u, ctx)) { ok = false; break; }
          const int r0 = valid, r1 = (valid + 15) & ~15;
          for (int c = tid; c < (r1 - r0) * 16; c += kCkSoftmax) {
            const int row = r0 + c / 16;
            *reinterpret_cast<uint4*>(reinterpret_cast<unsigned char*>(S.v[st][(c / 8) & 1]) +
                                      row * 128 + (c & 7) * 16) = make_uint4(0u, 0u, 0u, 0u);
          }
          fence_proxy_async_smem();
        }
        // pass 2: p = 2^(s - m), split into bf16 hi + lo, written over the chunk's own columns
        float rs = 0.f;
#pragma unroll
        for (int c = 0; c < kCkKeys; c += 32) {
          uint32_t raw[32];
          if (valid > 0) {
            tmem_ld32(sp + c, raw);
            tmem_wait_ld();
          }
          uint32_t w[32];
#pragma unroll
          for (int i = 0; i < 32; i += 2) {
            const float x0 = c + i < nvis ? __uint_as_float(raw[i]) * p.scale_log2 : -INFINITY;
            const float x1 = c + i + 1 < nvis ? __uint_as_float(raw[i + 1]) * p.scale_log2 : -INFINITY;
            const float p0 = mref == -INFINITY ? 0.f : fast_exp2(x0 - mref);
            const float p1 = mref == -INFINITY ? 0.f : fast_exp2(x1 - mref);
            rs += p0 + p1;
            const __nv_bfloat162 h2 = __floats2bfloat162_rn(p0, p1);
            const float2 hf = __bfloat1622float2(h2);
            w[i / 2] = *reinterpret_cast<const uint32_t*>(&h2);
            w[16 + i / 2] = pack_bf16x2(p0 - hf.x, p1 - hf.y);
          }
          tmem_st32(sp + c, w);
        }
        l = fmaf(l, alpha, rs);
        m = mref;
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&S.pfull[sb]);
      }
      if (!ok) break;

      // ---- epilogue: O / l and the LSE of every row of the tile ----
      if (!mbar_wait(&S.ofin, K & 1u, ctx)) break;
      tc_fence_after();
      const bool direct = it.nsplit == 1;
      const float inv = l > 0.f ? 1.f / l : 0.f;
      const float lse2 = l > 0.f ? m + log2f(l) : -INFINITY;
      const int hkv = it.h / p.g, g = it.h - hkv * p.g;
      const int64_t row = static_cast<int64_t>(it.row0) + r;
      const int64_t slot = static_cast<int64_t>(it.slot0) +
                           (static_cast<int64_t>(r) * p.hkv + hkv) * it.nsplit + it.split;
#pragma unroll
      for (int c = 0; c < kCkD; c += 32) {
        uint32_t o[32];
        tmem_ld32(tmem + lane_base + kColO + c, o);
        tmem_wait_ld();
        if (row_ok) {
          if (direct) {
            __nv_bfloat16* out = static_cast<__nv_bfloat16*>(p.out) + row * p.o_sr +
                                 static_cast<int64_t>(it.h) * p.o_sh + c;
#pragma unroll
            for (int i = 0; i < 32; i += 8) {
              uint4 v;
              v.x = pack_bf16x2(__uint_as_float(o[i + 0]) * inv, __uint_as_float(o[i + 1]) * inv);
              v.y = pack_bf16x2(__uint_as_float(o[i + 2]) * inv, __uint_as_float(o[i + 3]) * inv);
              v.z = pack_bf16x2(__uint_as_float(o[i + 4]) * inv, __uint_as_float(o[i + 5]) * inv);
              v.w = pack_bf16x2(__uint_as_float(o[i + 6]) * inv, __uint_as_float(o[i + 7]) * inv);
              *reinterpret_cast<uint4*>(out + i) = v;
            }
          } else {
            float* dst = p.part_o + (slot * p.g + g) * kCkD + c;
#pragma unroll
            for (int i = 0; i < 32; i += 4)
              *reinterpret_cast<float4*>(dst + i) =
                  make_float4(__uint_as_float(o[i]) * inv, __uint_as_float(o[i + 1]) * inv,
                              __uint_as_float(o[i + 2]) * inv, __uint_as_float(o[i + 3]) * inv);
          }
        }
      }
      if (row_ok) {
        if (direct) p.lse[row * p.hq + it.h] = lse2 * kLn2;
        else p.part_lse[slot * p.g + g] = lse2;
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&S.oempty);
      ++K;
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kCkMma) tmem_dealloc(tmem, kCkTmemCols);
}

}  // namespace

cudaError_t launch_chunk_tc(const TileParams& p, const CUtensorMap& tq, const CUtensorMap& tk,
                            const CUtensorMap& tv, int nctas, cudaStream_t stream) {
  const size_t smem = sizeof(CkSmem) + 1024;
  cudaError_t e = cudaFuncSetAttribute(chunk_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
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
  return cudaLaunchKernelEx(&cfg, chunk_tc_kernel, p, tq, tk, tv);
}

}  // namespace fd
