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
// Sᵀ and Oᵀ live in tensor memory, double-buffered; the softmax warps read them with tcgen05.ld,
// keep the running max m, the running sums l (per key lane) and the output accumulator (per d
// lane) in registers, and rescale by 2^(m - m') as the online softmax of
// "大语言模型长序列推理优化：ChunkedPrefill与FlashDecoding技术解析" §3.1 does. Splitting P into two
// bf16 terms keeps ~16 bits of each weight in the P·V product at no visible cost: the tensor
// pipe is far from busy in this memory-bound loop, and N must be a multiple of 16 anyway.
//
// Warp roles: 0-3 softmax / correction / epilogue (one thread per TMEM lane), 4 TMA producer,
// 5 MMA issuer and TMEM owner. K/V tiles arrive by 4-D TMA with 128-byte swizzle into a 3-stage
// ring; keys past the sequence end inside the last tile are masked to p = 0 and their V rows are
// zeroed in shared memory before the P·V product, so stale or poisoned cache rows never leak.
#include "common.cuh"
#include "internal.h"

namespace fd {

namespace {

constexpr int kTcKeys = 128;           // keys per tile = UMMA M of the Sᵀ product
constexpr int kTcD = 128;              // head dim = UMMA M of the Oᵀ product
constexpr int kTcStages = 3;
constexpr int kTcThreads = 192;
constexpr int kProducerWarp = 4;
constexpr int kMmaWarp = 5;
constexpr int kSoftmaxThreads = 128;
constexpr uint32_t kTmemCols = 128;
constexpr uint32_t kHalfBytes = kTcKeys * 64 * 2;   // one 64-column half of a K or V tile

template <int GPAD>
struct __align__(1024) TcSmem {
  static constexpr int kNO = 2 * GPAD;           // Oᵀ columns: hi then lo
  static constexpr int kPGroups = kNO / 8;       // 8-column core-matrix groups of Pᵀ
  __nv_bfloat16 k[kTcStages][2][kTcKeys * 64];   // [stage][d half][row*64 + col], SW128
  __nv_bfloat16 v[kTcStages][2][kTcKeys * 64];
  __nv_bfloat16 q[2][2][16 * 64];                // [item parity][d half], SW128
  __nv_bfloat16 p[2][kPGroups * kTcKeys * 8];    // [tile parity], MN-major core matrices
  float wmax[2][4][GPAD];
  float lred[4][GPAD];
  int32_t meta[kTcStages][2];                    // tile start, valid keys
  int32_t item_slot[2][2];                       // item index (-1: stop), tiles
  DecodeItem item[2];                            // the item's descriptor (by item parity)
  uint64_t kfull[kTcStages], vfull[kTcStages], empty[kTcStages];
  uint64_t qfull[2], qempty[2], sfull[2], sempty[2], pfull[2], pempty[2], ofull[2], oempty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
};

template <int GPAD>
__global__ void __launch_bounds__(kTcThreads, 1)
    decode_tc_kernel(const DecodeParams p, const __grid_constant__ CUtensorMap tmap_q,
                     const __grid_constant__ CUtensorMap tmap_k,
                     const __grid_constant__ CUtensorMap tmap_v) {
  using Smem = TcSmem<GPAD>;
  constexpr int kNO = Smem::kNO;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  // dynamic shared memory is only guaranteed 16-byte aligned: round up to 1024 for SW128
  Smem& S = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;

  if (tid == 0) {
    for (int s = 0; s < kTcStages; ++s) {
      mbar_init(&S.kfull[s], 1);
      mbar_init(&S.vfull[s], 1);
      mbar_init(&S.empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&S.qfull[i], 1);
      mbar_init(&S.qempty[i], 1 + 4);
      mbar_init(&S.sfull[i], 1);
      mbar_init(&S.sempty[i], 4);
      mbar_init(&S.pfull[i], 4);
      mbar_init(&S.pempty[i], 1);
      mbar_init(&S.ofull[i], 1);
      mbar_init(&S.oempty[i], 4);
    }
    mbar_init(&S.drain, 1);
    S.abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(&S.tmem_base, kTmemCols);
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
  // Everything above overlapped the planner (programmatic dependent launch); the plan it wrote
  // is read below. The combine kernel may launch now: it waits for this grid the same way.
  pdl_wait_prerequisites();
  pdl_launch_dependents();

  if (warp == kProducerWarp) {
    // ======================= TMA producer =======================
    if (lane == 0) {
      const int n_items = *reinterpret_cast<volatile int32_t*>(&p.hdr->num_dec_items);
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
      if (idx < n_items) it = p.items[idx];
      while (ok && idx < n_items) {
        int nidx = n_items;
        DecodeItem nit{};
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
          const int st = J % kTcStages;
          if (!mbar_wait(&S.empty[st], ((J / kTcStages) & 1u) ^ 1u, ctx)) { ok = false; break; }
          const int t = it.t0 + j * kTcKeys;
          const int valid = max(0, min(kTcKeys, it.t1 - t));
          S.meta[st][0] = t;
          S.meta[st][1] = valid;
          if (valid > 0) {
            const uint32_t tx = 2u * 128u * static_cast<uint32_t>(p.kv_box_rows);
            mbar_arrive_expect_tx(&S.kfull[st], tx);
            tma_load_4d_stream(S.k[st][0], &tmap_k, &S.kfull[st], 0, t, it.h, it.b, pol);
            tma_load_4d_stream(S.k[st][1], &tmap_k, &S.kfull[st], 64, t, it.h, it.b, pol);
            mbar_arrive_expect_tx(&S.vfull[st], tx);
            tma_load_4d_stream(S.v[st][0], &tmap_v, &S.vfull[st], 0, t, it.h, it.b, pol);
            tma_load_4d_stream(S.v[st][1], &tmap_v, &S.vfull[st], 64, t, it.h, it.b, pol);
          } else {
            mbar_arrive(&S.kfull[st]);
            mbar_arrive(&S.vfull[st]);
          }
          if (j == read_j && nidx < n_items) nit = p.items[nidx];
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
        for (uint32_t back = 1; back <= kTcStages && back <= J; ++back) {
          const uint32_t jj = J - back;
          mbar_drain(&S.kfull[jj % kTcStages], (jj / kTcStages) & 1u);
          mbar_drain(&S.vfull[jj % kTcStages], (jj / kTcStages) & 1u);
        }
      }
    }
    __syncwarp();
  } else if (warp == kMmaWarp) {
    // ======================= MMA issuer =======================
    if (lane == 0) {
      const uint32_t idesc_s = idesc_bf16_f32(kTcKeys, 16, false, false);
      const uint32_t idesc_o = idesc_bf16_f32(kTcD, kNO, true, true);
      uint32_t J = 0, K = 0;
      bool ok = true;
      bool have_prev = false;
      int prev_st = 0, prev_valid = 0;
      uint32_t prev_J = 0;
      auto issue_pv = [&](int st, int valid, uint32_t jt) -> bool {
        const int ob = jt & 1;
        if (!mbar_wait(&S.vfull[st], (jt / kTcStages) & 1u, ctx)) return false;
        if (!mbar_wait(&S.pfull[ob], (jt >> 1) & 1u, ctx)) return false;
        if (!mbar_wait(&S.oempty[ob], ((jt >> 1) & 1u) ^ 1u, ctx)) return false;
        tc_fence_after();
        const int nk = (valid + 15) / 16;
        const uint32_t vaddr = smem_u32(S.v[st][0]);
        const uint32_t paddr = smem_u32(S.p[ob]);
        for (int kk = 0; kk < nk; ++kk) {
          const uint64_t ad = smem_desc(vaddr + kk * 2048, kHalfBytes, 1024, kLayoutSW128);
          const uint64_t bd = smem_desc(paddr + kk * 256, 128, 2048, kLayoutNone);
          umma_bf16_ss(tmem + 32 + ob * kNO, ad, bd, idesc_o, kk > 0 ? 1u : 0u);
        }
        umma_commit(&S.ofull[ob]);
        umma_commit(&S.pempty[ob]);
        umma_commit(&S.empty[st]);
        return true;
      };
      while (ok) {
        const int ps = K & 1;
        if (!mbar_wait(&S.qfull[ps], (K >> 1) & 1u, ctx)) { ok = false; break; }
        const int idx = S.item_slot[ps][0];
        const int ntile = S.item_slot[ps][1];
        if (idx < 0) break;
        const uint32_t qaddr0 = smem_u32(S.q[ps][0]);
        const uint32_t qaddr1 = smem_u32(S.q[ps][1]);
        for (int j = 0; j < ntile; ++j, ++J) {
          const int st = J % kTcStages;
          const int sb = J & 1;
          if (!mbar_wait(&S.kfull[st], (J / kTcStages) & 1u, ctx)) { ok = false; break; }
          if (!mbar_wait(&S.sempty[sb], ((J >> 1) & 1u) ^ 1u, ctx)) { ok = false; break; }
          tc_fence_after();
          const int valid = S.meta[st][1];
          if (valid > 0) {
            const uint32_t k0 = smem_u32(S.k[st][0]);
            const uint32_t k1 = smem_u32(S.k[st][1]);
#pragma unroll
            for (int kk = 0; kk < kTcD / 16; ++kk) {
              const uint32_t ka = (kk < 4 ? k0 : k1) + (kk & 3) * 32;
              const uint32_t qa = (kk < 4 ? qaddr0 : qaddr1) + (kk & 3) * 32;
              umma_bf16_ss(tmem + sb * 16, smem_desc(ka, 16, 1024, kLayoutSW128),
                           smem_desc(qa, 16, 1024, kLayoutSW128), idesc_s, kk > 0 ? 1u : 0u);
            }
          }
          umma_commit(&S.sfull[sb]);
          if (j == ntile - 1) umma_commit(&S.qempty[ps]);
          if (have_prev && !issue_pv(prev_st, prev_valid, prev_J)) { ok = false; break; }
          have_prev = true;
          prev_st = st;
          prev_valid = valid;
          prev_J = J;
        }
        if (!ok) break;
        ++K;
      }
      if (ok && have_prev) ok = issue_pv(prev_st, prev_valid, prev_J);
      // every MMA this thread issued has completed once `drain` flips
      umma_commit(&S.drain);
      mbar_drain(&S.drain, 0);
    }
    __syncwarp();
  } else {
    // ======================= softmax / correction / epilogue =======================
    const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
    float m[GPAD], lp[GPAD], oacc[GPAD], alpha_prev[GPAD];
    uint32_t J = 0, K = 0;
    bool ok = true;
    auto accumulate = [&](uint32_t jt, int valid, const float* a) -> bool {
      const int ob = jt & 1;
      if (!mbar_wait(&S.ofull[ob], (jt >> 1) & 1u, ctx)) return false;
      tc_fence_after();
      float hi[GPAD], lo[GPAD];
      if (valid > 0) {
        if constexpr (kNO == 16) {
          uint32_t r[16];
          tmem_ld16(tmem + lane_base + 32 + ob * kNO, r);
          tmem_wait_ld();
#pragma unroll
          for (int g = 0; g < GPAD; ++g) { hi[g] = __uint_as_float(r[g]); lo[g] = __uint_as_float(r[GPAD + g]); }
        } else {
          uint32_t r[32];
          tmem_ld32(tmem + lane_base + 32 + ob * kNO, r);
          tmem_wait_ld();
#pragma unroll
          for (int g = 0; g < GPAD; ++g) { hi[g] = __uint_as_float(r[g]); lo[g] = __uint_as_float(r[GPAD + g]); }
        }
      } else {
#pragma unroll
        for (int g = 0; g < GPAD; ++g) { hi[g] = 0.f; lo[g] = 0.f; }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&S.oempty[ob]);
#pragma unroll
      for (int g = 0; g < GPAD; ++g) oacc[g] = fmaf(oacc[g], a[g], hi[g] + lo[g]);
      return true;
    };
    while (ok) {
      const int ps = K & 1;
      if (!mbar_wait(&S.qfull[ps], (K >> 1) & 1u, ctx)) break;
      const int idx = S.item_slot[ps][0];
      const int ntile = S.item_slot[ps][1];
      const DecodeItem it = S.item[ps];
      __syncwarp();
      if (lane == 0) mbar_arrive(&S.qempty[ps]);
      if (idx < 0) break;
#pragma unroll
      for (int g = 0; g < GPAD; ++g) { m[g] = -INFINITY; lp[g] = 0.f; oacc[g] = 0.f; alpha_prev[g] = 1.f; }
      int prev_valid = 0;
      for (int j = 0; j < ntile; ++j, ++J) {
        const int st = J % kTcStages;
        const int sb = J & 1;
        if (!mbar_wait(&S.sfull[sb], (J >> 1) & 1u, ctx)) { ok = false; break; }
        // the stage's metadata was published with the producer's arrival on kfull
        if (!mbar_wait(&S.kfull[st], (J / kTcStages) & 1u, ctx)) { ok = false; break; }
        tc_fence_after();
        const int valid = S.meta[st][1];
        uint32_t sr[16];
        if (valid > 0) {
          tmem_ld16(tmem + lane_base + sb * 16, sr);
          tmem_wait_ld();
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&S.sempty[sb]);

        const bool in = tid < valid;
        float x[GPAD];
#pragma unroll
        for (int g = 0; g < GPAD; ++g)
          x[g] = (in && g < p.g) ? __uint_as_float(sr[g]) * p.scale_log2 : -INFINITY;
#pragma unroll
        for (int g = 0; g < GPAD; ++g) {
          const float wm = warp_max_f32(x[g]);
          if (lane == 0) S.wmax[sb][warp][g] = wm;
        }
        named_bar_sync(1, kSoftmaxThreads);
        float alpha[GPAD], pr[GPAD];
#pragma unroll
        for (int g = 0; g < GPAD; ++g) {
          const float tmx = fmaxf(fmaxf(S.wmax[sb][0][g], S.wmax[sb][1][g]),
                                  fmaxf(S.wmax[sb][2][g], S.wmax[sb][3][g]));
          const float mn = fmaxf(m[g], tmx);
          alpha[g] = (mn == -INFINITY) ? 1.f : fast_exp2(m[g] - mn);
          pr[g] = (mn == -INFINITY) ? 0.f : fast_exp2(x[g] - mn);
          lp[g] = fmaf(lp[g], alpha[g], pr[g]);
          m[g] = mn;
        }
        // P_hi / P_lo for this key lane
        uint32_t hw[GPAD / 2], lw[GPAD / 2];
#pragma unroll
        for (int g = 0; g < GPAD; g += 2) {
          const __nv_bfloat162 h2 = __floats2bfloat162_rn(pr[g], pr[g + 1]);
          const float2 hf = __bfloat1622float2(h2);
          const __nv_bfloat162 l2 = __floats2bfloat162_rn(pr[g] - hf.x, pr[g + 1] - hf.y);
          hw[g / 2] = *reinterpret_cast<const uint32_t*>(&h2);
          lw[g / 2] = *reinterpret_cast<const uint32_t*>(&l2);
        }
        if (!mbar_wait(&S.pempty[sb], ((J >> 1) & 1u) ^ 1u, ctx)) { ok = false; break; }
        if ((valid & 15) != 0) {
          // zero V rows [valid, next multiple of 16): they may lie past the sequence end
          if (!mbar_wait(&S.vfull[st], (J / kTcStages) & 1u, ctx)) { ok = false; break; }
          const int r0 = valid, r1 = (valid + 15) & ~15;
          const int nchunks = (r1 - r0) * 2 * 8;
          for (int c = tid; c < nchunks; c += kSoftmaxThreads) {
            const int row = r0 + c / 16;
            const int half = (c / 8) & 1;
            const int ch = c & 7;
            *reinterpret_cast<uint4*>(reinterpret_cast<unsigned char*>(S.v[st][half]) + row * 128 + ch * 16) =
                make_uint4(0u, 0u, 0u, 0u);
          }
        }
        unsigned char* pb = reinterpret_cast<unsigned char*>(S.p[sb]);
#pragma unroll
        for (int grp = 0; grp < GPAD / 8; ++grp) {
          *reinterpret_cast<uint4*>(pb + grp * 2048 + tid * 16) =
              make_uint4(hw[grp * 4 + 0], hw[grp * 4 + 1], hw[grp * 4 + 2], hw[grp * 4 + 3]);
          *reinterpret_cast<uint4*>(pb + (GPAD / 8 + grp) * 2048 + tid * 16) =
              make_uint4(lw[grp * 4 + 0], lw[grp * 4 + 1], lw[grp * 4 + 2], lw[grp * 4 + 3]);
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&S.pfull[sb]);
        if (j > 0 && !accumulate(J - 1, prev_valid, alpha_prev)) { ok = false; break; }
#pragma unroll
        for (int g = 0; g < GPAD; ++g) alpha_prev[g] = alpha[g];
        prev_valid = valid;
      }
      if (!ok) break;
      if (!accumulate(J - 1, prev_valid, alpha_prev)) break;

      // ---- epilogue: l = sum over key lanes; O = acc / l ----
#pragma unroll
      for (int g = 0; g < GPAD; ++g) {
        const float s = warp_sum_f32(lp[g]);
        if (lane == 0) S.lred[warp][g] = s;
      }
      named_bar_sync(1, kSoftmaxThreads);
      const bool direct = it.nsplit == 1;
      const int64_t slot = direct ? 0 : static_cast<int64_t>(it.slot);
#pragma unroll
      for (int g = 0; g < GPAD; ++g) {
        if (g < p.g) {
          const float l = S.lred[0][g] + S.lred[1][g] + S.lred[2][g] + S.lred[3][g];
          const float ov = l > 0.f ? oacc[g] / l : 0.f;
          const float lse2 = l > 0.f ? m[g] + log2f(l) : -INFINITY;
          const int hq = it.h * p.g + g;
          if (direct) {
            __nv_bfloat16* out = static_cast<__nv_bfloat16*>(p.out) +
                                 static_cast<int64_t>(it.row) * p.o_sr + static_cast<int64_t>(hq) * p.o_sh;
            out[tid] = __float2bfloat16_rn(ov);
            if (tid == 0) p.lse[static_cast<int64_t>(it.row) * p.hq + hq] = lse2 * kLn2;
          } else {
            p.part_o[(slot * p.g + g) * kTcD + tid] = ov;
            if (tid == 0) p.part_lse[slot * p.g + g] = lse2;
          }
        }
      }
      named_bar_sync(1, kSoftmaxThreads);
      ++K;
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kMmaWarp) tmem_dealloc(tmem, kTmemCols);
}

template <int GPAD>
cudaError_t launch_tc_t(const DecodeParams& p, const CUtensorMap& tq, const CUtensorMap& tk,
                        const CUtensorMap& tv, int nctas, cudaStream_t stream) {
  const size_t smem = sizeof(TcSmem<GPAD>) + 1024;
  cudaError_t e = cudaFuncSetAttribute(decode_tc_kernel<GPAD>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(nctas);
  cfg.blockDim = dim3(kTcThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, decode_tc_kernel<GPAD>, p, tq, tk, tv);
}

}  // namespace

cudaError_t launch_decode_tc(const DecodeParams& p, const CUtensorMap& tmap_q,
                             const CUtensorMap& tmap_k, const CUtensorMap& tmap_v, int nctas,
                             cudaStream_t stream) {
  if (p.g <= 8) return launch_tc_t<8>(p, tmap_q, tmap_k, tmap_v, nctas, stream);
  return launch_tc_t<16>(p, tmap_q, tmap_k, tmap_v, nctas, stream);
}

}  // namespace fd
