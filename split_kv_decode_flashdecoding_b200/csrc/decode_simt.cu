// Split-KV decode kernel on CUDA cores (MHA / small groups, fp32 or bf16, D in {64, 128}).
//
// One persistent CTA per work slot pulls split items from the planner's list (longest first,
// dynamic cursor). A producer warp streams each split's K and V rows with bulk copies (TMA)
// into a 3-stage shared-memory ring; four consumer warps compute, per tile,
//   s_t = (q · k_t) * scale * log2(e)     lanes split D, 128-bit shared loads, shuffle reduction
//   m' = max(m, max_t s_t);  p_t = 2^(s_t - m');  l = l * 2^(m - m') + sum_t p_t
//   acc = acc * 2^(m - m') + sum_t p_t v_t     fp32
// which is the online softmax of "大语言模型长序列推理优化：ChunkedPrefill与FlashDecoding技术解析"
// §3.1 in base 2. At the end of a split the partial O = acc / l and LSE = m + log2 l are written
// for the combine pass ("大模型推理加速FlashDecoding算法原理与多GPU并行解码实战",
// "多GPU张量并行扩展下的FlashDecoding实现"), or the final output directly when the sequence has a
// single split. Keys at positions >= the split end are never touched: a copy moves only the
// valid rows and every loop stops at the valid count.
#include "common.cuh"
#include "internal.h"

namespace fd {

namespace {

constexpr int kSimtStages = 3;
constexpr int kSimtConsumerWarps = 4;
constexpr int kSimtThreads = (kSimtConsumerWarps + 1) * 32;
constexpr int kSimtConsumers = kSimtConsumerWarps * 32;

template <typename T, int D, int GP>
struct SimtCfg {
  static constexpr int kTile = 32768 / (2 * D * static_cast<int>(sizeof(T)));  // tokens/stage
  static constexpr int kLpt = D / 16;                  // lanes per token in the q·k phase
  static constexpr int kTokPerWarpPass = 32 / kLpt;
  static constexpr int kTokPerPass = kTokPerWarpPass * kSimtConsumerWarps;
  static constexpr int kPasses = kTile / kTokPerPass;
  static constexpr int kChunkElems = 16 / static_cast<int>(sizeof(T));  // per 16-byte chunk
  static constexpr int kChunksPerLane = 16 / kChunkElems;              // 16 elements per lane
  static constexpr int kDpl = D / 32;                  // P·V: elements of D per lane
  static constexpr int kTokPerWarpPV = kTile / kSimtConsumerWarps;
  static constexpr int kSlots = (GP * kTile + kSimtConsumers - 1) / kSimtConsumers;
  static_assert(kPasses * kTokPerPass == kTile, "tile must be a whole number of passes");
};

template <typename T, int D, int GP>
struct __align__(128) SimtSmem {
  using C = SimtCfg<T, D, GP>;
  T k[kSimtStages][C::kTile * D];
  T v[kSimtStages][C::kTile * D];
  T qs[kSimtStages][GP * D];       // the item's query rows, loaded with its first tile
  float sc[2][GP][C::kTile];       // scores, then probabilities, of the current tile
  float wmax[2][kSimtConsumerWarps][GP];
  float red[kSimtConsumerWarps][GP][D];
  float lsum[GP * C::kTile > kSimtConsumers ? GP * C::kTile : kSimtConsumers];
  float lfin[GP];
  float mlse[kMergeLseCap];        // split LSEs of a group being merged
  int mflag;
  int32_t meta[kSimtStages][4];    // item index (-1: stop), tile start, valid keys, flags
  DecodeItem item[kSimtStages];    // descriptor of the stage's item
  uint64_t full[kSimtStages];
  uint64_t empty[kSimtStages];
  int abort_flag;
};

constexpr int kFirstTile = 1;
constexpr int kLastTile = 2;

// 16-byte chunk of T -> kChunkElems floats
template <typename T>
__device__ __forceinline__ void load_chunk(const T* src, float* dst);
template <>
__device__ __forceinline__ void load_chunk<float>(const float* src, float* dst) {
  const float4 x = *reinterpret_cast<const float4*>(src);
  dst[0] = x.x; dst[1] = x.y; dst[2] = x.z; dst[3] = x.w;
}
template <>
__device__ __forceinline__ void load_chunk<__nv_bfloat16>(const __nv_bfloat16* src, float* dst) {
  const uint4 x = *reinterpret_cast<const uint4*>(src);
  const uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    dst[2 * i] = __uint_as_float(w[i] << 16);
    dst[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

// kDpl consecutive elements of T -> floats
template <typename T, int N>
__device__ __forceinline__ void load_vec(const T* src, float* dst) {
#pragma unroll
  for (int i = 0; i < N; ++i) dst[i] = to_f32<T>(src[i]);
}

template <typename T, int D, int GP>
__global__ void __launch_bounds__(kSimtThreads) decode_simt_kernel(DecodeParams p) {
  using C = SimtCfg<T, D, GP>;
  extern __shared__ __align__(128) unsigned char smem_raw[];
  auto& S = *reinterpret_cast<SimtSmem<T, D, GP>*>(smem_raw);
  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;

  if (tid == 0) {
    for (int s = 0; s < kSimtStages; ++s) {
      mbar_init(&S.full[s], 1);
      mbar_init(&S.empty[s], kSimtConsumerWarps);
    }
    S.abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  const WaitCtx ctx{&S.abort_flag, &p.hdr->status};
  // the barrier set-up above overlapped the planner (programmatic dependent launch)
  pdl_wait_prerequisites();
  pdl_launch_dependents();
  const T* kbase = static_cast<const T*>(p.k);
  const T* vbase = static_cast<const T*>(p.v);
  const T* qbase = static_cast<const T*>(p.q);

  if (warp == kSimtConsumerWarps) {
    // ---------------- producer: one thread streams K/V tiles ----------------
    if (lane != 0) return;
    const bool paged = p.block_table != nullptr;
    const int n_items = *reinterpret_cast<volatile int32_t*>(&p.hdr->num_dec_items);
    const uint64_t pol = l2_evict_first_policy();
    uint32_t J = 0;
    bool ok = true;
    // The next item is claimed three tiles before the current one ends and its descriptor is
    // read one tile later: both global round trips then overlap the ring's lookahead instead of
    // stalling the stream at every item boundary.
    int idx = atomicAdd(&p.hdr->dec_counter, 1);
    DecodeItem it{};
    if (idx < n_items) it = p.items[idx];
    while (ok && idx < n_items) {
      int nidx = n_items;
      DecodeItem nit{};
      const int len = it.t1 - it.t0;
      const int ntile = len > 0 ? (len + C::kTile - 1) / C::kTile : 1;
      const int claim_j = max(0, ntile - 3), read_j = max(0, ntile - 2);
      const int64_t off = static_cast<int64_t>(it.b) * p.kv_sb + static_cast<int64_t>(it.h) * p.kv_sh;
      for (int j = 0; j < ntile; ++j, ++J) {
        if (j == claim_j) nidx = atomicAdd(&p.hdr->dec_counter, 1);
        const int st = J % kSimtStages;
        const int t = it.t0 + j * C::kTile;
        const int valid = max(0, min(C::kTile, it.t1 - t));
        // paged cache: the tile's page segments (tiles start on multiples of kTile, which
        // divides 128, and page sizes divide 128 or are multiples of it). The first segment's
        // page is loaded before the stage wait, so that the load overlaps it; a tile that spans
        // several (short) pages reads the others after the wait.
        const int32_t* trow = nullptr;
        int32_t pid0 = -1;
        int nseg = 0, row0 = 0, first = 0;
        if (paged && valid > 0) {
          const int P = p.page_size;
          first = t / P;
          row0 = t - first * P;
          nseg = (row0 + valid + P - 1) / P;
          trow = p.block_table + static_cast<int64_t>(it.b) * p.pages_per_seq + first;
          pid0 = trow[0];
        }
        if (!mbar_wait(&S.empty[st], ((J / kSimtStages) & 1u) ^ 1u, ctx)) { ok = false; break; }
        S.meta[st][0] = idx;
        S.meta[st][1] = t;
        S.meta[st][2] = valid;
        S.meta[st][3] = (j == 0 ? kFirstTile : 0) | (j == ntile - 1 ? kLastTile : 0);
        S.item[st] = it;
        uint32_t bytes = static_cast<uint32_t>(valid) * D * sizeof(T);
        if (paged && valid > 0) {
          // a segment whose page index lies outside the pool is not read (FD_FLAG_BAD_PAGE)
          bool bad = false;
#pragma unroll 1  // kept rolled: the producer loop must stay small in the instruction cache
          for (int i = 0; i < nseg; ++i) {
            const int32_t id = i == 0 ? pid0 : trow[i];
            if (id < 0 || id >= p.num_pages) {
              bad = true;
              const int lo = i == 0 ? 0 : i * p.page_size - row0;
              const int hi = min(valid, (i + 1) * p.page_size - row0);
              bytes -= static_cast<uint32_t>(hi - lo) * D * sizeof(T);
            }
          }
          if (bad) atomicOr(&p.hdr->status, FD_FLAG_BAD_PAGE);
        }
        const uint32_t qbytes = j == 0 ? static_cast<uint32_t>(p.g) * D * sizeof(T) : 0u;
        if (bytes + qbytes > 0) {
          mbar_arrive_expect_tx(&S.full[st], 2u * bytes + qbytes);
          if (qbytes) {
            const T* qrow = qbase + static_cast<int64_t>(it.row) * p.q_sr;
            for (int g = 0; g < p.g; ++g)
              bulk_load(S.qs[st] + g * D, qrow + static_cast<int64_t>(it.h * p.g + g) * p.q_sh,
                        D * sizeof(T), &S.full[st]);
          }
          if (paged) {
            // segment i: tile rows [lo, hi) from rows [row0 + lo - i P, ...) of page pid[i]
#pragma unroll 1  // kept rolled: the producer loop must stay small in the instruction cache
            for (int i = 0; i < nseg; ++i) {
              const int32_t id = i == 0 ? pid0 : trow[i];
              if (id >= 0 && id < p.num_pages) {
                const int lo = i == 0 ? 0 : i * p.page_size - row0;
                const int hi = min(valid, (i + 1) * p.page_size - row0);
                const int64_t src = static_cast<int64_t>(id) * p.kv_sb +
                                    static_cast<int64_t>(it.h) * p.kv_sh +
                                    static_cast<int64_t>(row0 + lo - i * p.page_size) * D;
                const uint32_t nb = static_cast<uint32_t>(hi - lo) * D * sizeof(T);
                bulk_load(S.k[st] + lo * D, kbase + src, nb, &S.full[st]);
                bulk_load(S.v[st] + lo * D, vbase + src, nb, &S.full[st]);
              }
            }
          } else if (bytes) {
            bulk_load(S.k[st], kbase + off + static_cast<int64_t>(t) * D, bytes, &S.full[st]);
            bulk_load(S.v[st], vbase + off + static_cast<int64_t>(t) * D, bytes, &S.full[st]);
          }
        } else {
          mbar_arrive(&S.full[st]);
        }
        if (j == read_j && nidx < n_items) nit = p.items[nidx];
      }
      idx = nidx;
      it = nit;
    }
    if (ok) {
      const int st = J % kSimtStages;
      if (mbar_wait(&S.empty[st], ((J / kSimtStages) & 1u) ^ 1u, ctx)) {
        S.meta[st][0] = -1;
        mbar_arrive(&S.full[st]);
        release_work_cursor(&p.hdr->dec_counter, &p.hdr->dec_exit);
        return;
      }
    }
    // aborted: let the copies already issued land before the CTA's shared memory goes away
    for (uint32_t back = 1; back <= kSimtStages && back <= J; ++back) {
      const uint32_t jj = J - back;
      mbar_drain(&S.full[jj % kSimtStages], (jj / kSimtStages) & 1u);
    }
    release_work_cursor(&p.hdr->dec_counter, &p.hdr->dec_exit);
    return;
  }

  // ---------------- consumers: four warps ----------------
  float q[GP][16];
  float acc[GP][C::kDpl];
  float m[GP];
  float lp[C::kSlots];
  DecodeItem it{};
  uint32_t J = 0;
  while (true) {
    const int st = J % kSimtStages;
    // The consumer warps meet at named barriers below, which have no time limit; a warp whose
    // wait timed out must not leave alone, so they vote and leave together.
    const bool ok = mbar_wait(&S.full[st], (J / kSimtStages) & 1u, ctx);
    if (named_bar_or(1, kSimtConsumers, !ok)) break;
    const int idx = S.meta[st][0];
    if (idx < 0) break;
    const int valid = S.meta[st][2];
    const int flags = S.meta[st][3];
    const int buf = J & 1;
    const T* ks = S.k[st];
    const T* vs = S.v[st];

    if (flags & kFirstTile) {
      it = S.item[st];
#pragma unroll
      for (int g = 0; g < GP; ++g) {
        if (g < p.g) {
          const T* qh = S.qs[st] + g * D;
#pragma unroll
          for (int j = 0; j < C::kChunksPerLane; ++j) {
            const int c = (lane % C::kLpt) + j * C::kLpt;
            float x[C::kChunkElems];
            load_chunk<T>(qh + c * C::kChunkElems, x);
#pragma unroll
            for (int e = 0; e < C::kChunkElems; ++e) q[g][j * C::kChunkElems + e] = x[e] * p.scale_log2;
          }
        } else {
#pragma unroll
          for (int e = 0; e < 16; ++e) q[g][e] = 0.f;
        }
        m[g] = -INFINITY;
#pragma unroll
        for (int e = 0; e < C::kDpl; ++e) acc[g][e] = 0.f;
      }
#pragma unroll
      for (int s = 0; s < C::kSlots; ++s) lp[s] = 0.f;
    }

    // ---- q·k: kLpt lanes per key, 128-bit shared loads, shuffle reduction ----
    float wm[GP];
#pragma unroll
    for (int g = 0; g < GP; ++g) wm[g] = -INFINITY;
#pragma unroll
    for (int pass = 0; pass < C::kPasses; ++pass) {
      const int t = pass * C::kTokPerPass + warp * C::kTokPerWarpPass + lane / C::kLpt;
      const bool in = t < valid;
      float dot[GP];
#pragma unroll
      for (int g = 0; g < GP; ++g) dot[g] = 0.f;
      if (in) {
#pragma unroll
        for (int j = 0; j < C::kChunksPerLane; ++j) {
          const int c = (lane % C::kLpt) + j * C::kLpt;
          float x[C::kChunkElems];
          load_chunk<T>(ks + t * D + c * C::kChunkElems, x);
#pragma unroll
          for (int g = 0; g < GP; ++g)
#pragma unroll
            for (int e = 0; e < C::kChunkElems; ++e) dot[g] = fmaf(q[g][j * C::kChunkElems + e], x[e], dot[g]);
        }
      }
#pragma unroll
      for (int o = 1; o < C::kLpt; o <<= 1)
#pragma unroll
        for (int g = 0; g < GP; ++g) dot[g] += __shfl_xor_sync(0xffffffffu, dot[g], o);
#pragma unroll
      for (int g = 0; g < GP; ++g) {
        const float s = in ? dot[g] : -INFINITY;
        wm[g] = fmaxf(wm[g], s);
        if ((lane % C::kLpt) == 0) S.sc[buf][g][t] = s;
      }
    }
#pragma unroll
    for (int g = 0; g < GP; ++g) wm[g] = warp_max_f32(wm[g]);
    if (lane == 0) {
#pragma unroll
      for (int g = 0; g < GP; ++g) S.wmax[buf][warp][g] = wm[g];
    }
    named_bar_sync(1, kSimtConsumers);

    // ---- new running max, probabilities, running sums ----
    float alpha[GP];
    float mnew[GP];
#pragma unroll
    for (int g = 0; g < GP; ++g) {
      float tm = S.wmax[buf][0][g];
#pragma unroll
      for (int w = 1; w < kSimtConsumerWarps; ++w) tm = fmaxf(tm, S.wmax[buf][w][g]);
      mnew[g] = fmaxf(m[g], tm);
      alpha[g] = (mnew[g] == -INFINITY) ? 1.f : fast_exp2(m[g] - mnew[g]);
    }
#pragma unroll
    for (int s = 0; s < C::kSlots; ++s) {
      const int i2 = tid + s * kSimtConsumers;
      if (i2 < GP * C::kTile) {
        const int g = i2 / C::kTile;
        const int t = i2 - g * C::kTile;
        float pv = 0.f;
        if (t < valid && mnew[g] != -INFINITY) pv = fast_exp2(S.sc[buf][g][t] - mnew[g]);
        S.sc[buf][g][t] = pv;
        lp[s] = lp[s] * alpha[g] + pv;
      }
    }
#pragma unroll
    for (int g = 0; g < GP; ++g) m[g] = mnew[g];
    named_bar_sync(1, kSimtConsumers);

    // ---- P·V: each warp a quarter of the keys, each lane kDpl elements of D ----
#pragma unroll
    for (int g = 0; g < GP; ++g)
#pragma unroll
      for (int e = 0; e < C::kDpl; ++e) acc[g][e] *= alpha[g];
    const int tb = warp * C::kTokPerWarpPV;
    const int te = min(valid, tb + C::kTokPerWarpPV);
    for (int t = tb; t < te; ++t) {
      float x[C::kDpl];
      load_vec<T, C::kDpl>(vs + t * D + lane * C::kDpl, x);
#pragma unroll
      for (int g = 0; g < GP; ++g) {
        const float pv = S.sc[buf][g][t];
#pragma unroll
        for (int e = 0; e < C::kDpl; ++e) acc[g][e] = fmaf(pv, x[e], acc[g][e]);
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&S.empty[st]);

    // ---- end of the split: reduce over warps and threads, normalise, write ----
    if (flags & kLastTile) {
#pragma unroll
      for (int s = 0; s < C::kSlots; ++s) {
        const int i2 = tid + s * kSimtConsumers;
        if (i2 < GP * C::kTile) S.lsum[i2] = lp[s];
      }
#pragma unroll
      for (int g = 0; g < GP; ++g)
#pragma unroll
        for (int e = 0; e < C::kDpl; ++e) S.red[warp][g][lane * C::kDpl + e] = acc[g][e];
      named_bar_sync(1, kSimtConsumers);
      for (int g = warp; g < GP; g += kSimtConsumerWarps) {
        float sum = 0.f;
        for (int t = lane; t < C::kTile; t += 32) sum += S.lsum[g * C::kTile + t];
        sum = warp_sum_f32(sum);
        if (lane == 0) S.lfin[g] = sum;
      }
      named_bar_sync(1, kSimtConsumers);
      const bool direct = it.nsplit == 1;
      const int64_t slot = direct ? 0 : static_cast<int64_t>(it.slot);
      for (int i3 = tid; i3 < p.g * D; i3 += kSimtConsumers) {
        const int g = i3 / D;
        const int d = i3 - g * D;
        float o = 0.f;
#pragma unroll
        for (int w = 0; w < kSimtConsumerWarps; ++w) o += S.red[w][g][d];
        const float l = S.lfin[g];
        float mg = -INFINITY;
#pragma unroll
        for (int gg = 0; gg < GP; ++gg) if (gg == g) mg = m[gg];
        const float ov = l > 0.f ? o / l : 0.f;
        const float lse2 = l > 0.f ? mg + log2f(l) : -INFINITY;
        const int hq = it.h * p.g + g;
        if (direct) {
          T* out = static_cast<T*>(p.out) + static_cast<int64_t>(it.row) * p.o_sr +
                   static_cast<int64_t>(hq) * p.o_sh;
          out[d] = from_f32<T>(ov);
          if (d == 0) p.lse[static_cast<int64_t>(it.row) * p.hq + hq] = lse2 * kLn2;
        } else {
          p.part_o[(slot * p.g + g) * D + d] = ov;
          if (d == 0) p.part_lse[slot * p.g + g] = lse2;
        }
      }
      if (!direct)
        finish_split_and_merge<T, (GP * D + 127) / 128>(merge_target(p), it.row, it.h, it.nsplit,
                                                        it.slot - it.split, tid, 1, &S.mflag,
                                                        S.mlse);
      named_bar_sync(1, kSimtConsumers);
    }
    ++J;
  }
}

template <typename T, int D, int GP>
cudaError_t launch_simt_t(const DecodeParams& p, int nctas, cudaStream_t stream) {
  const size_t smem = sizeof(SimtSmem<T, D, GP>) + 128;
  cudaError_t e = cudaFuncSetAttribute(decode_simt_kernel<T, D, GP>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(nctas);
  cfg.blockDim = dim3(kSimtThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, decode_simt_kernel<T, D, GP>, p);
}

template <typename T, int D>
cudaError_t launch_simt_d(const DecodeParams& p, int nctas, cudaStream_t stream) {
  if (p.g <= 1) return launch_simt_t<T, D, 1>(p, nctas, stream);
  if (p.g <= 2) return launch_simt_t<T, D, 2>(p, nctas, stream);
  if (p.g <= 4) return launch_simt_t<T, D, 4>(p, nctas, stream);
  return launch_simt_t<T, D, 8>(p, nctas, stream);
}

}  // namespace

int simt_ctas_per_sm() { return 2; }

cudaError_t launch_decode_simt(const DecodeParams& p, int dtype, int nctas, cudaStream_t stream) {
  if (dtype == FD_F32) {
    return p.d == 64 ? launch_simt_d<float, 64>(p, nctas, stream)
                     : launch_simt_d<float, 128>(p, nctas, stream);
  }
  return p.d == 64 ? launch_simt_d<__nv_bfloat16, 64>(p, nctas, stream)
                   : launch_simt_d<__nv_bfloat16, 128>(p, nctas, stream);
}

}  // namespace fd
