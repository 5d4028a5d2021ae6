// LSE combine: merge the per-split partials of every (row, query head) whose row has more
// than one split.
//
//   M = max_s LSE_s;  w_s = 2^(LSE_s - M);  O = sum_s w_s O_s / sum_s w_s;  LSE = M + log2 sum_s w_s
//
// (partials and LSE_s in base 2; the output LSE is converted to the natural log). This is the
// merge of "大模型推理加速FlashDecoding算法原理与多GPU并行解码实战", section
// "多GPU张量并行扩展下的FlashDecoding实现", read with the per-split sum of exponentials (the
// printed "lse_i" factor) folded into w_s, and the stabilised two-stage reduce that
// "部署落地的工程细节" item 2 asks for: every weight is taken relative to a running maximum and
// at the end to the global one, in fp32, so no term underflows unless it is negligible. Splits with LSE_s = -inf (no visible key)
// get weight 0; a row whose splits are all empty gets O = 0 and LSE = -inf. Every split goes to
// a fixed warp and every merge runs in a fixed order, so results are bitwise reproducible.
//
// Calls with few (row, query head) pairs get one CTA per pair, whose eight warps take interleaved
// splits and merge them online (running max, rescaled sums, eight loads in flight per lane), then
// merge the warps' results in warp order; calls with many pairs get one warp per pair, which
// merges all its splits the same way. Partials of one (row, KV head) group are consecutive slots
// of G query heads each: slot = row_base[row] * Hkv + h * n_row + split, O at [slot][g][d], LSE
// at [slot][g]. The K/V
// stream is loaded with an L2 evict-first policy, so these partials are normally still in L2.
// Launched with programmatic dependent launch: the CTAs become resident while the split kernel
// runs and wait for its completion before reading anything; they let the next kernel start its
// set-up right away.
#include "common.cuh"
#include "internal.h"

namespace fd {

namespace {

constexpr int kCombineWarps = 8;
constexpr int kBatch = 8;  // splits whose loads one warp keeps in flight together
// Calls of at least this many (row, query head) pairs (chunked prefill: every packed row of every
// head) use a warp kernel that keeps 4 splits in flight and 48 registers a thread, for 5 CTAs
// per multiprocessor instead of 3: their pairs have few splits each and fill several waves, so
// more warps in flight beat more loads per warp.
constexpr int64_t kManyPairs = 8192;
// Above this many (row, query head) pairs every warp merges a pair of its own (eight pairs per
// CTA); below, the eight warps of a CTA share one pair's splits.
constexpr int64_t kWarpPerPairMin = 1024;

// Online merge of splits s = first, first + step, ... < n of one (row, query head) by one warp:
// running max m, weight sum wsum, weighted sum acc (kVec elements of D per lane).
template <int kVec, int kB = kBatch>
__device__ __forceinline__ void merge_splits(const float* lse_base, int64_t lse_step,
                                             const float* o_base, int64_t o_step, int n,
                                             int first, int step, float& m, float& wsum,
                                             float (&acc)[kVec]) {
  m = -INFINITY;
  wsum = 0.f;
#pragma unroll
  for (int e = 0; e < kVec; ++e) acc[e] = 0.f;
  for (int s0 = first; s0 < n; s0 += kB * step) {
    float l[kB];
    float x[kB][kVec];
#pragma unroll
    for (int j = 0; j < kB; ++j) {
      const int s = s0 + j * step;
      l[j] = -INFINITY;
#pragma unroll
      for (int e = 0; e < kVec; ++e) x[j][e] = 0.f;
      if (s < n) {
        l[j] = lse_base[s * lse_step];
        const float* o = o_base + s * o_step;
        if constexpr (kVec == 4) {
          const float4 v = *reinterpret_cast<const float4*>(o);
          x[j][0] = v.x; x[j][1] = v.y; x[j][2] = v.z; x[j][3] = v.w;
        } else {
          const float2 v = *reinterpret_cast<const float2*>(o);
          x[j][0] = v.x; x[j][1] = v.y;
        }
      }
    }
    float mn = m;
#pragma unroll
    for (int j = 0; j < kB; ++j) mn = fmaxf(mn, l[j]);
    if (mn == -INFINITY) continue;  // nothing visible yet
    const float scale = fast_exp2(m - mn);  // 0 while m = -inf
    wsum *= scale;
#pragma unroll
    for (int e = 0; e < kVec; ++e) acc[e] *= scale;
#pragma unroll
    for (int j = 0; j < kB; ++j) {
      const float w = fast_exp2(l[j] - mn);  // 0 for an empty split (l = -inf)
      wsum += w;
#pragma unroll
      for (int e = 0; e < kVec; ++e) acc[e] = fmaf(w, x[j][e], acc[e]);
    }
    m = mn;
  }
}

struct PairView {
  int row, hq, n;
  const float* lse_base;
  const float* o_base;  // lane 0's elements
  int64_t lse_step, o_step;
};

template <int D>
__device__ __forceinline__ PairView pair_view(const CombineParams& p, int64_t pair, int lane) {
  PairView v;
  v.row = static_cast<int>(pair / p.hq);
  v.hq = static_cast<int>(pair - static_cast<int64_t>(v.row) * p.hq);
  v.n = p.row_nsplit[v.row];
  const int h = v.hq / p.g, g = v.hq - h * p.g;
  const int64_t slot0 = static_cast<int64_t>(p.row_base[v.row]) * p.hkv + static_cast<int64_t>(h) * v.n;
  v.lse_base = p.part_lse + slot0 * p.g + g;
  v.o_base = p.part_o + (slot0 * p.g + g) * D + lane * (D / 32);
  v.lse_step = p.g;
  v.o_step = static_cast<int64_t>(p.g) * D;
  return v;
}

template <typename T>
__device__ __forceinline__ void write_out(const CombineParams& p, int row, int hq, int d,
                                          float v) {
  T* out = static_cast<T*>(p.out) + static_cast<int64_t>(row) * p.o_sr + static_cast<int64_t>(hq) * p.o_sh;
  out[d] = from_f32<T>(v);
}

// One CTA per (row, query head): the eight warps take interleaved splits, then their results are
// merged in warp order.
template <typename T, int D>
__global__ void __launch_bounds__(kCombineWarps * 32) combine_cta_kernel(CombineParams p) {
  constexpr int kVec = D / 32;
  __shared__ float s_m[kCombineWarps], s_w[kCombineWarps];
  __shared__ float s_acc[kCombineWarps][D];
  // The next call's split kernel may start its set-up (barriers, tensor memory, its own plan)
  // now; it touches the workspace and the outputs only after waiting for this grid.
  pdl_launch_dependents();
  pdl_wait_prerequisites();
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const PairView v = pair_view<D>(p, blockIdx.x, lane);
  if (v.n <= 1) return;  // single split: the split kernel wrote the output directly
  float m, wsum, acc[kVec];
  merge_splits<kVec>(v.lse_base, v.lse_step, v.o_base, v.o_step, v.n, warp, kCombineWarps, m,
                     wsum, acc);
  if (lane == 0) {
    s_m[warp] = m;
    s_w[warp] = wsum;
  }
#pragma unroll
  for (int e = 0; e < kVec; ++e) s_acc[warp][lane * kVec + e] = acc[e];
  __syncthreads();
  float M = -INFINITY;
#pragma unroll
  for (int w = 0; w < kCombineWarps; ++w) M = fmaxf(M, s_m[w]);
  float W = 0.f, ov = 0.f;
  if (M != -INFINITY) {
#pragma unroll
    for (int w = 0; w < kCombineWarps; ++w) {
      const float f = fast_exp2(s_m[w] - M);  // 0 for a warp that saw nothing
      W = fmaf(f, s_w[w], W);
      if (threadIdx.x < D) ov = fmaf(f, s_acc[w][threadIdx.x], ov);
    }
  }
  if (threadIdx.x < D) write_out<T>(p, v.row, v.hq, threadIdx.x, W > 0.f ? ov / W : 0.f);
  if (threadIdx.x == 0)
    p.lse[static_cast<int64_t>(v.row) * p.hq + v.hq] = W > 0.f ? (M + log2f(W)) * kLn2 : -INFINITY;
}

// One warp per (row, query head), eight pairs per CTA: every warp merges all splits of its pair,
// kB at a time.
template <typename T, int D, int kB, int kMinCtas>
__global__ void __launch_bounds__(kCombineWarps * 32, kMinCtas) combine_warp_kernel(CombineParams p) {
  constexpr int kVec = D / 32;
  pdl_launch_dependents();
  pdl_wait_prerequisites();
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int64_t pair = static_cast<int64_t>(blockIdx.x) * kCombineWarps + warp;
  if (pair >= static_cast<int64_t>(p.rows) * p.hq) return;
  const PairView v = pair_view<D>(p, pair, lane);
  if (v.n <= 1) return;
  float m, wsum, acc[kVec];
  merge_splits<kVec, kB>(v.lse_base, v.lse_step, v.o_base, v.o_step, v.n, 0, 1, m, wsum, acc);
  const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
#pragma unroll
  for (int e = 0; e < kVec; ++e) write_out<T>(p, v.row, v.hq, lane * kVec + e, acc[e] * inv);
  if (lane == 0)
    p.lse[static_cast<int64_t>(v.row) * p.hq + v.hq] = wsum > 0.f ? (m + log2f(wsum)) * kLn2 : -INFINITY;
}

template <typename T, int D>
cudaError_t launch_combine_t(const CombineParams& p, int64_t pairs, cudaStream_t stream) {
  const bool per_warp = pairs >= kWarpPerPairMin;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(static_cast<unsigned>(per_warp ? (pairs + kCombineWarps - 1) / kCombineWarps : pairs));
  cfg.blockDim = dim3(kCombineWarps * 32);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (!per_warp) return cudaLaunchKernelEx(&cfg, combine_cta_kernel<T, D>, p);
  return pairs >= kManyPairs ? cudaLaunchKernelEx(&cfg, combine_warp_kernel<T, D, 4, 5>, p)
                             : cudaLaunchKernelEx(&cfg, combine_warp_kernel<T, D, kBatch, 3>, p);
}

}  // namespace

cudaError_t launch_combine(const CombineParams& p, cudaStream_t stream) {
  const int64_t pairs = static_cast<int64_t>(p.rows) * p.hq;
  if (pairs == 0) return cudaSuccess;
  if (pairs > 0x7fffffff) return cudaErrorInvalidConfiguration;
  if (p.dtype == FD_F32)
    return p.d == 64 ? launch_combine_t<float, 64>(p, pairs, stream)
                     : launch_combine_t<float, 128>(p, pairs, stream);
  return p.d == 64 ? launch_combine_t<__nv_bfloat16, 64>(p, pairs, stream)
                   : launch_combine_t<__nv_bfloat16, 128>(p, pairs, stream);
}

}  // namespace fd
