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
// One CTA per (row, query head): its eight warps take interleaved splits and merge them online
// (running max, rescaled sums), eight loads in flight per lane, then the warps' results are merged
// in warp order. Partials of one (row, KV head) group are consecutive slots of G query heads each:
// slot = row_base[row] * Hkv + h * n_row + split, O at [slot][g][d], LSE at [slot][g]. The K/V
// stream is loaded with an L2 evict-first policy, so these partials are normally still in L2.
// Launched with programmatic dependent launch: the CTAs become resident while the split kernel
// runs and wait for its completion before reading anything; they let the next kernel start its
// set-up right away.
#include "common.cuh"
#include "internal.h"

namespace fd {

namespace {

constexpr int kCombineWarps = 8;  // one CTA per (row, query head); warp w takes splits w, w + 8, ...
constexpr int kBatch = 8;         // splits whose loads one warp keeps in flight together

template <typename T, int D>
__global__ void __launch_bounds__(kCombineWarps * 32) combine_kernel(CombineParams p) {
  constexpr int kVec = D / 32;  // elements per lane
  __shared__ float s_m[kCombineWarps], s_w[kCombineWarps];
  __shared__ float s_acc[kCombineWarps][D];
  // The next call's split kernel may start its set-up (barriers, tensor memory, its own plan)
  // now; it touches the workspace and the outputs only after waiting for this grid.
  pdl_launch_dependents();
  pdl_wait_prerequisites();
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int row = static_cast<int>(blockIdx.x / static_cast<unsigned>(p.hq));
  const int hq = static_cast<int>(blockIdx.x - static_cast<unsigned>(row) * p.hq);
  const int n = p.row_nsplit[row];
  if (n <= 1) return;  // single split: the split kernel wrote the output directly
  const int h = hq / p.g, g = hq - h * p.g;
  const int64_t slot0 = static_cast<int64_t>(p.row_base[row]) * p.hkv + static_cast<int64_t>(h) * n;
  const float* lse_base = p.part_lse + slot0 * p.g + g;
  const float* o_base = p.part_o + (slot0 * p.g + g) * D + lane * kVec;
  const int64_t lse_step = p.g;
  const int64_t o_step = static_cast<int64_t>(p.g) * D;

  // this warp's splits, merged online: running max m, weight sum w, weighted sum acc
  float m = -INFINITY, wsum = 0.f;
  float acc[kVec];
#pragma unroll
  for (int e = 0; e < kVec; ++e) acc[e] = 0.f;
  for (int s0 = warp; s0 < n; s0 += kBatch * kCombineWarps) {
    float l[kBatch];
    float x[kBatch][kVec];
#pragma unroll
    for (int j = 0; j < kBatch; ++j) {
      const int s = s0 + j * kCombineWarps;
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
    for (int j = 0; j < kBatch; ++j) mn = fmaxf(mn, l[j]);
    if (mn == -INFINITY) continue;  // nothing visible yet
    const float scale = fast_exp2(m - mn);  // 0 while m = -inf
    wsum *= scale;
#pragma unroll
    for (int e = 0; e < kVec; ++e) acc[e] *= scale;
#pragma unroll
    for (int j = 0; j < kBatch; ++j) {
      const float w = fast_exp2(l[j] - mn);  // 0 for an empty split (l = -inf)
      wsum += w;
#pragma unroll
      for (int e = 0; e < kVec; ++e) acc[e] = fmaf(w, x[j][e], acc[e]);
    }
    m = mn;
  }
  if (lane == 0) {
    s_m[warp] = m;
    s_w[warp] = wsum;
  }
#pragma unroll
  for (int e = 0; e < kVec; ++e) s_acc[warp][lane * kVec + e] = acc[e];
  __syncthreads();

  // merge the warps' results in warp order
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
  T* out = static_cast<T*>(p.out) + static_cast<int64_t>(row) * p.o_sr + static_cast<int64_t>(hq) * p.o_sh;
  if (threadIdx.x < D) out[threadIdx.x] = from_f32<T>(W > 0.f ? ov / W : 0.f);
  if (threadIdx.x == 0)
    p.lse[static_cast<int64_t>(row) * p.hq + hq] = W > 0.f ? (M + log2f(W)) * kLn2 : -INFINITY;
}

template <typename T, int D>
cudaError_t launch_combine_t(const CombineParams& p, unsigned grid, cudaStream_t stream) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kCombineWarps * 32);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, combine_kernel<T, D>, p);
}

}  // namespace

cudaError_t launch_combine(const CombineParams& p, cudaStream_t stream) {
  const int64_t pairs = static_cast<int64_t>(p.rows) * p.hq;
  if (pairs == 0) return cudaSuccess;
  if (pairs > 0x7fffffff) return cudaErrorInvalidConfiguration;
  const unsigned grid = static_cast<unsigned>(pairs);
  if (p.dtype == FD_F32)
    return p.d == 64 ? launch_combine_t<float, 64>(p, grid, stream)
                     : launch_combine_t<float, 128>(p, grid, stream);
  return p.d == 64 ? launch_combine_t<__nv_bfloat16, 64>(p, grid, stream)
                   : launch_combine_t<__nv_bfloat16, 128>(p, grid, stream);
}

}  // namespace fd
