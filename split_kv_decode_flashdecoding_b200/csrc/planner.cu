// Device split planner: one CTA turns the device-resident lengths into the work-item list, the
// per-row split counts and the partial-slot bases, so a call needs no host synchronisation.
// The arithmetic is plan.h's, shared with the host planner fd_split_plan.
#include "common.cuh"
#include "internal.h"

namespace fd {

namespace {

constexpr int kPlanThreads = 1024;

__device__ __forceinline__ long long warp_sum_i64(long long v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ int warp_incl_scan(int v) {
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int n = __shfl_up_sync(0xffffffffu, v, o);
    if (lane_id() >= static_cast<uint32_t>(o)) v += n;
  }
  return v;
}

// Exclusive prefix sum of in[0..n) into out[0..n], out[n] = total. All threads of the CTA call
// it; `scratch` holds 33 ints of shared memory. n <= 4 * kPlanThreads.
__device__ void block_exclusive_scan(const int32_t* in, int32_t* out, int n, int* scratch) {
  const int tid = threadIdx.x;
  const int per = (n + kPlanThreads - 1) / kPlanThreads;
  const int lo = tid * per;
  int local = 0;
  for (int i = 0; i < per; ++i)
    if (lo + i < n) local += in[lo + i];
  int incl = warp_incl_scan(local);
  const int warp = tid >> 5;
  if (lane_id() == 31) scratch[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int w = (lane_id() < kPlanThreads / 32) ? scratch[lane_id()] : 0;
    int wi = warp_incl_scan(w);
    scratch[lane_id()] = wi - w;  // exclusive warp offsets
    if (lane_id() == 31) scratch[32] = wi;
  }
  __syncthreads();
  int run = scratch[warp] + incl - local;
  for (int i = 0; i < per; ++i) {
    if (lo + i < n) {
      out[lo + i] = run;
      run += in[lo + i];
    }
  }
  if (tid == 0) out[n] = scratch[32];
  __syncthreads();
}

// Decode plan over sequences whose lengths are len[0..B): items in longest-first order.
// `row_of` maps sequence index -> output row (identity for decode calls).
__device__ void plan_decode_body(const PlanParams& p, const int32_t* len_src, int B,
                                 const int32_t* row_of, uint32_t* s_flags) {
  extern __shared__ int32_t smem[];
  int32_t* s_len = smem;
  int32_t* s_n = s_len + kMaxPlanBatch;
  int32_t* s_key = s_n + kMaxPlanBatch;
  int32_t* s_order = s_key + kMaxPlanBatch;
  int32_t* s_ioff = s_order + kMaxPlanBatch;        // kMaxPlanBatch + 1
  int32_t* s_tmp = s_ioff + kMaxPlanBatch + 1;      // kMaxPlanBatch
  int32_t* s_rbase = s_tmp + kMaxPlanBatch;         // kMaxPlanBatch + 1
  __shared__ int s_scan[33];
  __shared__ unsigned long long s_total;
  const int tid = threadIdx.x;

  if (tid == 0) s_total = 0ull;
  __syncthreads();
  long long local = 0;
  uint32_t clamped = 0;
  for (int b = tid; b < B; b += kPlanThreads) {
    const int32_t raw = len_src[b];
    const int32_t L = clamp_len(raw, p.cap);
    clamped |= (L != raw) ? 1u : 0u;
    s_len[b] = L;
    local += L;
  }
  local = warp_sum_i64(local);
  if (lane_id() == 0 && local != 0) atomicAdd(&s_total, static_cast<unsigned long long>(local));
  if (clamped) atomicOr(s_flags, FD_FLAG_LEN_CLAMPED);
  __syncthreads();

  const int32_t chunk =
      p.fixed > 0 ? 0 : plan_chunk_tokens(static_cast<int64_t>(s_total), p.hkv, p.nctas);
  for (int b = tid; b < B; b += kPlanThreads) {
    const int32_t n = plan_num_splits(s_len[b], chunk, p.fixed);
    s_n[b] = n;
    s_key[b] = plan_sort_key(s_len[b], n);
  }
  __syncthreads();
  // Longest first: rank = number of sequences with a larger key, or an equal key and a smaller
  // index. A stable counting rank, deterministic for any B.
  for (int b = tid; b < B; b += kPlanThreads) {
    const int32_t kb = s_key[b];
    int r = 0;
    for (int j = 0; j < B; ++j) {
      const int32_t kj = s_key[j];
      r += (kj > kb || (kj == kb && j < b)) ? 1 : 0;
    }
    s_order[r] = b;
  }
  __syncthreads();
  // items per sequence in rank order, and split counts in row order
  for (int r = tid; r < B; r += kPlanThreads) s_tmp[r] = s_n[s_order[r]] * p.hkv;
  __syncthreads();
  block_exclusive_scan(s_tmp, s_ioff, B, s_scan);
  block_exclusive_scan(s_n, s_rbase, B, s_scan);

  const int32_t total_items = s_ioff[B];
  const bool overflow = total_items > p.max_dec_items;
  if (tid == 0) {
    p.hdr->num_dec_items = overflow ? 0 : total_items;
    p.hdr->dec_counter = 0;
    if (overflow) atomicOr(s_flags, FD_FLAG_PLAN_OVERFLOW);
    if (p.out_total) *p.out_total = total_items;
  }
  for (int b = tid; b < B; b += kPlanThreads) {
    const int row = row_of ? row_of[b] : b;
    p.row_nsplit[row] = s_n[b];
    p.row_base[row] = s_rbase[b];
    if (p.out_splits) p.out_splits[b] = s_n[b];
  }
  for (int i = tid; i < total_items; i += kPlanThreads) {
    // the sequence whose item range holds i: largest r with s_ioff[r] <= i
    int lo = 0, hi = B - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (s_ioff[mid] <= i) lo = mid; else hi = mid - 1;
    }
    const int b = s_order[lo];
    const int32_t n = s_n[b];
    const int32_t local_i = i - s_ioff[lo];
    const int32_t h = local_i / n;
    const int32_t s = local_i - h * n;
    int32_t t0, t1;
    plan_split_range(s_len[b], n, s, p.fixed, &t0, &t1);
    if (!overflow) {
      DecodeItem it;
      it.row = row_of ? row_of[b] : b;
      it.b = b;
      it.h = h;
      it.split = s;
      it.t0 = t0;
      it.t1 = t1;
      it.nsplit = n;
      it.seqlen = s_len[b];
      p.items[i] = it;
    }
    if (p.out_items && i < p.out_cap) {
      int32_t* o = p.out_items + 5 * static_cast<int64_t>(i);
      o[0] = b; o[1] = h; o[2] = s; o[3] = t0; o[4] = t1;
    }
  }
}

__global__ void __launch_bounds__(kPlanThreads, 1) plan_decode_kernel(PlanParams p) {
  __shared__ uint32_t s_flags;
  if (threadIdx.x == 0) s_flags = 0;
  __syncthreads();
  plan_decode_body(p, p.lens, p.B, nullptr, &s_flags);
  __syncthreads();
  if (threadIdx.x == 0 && s_flags) atomicOr(&p.hdr->status, s_flags);
}

}  // namespace

size_t plan_smem_bytes() { return sizeof(int32_t) * (7 * static_cast<size_t>(kMaxPlanBatch) + 2); }

cudaError_t launch_plan_decode(const PlanParams& p, cudaStream_t stream) {
  const size_t smem = plan_smem_bytes();
  cudaError_t e = cudaFuncSetAttribute(plan_decode_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  plan_decode_kernel<<<1, kPlanThreads, smem, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace fd
