// Device split planners (decode: one CTA; chunked prefill: several CTAs that derive the same
// per-request plan and share the item stores) turn the device-resident lengths into the
// work-item list, the per-row split counts and the partial-slot bases, so a call needs no host
// synchronisation. The arithmetic is plan.h's, shared with the host planner fd_split_plan.
#include "common.cuh"
#include "internal.h"

namespace fd {

namespace {

constexpr int kMaxPlanThreads = 1024;
constexpr int kPlanChunkCtas = 16;  // CTAs of the chunked-prefill planner (see plan_chunk_kernel)

__device__ __forceinline__ int plan_threads() { return static_cast<int>(blockDim.x); }

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
// it; `scratch` holds 33 ints of shared memory.
__device__ void block_exclusive_scan(const int32_t* in, int32_t* out, int n, int* scratch) {
  const int tid = threadIdx.x;
  const int nthr = plan_threads();
  const int per = (n + nthr - 1) / nthr;
  const int lo = tid * per;
  int local = 0;
  for (int i = 0; i < per; ++i)
    if (lo + i < n) local += in[lo + i];
  int incl = warp_incl_scan(local);
  const int warp = tid >> 5;
  if (lane_id() == 31) scratch[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int w = (lane_id() < static_cast<uint32_t>(nthr / 32)) ? scratch[lane_id()] : 0;
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

// The planner's chunk (plan.h, plan_pick_chunk) for the lengths len[0..B) whose sum is `total`;
// entries < 0 are not sequences (chunk mode: requests that are not decode rows). All threads of
// the CTA call it; `sums` holds kPlanWaveChoices zeroed 64-bit counters of shared memory.
__device__ int32_t plan_pick_chunk_block(const int32_t* len, int B, int64_t total, int32_t hkv,
                                         int32_t nctas, unsigned long long* sums) {
  // the candidate chunks and the pick are the same for every thread: computed once (64-bit
  // divisions) and shared
  __shared__ int32_t s_chunks[kPlanWaveChoices];
  __shared__ int32_t s_pick;
  if (threadIdx.x < kPlanWaveChoices)
    s_chunks[threadIdx.x] = plan_chunk_for_waves(total, hkv, nctas, plan_waves(threadIdx.x));
  __syncthreads();
  int32_t chunks[kPlanWaveChoices];
  long long local[kPlanWaveChoices];
#pragma unroll
  for (int i = 0; i < kPlanWaveChoices; ++i) {
    chunks[i] = s_chunks[i];
    local[i] = 0;
  }
  for (int b = threadIdx.x; b < B; b += plan_threads()) {
    if (len[b] < 0) continue;
#pragma unroll
    for (int i = 0; i < kPlanWaveChoices; ++i) local[i] += plan_num_splits(len[b], chunks[i], 0);
  }
#pragma unroll
  for (int i = 0; i < kPlanWaveChoices; ++i) {
    const long long s = warp_sum_i64(local[i]);
    if (lane_id() == 0 && s != 0) atomicAdd(&sums[i], static_cast<unsigned long long>(s));
  }
  __syncthreads();
  // the candidates' costs in parallel, then plan_pick_chunk's choice (the first least cost)
  __shared__ long long s_cost[kPlanWaveChoices];
  if (threadIdx.x < kPlanWaveChoices)
    s_cost[threadIdx.x] = plan_chunk_cost(static_cast<int64_t>(sums[threadIdx.x]),
                                          s_chunks[threadIdx.x], hkv, nctas);
  __syncthreads();
  if (threadIdx.x == 0) {
    int best = 0;
#pragma unroll
    for (int i = 1; i < kPlanWaveChoices; ++i)
      if (s_cost[i] < s_cost[best]) best = i;
    s_pick = s_chunks[best];
  }
  __syncthreads();
  return s_pick;
}

// Decode plan over sequences whose lengths are len[0..B): items in longest-first order.
// `row_of` maps sequence index -> output row (identity for decode calls).
__device__ void plan_decode_body(const PlanParams& p, const int32_t* len_src, int B,
                                 const int32_t* row_of, uint32_t* s_flags) {
  // shared memory sized by the batch: 7 * B + 2 ints
  extern __shared__ int32_t smem[];
  int32_t* s_len = smem;
  int32_t* s_n = s_len + B;
  int32_t* s_key = s_n + B;
  int32_t* s_order = s_key + B;
  int32_t* s_ioff = s_order + B;        // B + 1
  int32_t* s_tmp = s_ioff + B + 1;      // B
  int32_t* s_rbase = s_tmp + B;         // B + 1
  const int kPlanThreads = plan_threads();
  __shared__ int s_scan[33];
  __shared__ unsigned long long s_total;
  __shared__ unsigned long long s_sums[kPlanWaveChoices];
  const int tid = threadIdx.x;

  if (tid == 0) s_total = 0ull;
  if (tid < kPlanWaveChoices) s_sums[tid] = 0ull;
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

  const int32_t chunk = p.fixed > 0 ? 0
                                    : plan_pick_chunk_block(s_len, B, static_cast<int64_t>(s_total),
                                                            p.hkv, p.nctas, s_sums);
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
  // One warp per sequence (in rank order) writes that sequence's items; lanes take splits, so each
  // key range is computed once and written for every KV head (no per-item search or division).
  const int warp = tid >> 5;
  const int lane = static_cast<int>(lane_id());
  for (int r = warp; r < B; r += kPlanThreads / 32) {
    const int b = s_order[r];
    const int32_t n = s_n[b];
    const int32_t L = s_len[b];
    const int32_t first = s_ioff[r];
    const int32_t rbase = s_rbase[b];
    const int row = row_of ? row_of[b] : b;
    for (int32_t s = lane; s < n; s += 32) {
      int32_t t0, t1;
      plan_split_range(L, n, s, p.fixed, p.align, &t0, &t1);
      for (int32_t h = 0; h < p.hkv; ++h) {
        const int32_t i = first + h * n + s;
        if (!overflow) {
          // two 16-byte stores per 32-byte item: scalar stores from lanes 32 bytes apart would
          // throttle this single CTA's load/store unit on partial-sector writes
          int4* dst = reinterpret_cast<int4*>(p.items + i);
          dst[0] = make_int4(row, b, h, s);
          dst[1] = make_int4(t0, t1, n, rbase * p.hkv + h * n + s);
        }
        if (p.out_items && i < p.out_cap) {
          int32_t* o = p.out_items + 5 * static_cast<int64_t>(i);
          o[0] = b; o[1] = h; o[2] = s; o[3] = t0; o[4] = t1;
        }
      }
    }
  }
  // arrival counters of the in-kernel merge start every call at zero
  if (p.arrivals)
    for (int i = tid; i < B * p.hkv; i += kPlanThreads) {
      const int row = row_of ? row_of[i / p.hkv] : i / p.hkv;
      p.arrivals[row * p.hkv + i % p.hkv] = 0;
    }
}

__global__ void __launch_bounds__(kMaxPlanThreads, 1) plan_decode_kernel(PlanParams p) {
  // the split kernel may launch now (programmatic dependent launch); it waits for this grid's
  // completion before it reads the plan
  pdl_launch_dependents();
  __shared__ uint32_t s_flags;
  if (threadIdx.x == 0) s_flags = 0;
  __syncthreads();
  plan_decode_body(p, p.lens, p.B, nullptr, &s_flags);
  __syncthreads();
  if (threadIdx.x == 0 && s_flags) atomicOr(&p.hdr->status, s_flags);
}

// Exclusive prefix sums of K arrays of n ints at once (out[k][n] = the total of in[k]), with
// the three barriers of one scan. All threads of the CTA call it; `scratch` holds 33 * K ints.
template <int K>
__device__ void block_exclusive_scan_k(const int32_t* const* in, int32_t* const* out, int n,
                                       int* scratch) {
  const int tid = threadIdx.x;
  const int nthr = plan_threads();
  const int per = (n + nthr - 1) / nthr;
  const int lo = tid * per;
  const int warp = tid >> 5;
  int local[K], incl[K];
#pragma unroll
  for (int k = 0; k < K; ++k) {
    local[k] = 0;
    for (int i = 0; i < per; ++i)
      if (lo + i < n) local[k] += in[k][lo + i];
    incl[k] = warp_incl_scan(local[k]);
    if (lane_id() == 31) scratch[k * 33 + warp] = incl[k];
  }
  __syncthreads();
  if (warp == 0) {
#pragma unroll
    for (int k = 0; k < K; ++k) {
      const int w = (lane_id() < static_cast<uint32_t>(nthr / 32)) ? scratch[k * 33 + lane_id()] : 0;
      const int wi = warp_incl_scan(w);
      scratch[k * 33 + lane_id()] = wi - w;  // exclusive warp offsets
      if (lane_id() == 31) scratch[k * 33 + 32] = wi;
    }
  }
  __syncthreads();
#pragma unroll
  for (int k = 0; k < K; ++k) {
    int run = scratch[k * 33 + warp] + incl[k] - local[k];
    for (int i = 0; i < per; ++i) {
      if (lo + i < n) {
        out[k][lo + i] = run;
        run += in[k][lo + i];
      }
    }
    if (tid == 0) out[k][n] = scratch[k * 33 + 32];
  }
  __syncthreads();
}

// The largest i in [0, n) with off[i] <= x (off non-decreasing, off[0] <= x): the request (or
// rank) whose range [off[i], off[i + 1]) holds x, skipping empty ranges before it.
__device__ __forceinline__ int owner_of(const int32_t* off, int n, int32_t x) {
  int lo = 0, hi = n;
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (off[mid] <= x) lo = mid; else hi = mid;
  }
  return lo;
}

// Chunked-prefill plan: requests with chunk_len == 1 are decode rows over prefix + 1 keys,
// planned like a decode call over those requests; longer chunks become query tiles of kQTile
// rows whose keys are cut on a fixed kChunkKvSplit grid, items ordered (request, query head,
// split, tile). Every packed row gets its partial slots (its split count and the base of its
// slots, the exclusive sum of the split counts of the rows before it), so the same combine
// merges decode rows and tile rows.
//
// Launched on kPlanChunkCtas CTAs: each CTA derives the whole per-request plan (a few scans over
// the B requests, latency-bound) in its own shared memory, identically, then writes its share
// of the items and row tables, so the item stores, which one multiprocessor would serialise,
// spread over the CTAs. CTA 0 alone writes the header.
__global__ void __launch_bounds__(kMaxPlanThreads, 1) plan_chunk_kernel(PlanParams p) {
  pdl_launch_dependents();
  extern __shared__ int32_t smem[];
  const int B = p.B;
  const int T = p.total_rows;
  const int nthr = plan_threads();
  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = static_cast<int>(lane_id());
  const int g = p.hq / p.hkv;
  // this CTA's share: threads take indices blockIdx.x * nthr + tid, ... (stride gt_step); warps
  // take warp * gridDim.x + blockIdx.x, ... (stride gw_step), so a short warp loop spreads too
  const int gt0 = static_cast<int>(blockIdx.x) * nthr + tid;
  const int gt_step = static_cast<int>(gridDim.x) * nthr;
  const int gw0 = warp * static_cast<int>(gridDim.x) + static_cast<int>(blockIdx.x);
  const int gw_step = static_cast<int>(gridDim.x) * (nthr / 32);
  const bool lead = blockIdx.x == 0;
  int32_t* s_c = smem;                 // chunk rows (>= 0)
  int32_t* s_p = s_c + B;              // prefix, clamped to [0, S_cap]
  int32_t* s_dlen = s_p + B;           // decode length (0 for tile requests)
  int32_t* s_n = s_dlen + B;           // decode splits
  int32_t* s_key = s_n + B;            // decode ordering key; then the rank-ordered item counts
  int32_t* s_order = s_key + B;        // decode requests, longest first
  int32_t* s_tcnt = s_order + B;       // tile items per request
  int32_t* s_nmax = s_tcnt + B;        // key splits of a multi-tile request's last query tile
  int32_t* s_slots = s_nmax + B;       // partial slots of the request's rows
  int32_t* s_roff = s_slots + B;       // B + 1: first packed row of each request
  int32_t* s_dioff = s_roff + B + 1;   // B + 1: decode item offsets (rank order)
  int32_t* s_tioff = s_dioff + B + 1;  // B + 1: tile item offsets (request order)
  int32_t* s_soff = s_tioff + B + 1;   // B + 1: first (request, split) pair of each request
  int32_t* s_rb = s_soff + B + 1;      // B + 1: partial-slot base of each request's first row
  __shared__ int s_scan[3 * 33];
  __shared__ unsigned long long s_total;
  __shared__ unsigned long long s_key_tiles;  // 128-key tiles of all tile items
  __shared__ unsigned long long s_sums[kPlanWaveChoices];
  __shared__ uint32_t s_flags;
  __shared__ int s_ndec;
  if (tid == 0) { s_total = 0ull; s_key_tiles = 0ull; s_flags = 0u; s_ndec = 0; }
  if (tid < kPlanWaveChoices) s_sums[tid] = 0ull;
  __syncthreads();

  if (B <= 32) {
    // Up to 32 requests: one warp derives the same per-request plan as the block path below, a
    // request per lane, with shuffles in place of barrier-separated phases (each ~2 µs of
    // latency there: loads, block scans, the chunk choice, the ranking).
    if (warp == 0) {
      const bool has = lane < B;
      const int32_t raw_p = has ? p.lens[lane] : 0, raw_c = has ? p.chunk_lens[lane] : 0;
      const int32_t c = raw_c < 0 ? 0 : raw_c;
      const int32_t pp = clamp_len(raw_p, p.cap);
      const bool clamped =
          has && (raw_c < 0 || pp != raw_p || static_cast<int64_t>(pp) + c > p.cap);
      const bool dec = has && c == 1;
      const int32_t dlen = dec ? clamp_len(static_cast<int64_t>(pp) + 1, p.cap) : 0;
      int32_t cnt = 0, slots = 0;
      long long ktiles = 0;
      if (has && c > 1) {
        for (int32_t t = 0; t * kQTile < c; ++t) {
          const int32_t kt = chunk_tile_keys(pp, c, t, p.cap);
          const int32_t nt = chunk_tile_splits(kt);
          cnt += nt;
          slots += min(kQTile, c - t * kQTile) * nt;
          ktiles += cdiv64(kt, kQTile);
        }
        const int32_t nheads = chunk_packed(c, g) ? p.hkv : p.hq;
        cnt *= nheads;
        ktiles *= nheads;
      }
      const int32_t nmax =
          (has && c > kQTile) ? chunk_tile_splits(chunk_tile_keys(pp, c, (c - 1) / kQTile, p.cap)) : 0;
      const long long total = warp_sum_i64(dlen);
      const long long key_tiles = warp_sum_i64(ktiles);
      const uint32_t dmask = __ballot_sync(0xffffffffu, dec);
      const int nd = __popc(dmask);
      // the decode rows' chunk (plan_pick_chunk over their lengths)
      int32_t chunks[kPlanWaveChoices];
      int64_t sums[kPlanWaveChoices];
#pragma unroll
      for (int i = 0; i < kPlanWaveChoices; ++i) {
        chunks[i] = plan_chunk_for_waves(total, p.hkv, p.nctas, plan_waves(i));
        sums[i] = warp_sum_i64(dec ? plan_num_splits(dlen, chunks[i], 0) : 0);
      }
      const int32_t chunk = plan_pick_chunk(chunks, sums, p.hkv, p.nctas);
      const int32_t n = dec ? plan_num_splits(dlen, chunk, 0) : 0;
      const int32_t key = dec ? plan_sort_key(dlen, n) : -1;
      if (dec) slots = n;
      // longest-first rank among the decode requests (stable) and the first decode item of the
      // request in rank order
      int r = 0, ioff = 0;
      for (int j = 0; j < 32; ++j) {
        const int32_t kj = __shfl_sync(0xffffffffu, key, j);
        const int32_t nj = __shfl_sync(0xffffffffu, n, j);
        const bool before = ((dmask >> j) & 1u) && (kj > key || (kj == key && j < lane));
        r += before ? 1 : 0;
        ioff += before ? nj * p.hkv : 0;
      }
      const int dec_items = static_cast<int>(warp_sum_i64(n * p.hkv));
      // exclusive scans over the requests: rows, tile items, (request, split) pairs, slots
      const int i_c = warp_incl_scan(c), i_t = warp_incl_scan(cnt), i_s = warp_incl_scan(nmax);
      const int i_r = warp_incl_scan(slots);
      if (has) {
        s_c[lane] = c;
        s_p[lane] = pp;
        s_dlen[lane] = dlen;
        s_n[lane] = n;
        s_tcnt[lane] = cnt;
        s_nmax[lane] = nmax;
        s_slots[lane] = slots;
        s_roff[lane] = i_c - c;
        s_tioff[lane] = i_t - cnt;
        s_soff[lane] = i_s - nmax;
        s_rb[lane] = i_r - slots;
        if (dec) {
          s_order[r] = lane;
          s_dioff[r] = ioff;
        }
      }
      for (int j = nd + lane; j <= B; j += 32) s_dioff[j] = dec_items;
      const bool any_clamped = __any_sync(0xffffffffu, clamped);
      if (lane == B - 1) {
        s_roff[B] = i_c;
        s_tioff[B] = i_t;
        s_soff[B] = i_s;
        s_rb[B] = i_r;
      }
      if (lane == 0) {
        s_total = static_cast<unsigned long long>(total);
        s_key_tiles = static_cast<unsigned long long>(key_tiles);
        s_ndec = nd;
        if (any_clamped) s_flags = FD_FLAG_LEN_CLAMPED;
      }
    }
    __syncthreads();
  } else {
    // per request: what does not depend on the decode rows' chunk
    long long local = 0;
    int ndec = 0;
    for (int b = tid; b < B; b += nthr) {
      const int32_t raw_p = p.lens[b], raw_c = p.chunk_lens[b];
      const int32_t c = raw_c < 0 ? 0 : raw_c;
      const int32_t pp = clamp_len(raw_p, p.cap);
      if (raw_c < 0 || pp != raw_p || static_cast<int64_t>(pp) + c > p.cap)
        atomicOr(&s_flags, FD_FLAG_LEN_CLAMPED);
      const int32_t dlen = c == 1 ? clamp_len(static_cast<int64_t>(pp) + 1, p.cap) : 0;
      s_c[b] = c;
      s_p[b] = pp;
      s_dlen[b] = dlen;
      s_key[b] = c == 1 ? dlen : -1;  // the decode rows' lengths, for the chunk choice below
      int32_t cnt = 0, slots = 0;
      int64_t ktiles = 0;
      if (c > 1) {
        for (int32_t t = 0; t * kQTile < c; ++t) {
          const int32_t kt = chunk_tile_keys(pp, c, t, p.cap);
          const int32_t nt = chunk_tile_splits(kt);
          cnt += nt;
          slots += min(kQTile, c - t * kQTile) * nt;
          ktiles += cdiv64(kt, kQTile);  // the split grid is a multiple of the key tile
        }
        const int32_t nheads = chunk_packed(c, g) ? p.hkv : p.hq;
        atomicAdd(&s_key_tiles, static_cast<unsigned long long>(ktiles * nheads));
        cnt *= nheads;
      }
      s_tcnt[b] = cnt;
      s_slots[b] = slots;  // decode rows: their split count, once the chunk is known
      // (request, split) pairs of the requests of more than one query tile; single-tile requests
      // have their items written one per thread
      s_nmax[b] = c > kQTile ? chunk_tile_splits(chunk_tile_keys(pp, c, (c - 1) / kQTile, p.cap)) : 0;
      local += dlen;
      ndec += c == 1 ? 1 : 0;
    }
    local = warp_sum_i64(local);
    if (lane == 0 && local != 0) atomicAdd(&s_total, static_cast<unsigned long long>(local));
    if (ndec) atomicAdd(&s_ndec, ndec);
    __syncthreads();
    {
      const int32_t* in[3] = {s_c, s_tcnt, s_nmax};
      int32_t* out[3] = {s_roff, s_tioff, s_soff};
      block_exclusive_scan_k<3>(in, out, B, s_scan);
    }

    const int32_t chunk =
        plan_pick_chunk_block(s_key, B, static_cast<int64_t>(s_total), p.hkv, p.nctas, s_sums);
    for (int b = tid; b < B; b += nthr) {
      if (s_c[b] == 1) {
        const int32_t n = plan_num_splits(s_dlen[b], chunk, 0);
        s_n[b] = n;
        s_key[b] = plan_sort_key(s_dlen[b], n);
        s_slots[b] = n;
      } else {
        s_n[b] = 0;
        s_key[b] = -1;
      }
    }
    __syncthreads();
    // decode requests longest first (stable counting rank among decode requests)
    for (int b = tid; b < B; b += nthr) {
      if (s_c[b] != 1) continue;
      const int32_t kb = s_key[b];
      int r = 0;
      for (int j = 0; j < B; ++j) {
        const int32_t kj = s_key[j];
        r += (s_c[j] == 1 && (kj > kb || (kj == kb && j < b))) ? 1 : 0;
      }
      s_order[r] = b;
    }
    __syncthreads();
    const int ndb = s_ndec;
    // the keys are consumed: s_key now holds the item counts in rank order (zero past the last)
    for (int r = tid; r < B; r += nthr) s_key[r] = r < ndb ? s_n[s_order[r]] * p.hkv : 0;
    __syncthreads();
    {
      const int32_t* in[2] = {s_key, s_slots};
      int32_t* out[2] = {s_dioff, s_rb};
      block_exclusive_scan_k<2>(in, out, B, s_scan);
    }
  }
  const int nd = s_ndec;
  // chunk lengths that do not add up to the packed rows of q_chunk: nothing is computed (the
  // outputs are left as they were) and the status word says why
  const bool inconsistent = s_roff[B] != T;
  const int32_t n_dec_items = s_dioff[B];
  const int32_t n_tile_items = s_tioff[B];
  const bool overflow =
      inconsistent || n_dec_items > p.max_dec_items || n_tile_items > p.max_tile_items;

  // split count and partial-slot base of every packed row: a decode row has its request's n
  // slots (1 when it merges inside its split kernel: the combine skips it); row j of a tile
  // request sits in query tile t = j / kQTile, after the full tiles before it, with nt(t) slots
  for (int r = gt0; r < T; r += gt_step) {
    if (inconsistent) {
      p.row_nsplit[r] = 0;
      p.row_base[r] = 0;
      continue;
    }
    const int b = owner_of(s_roff, B, r);
    const int32_t c = s_c[b], j = r - s_roff[b];
    int32_t nsplit, base = s_rb[b];
    if (c == 1) {
      nsplit = p.decode_merged_in_kernel ? 1 : s_n[b];
    } else {
      const int32_t t = j / kQTile;
      for (int32_t u = 0; u < t; ++u) base += kQTile * chunk_tile_splits(chunk_tile_keys(s_p[b], c, u, p.cap));
      nsplit = chunk_tile_splits(chunk_tile_keys(s_p[b], c, t, p.cap));
      base += (j - t * kQTile) * nsplit;
    }
    p.row_nsplit[r] = nsplit;
    p.row_base[r] = base;
  }
  // decode items, one per thread: item i of rank r's request is (head e / n, split e mod n),
  // e = i - first, so item (h, s) sits at first + h n + s
  for (int i = gt0; i < (overflow ? 0 : n_dec_items); i += gt_step) {
    const int r = owner_of(s_dioff, nd, i);
    const int b = s_order[r];
    const int32_t n = s_n[b], e = i - s_dioff[r];
    const int32_t h = e / n, s = e - h * n;
    int32_t t0, t1;
    plan_split_range(s_dlen[b], n, s, 0, p.align, &t0, &t1);
    int4* dst = reinterpret_cast<int4*>(p.items + i);
    dst[0] = make_int4(s_roff[b], b, h, s);
    dst[1] = make_int4(t0, t1, n, s_rb[b] * p.hkv + h * n + s);
  }
  // tile items of single-tile requests (2 <= c <= 128 rows: verification steps, short chunks):
  // one thread per item. Item e of the request is head e / n, split e mod n (n splits).
  for (int i = gt0; i < (overflow ? 0 : n_tile_items); i += gt_step) {
    const int b = owner_of(s_tioff, B, i);
    const int32_t c = s_c[b];
    if (c > kQTile) continue;  // written below, per (request, split) pair
    const int32_t pp = s_p[b];
    const int32_t kt = chunk_tile_keys(pp, c, 0, p.cap);
    const int32_t nt = chunk_tile_splits(kt);
    const int32_t e = i - s_tioff[b];
    const int32_t h = e / nt, s = e - h * nt;
    const int32_t k0 = min(s * kChunkKvSplit, kt), k1 = min((s + 1) * kChunkKvSplit, kt);
    int4* dst = reinterpret_cast<int4*>(p.tiles + i);
    dst[0] = make_int4(b, h, s, nt);
    dst[1] = make_int4(k0, k1, s_roff[b], 0);
    dst[2] = make_int4(c, pp, s_rb[b] * p.hkv, chunk_packed(c, g) ? 1 : 0);
    dst[3] = make_int4(0, 0, 0, 0);
  }
  // tile items of longer requests: one warp per (request, split) pair, lanes over query heads
  // (KV heads for head-packed tiles). Per head the items run split by split and, within a
  // split, tile by tile over the query tiles that see that split's keys.
  const int32_t n_pairs = s_soff[B];
  for (int k = gw0; k < (overflow ? 0 : n_pairs); k += gw_step) {
    const int b = owner_of(s_soff, B, k);
    const int32_t s = k - s_soff[b];
    const int32_t c = s_c[b], pp = s_p[b], r0 = s_roff[b];
    const int32_t ntiles = (c + kQTile - 1) / kQTile;
    const int32_t head_packed = chunk_packed(c, g) ? 1 : 0;
    const int32_t nheads = head_packed ? p.hkv : p.hq;
    const int32_t per_head = s_tcnt[b] / nheads;
    // items of the earlier splits in each head's run: query tile t has min(nt(t), s) of them
    int32_t before = 0;
    for (int32_t t = 0; t < ntiles; ++t)
      before += min(chunk_tile_splits(chunk_tile_keys(pp, c, t, p.cap)), s);
    // the bases of the request's later tiles follow from its first row's: every row of tile t
    // has nt(t) slots and the tiles before the last are full
    const int32_t rb0 = s_rb[b];
    for (int32_t h = lane; h < nheads; h += 32) {
      int32_t i = s_tioff[b] + h * per_head + before;
      int32_t next_base = rb0;
      for (int32_t t = 0; t < ntiles; ++t) {
        const int32_t kt = chunk_tile_keys(pp, c, t, p.cap);
        const int32_t nt = chunk_tile_splits(kt);
        const int32_t tbase = next_base;  // row_base of tile t's first row
        next_base += kQTile * nt;
        if (s >= nt) continue;
        const int32_t row0 = r0 + t * kQTile;
        const int32_t rows = min(kQTile, c - t * kQTile);
        const int32_t k0 = min(s * kChunkKvSplit, kt), k1 = min((s + 1) * kChunkKvSplit, kt);
        int4* dst = reinterpret_cast<int4*>(p.tiles + i);
        dst[0] = make_int4(b, h, s, nt);
        dst[1] = make_int4(k0, k1, row0, t * kQTile);
        dst[2] = make_int4(rows, pp, tbase * p.hkv, head_packed);
        dst[3] = make_int4(0, 0, 0, 0);
        ++i;
      }
    }
  }
  // the split kernels' completion counters of the decode rows
  for (int e = gt0; e < (inconsistent ? 0 : nd * p.hkv); e += gt_step) {
    const int r = e / p.hkv, h = e - r * p.hkv;
    p.arrivals[s_roff[s_order[r]] * p.hkv + h] = 0;
  }
  if (!lead) return;
  if (warp == 0) {
    // the tile kernel's CTAs: the n of least chunk_tile_cost, smallest on ties; lane l weighs
    // n = l + 1, l + 33, ... and the warp keeps the lexicographic minimum of (cost, n)
    const int64_t key_tiles = static_cast<int64_t>(s_key_tiles);
    const int64_t dec_bytes = static_cast<int64_t>(s_total) * p.kv_key_bytes;
    const int32_t nsm = p.tile_sms;
    int32_t n_best;
    if (overflow || key_tiles <= 0) {
      n_best = 0;
    } else if (dec_bytes <= 0 || nsm <= 1) {
      n_best = nsm;
    } else {
      const float dec = static_cast<float>(dec_bytes);
      float t_best = 0.f;
      n_best = 0;
      for (int32_t n = lane + 1; n <= nsm; n += 32) {
        const float t = chunk_tile_cost(key_tiles, dec, nsm, n);
        if (n_best == 0 || t < t_best) { t_best = t; n_best = n; }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const float t2 = __shfl_xor_sync(0xffffffffu, t_best, o);
        const int32_t n2 = __shfl_xor_sync(0xffffffffu, n_best, o);
        const bool take = n2 != 0 && (n_best == 0 || t2 < t_best || (t2 == t_best && n2 < n_best));
        if (take) { t_best = t2; n_best = n2; }
      }
    }
    if (lane == 0) p.hdr->tile_ctas = n_best;
  }
  if (tid == 0) {
    p.row_base[T] = inconsistent ? 0 : s_rb[B];
    p.hdr->num_dec_items = overflow ? 0 : n_dec_items;
    p.hdr->num_tile_items = overflow ? 0 : n_tile_items;
    p.hdr->dec_counter = 0;
    p.hdr->tile_counter = 0;
    uint32_t f = s_flags | (inconsistent ? FD_FLAG_LEN_CLAMPED : 0u) | (overflow ? FD_FLAG_PLAN_OVERFLOW : 0u);
    if (f) atomicOr(&p.hdr->status, f);
  }
}

}  // namespace

cudaError_t launch_plan_chunk(const PlanParams& p, cudaStream_t stream) {
  const size_t smem = sizeof(int32_t) * (14 * static_cast<size_t>(p.B) + 5);
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(plan_chunk_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
  }
  plan_chunk_kernel<<<kPlanChunkCtas, kMaxPlanThreads, smem, stream>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_plan_decode(const PlanParams& p, cudaStream_t stream) {
  const size_t smem = sizeof(int32_t) * (7 * static_cast<size_t>(p.B) + 2);
  const int threads = kMaxPlanThreads;
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(plan_decode_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
  }
  plan_decode_kernel<<<1, threads, smem, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace fd
