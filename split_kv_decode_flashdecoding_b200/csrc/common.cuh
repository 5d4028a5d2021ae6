// Device primitives shared by the kernels: mbarriers with bounded waits, TMA / bulk copies,
// tcgen05 (tensor memory + UMMA) wrappers, and small numeric helpers. sm_100a only.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "plan.h"

namespace fd {

// A wait longer than this is treated as a hang: the kernel raises FD_FLAG_WAIT_TIMEOUT in the
// workspace status word and its roles leave their loops instead of spinning forever.
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t global_timer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ uint32_t lane_id() { return threadIdx.x & 31u; }

// ---- mbarrier ---------------------------------------------------------------------------------

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
               : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Where a timed-out wait reports itself.
struct WaitCtx {
  volatile int* abort_flag;  // shared memory: set once any wait in the CTA has timed out
  uint32_t* status;          // global workspace status word (FD_FLAG_*)
};

// Wait until the phase with the given parity of `bar` has completed; give up after
// kWaitLimitNs, raising FD_FLAG_WAIT_TIMEOUT and the CTA's abort flag. The decision depends only
// on the barrier and this thread's own clock, never on other threads: a phase that never
// completes makes every thread waiting on it give up at the same program point, so threads of
// one role cannot split between leaving the loop and entering a named barrier.
//
// Only the first try is inlined; the polling loop with its clock reads is one out-of-line copy.
// The warp-specialised kernels wait at ~40 sites, and with the loop inlined at each their hot
// code outgrew the instruction cache: measured on B200 at the 70B-like shape, out-of-line
// polling took the E4M3 call from 258 to 226 us, 16-key pages from 386 to 335 us and the mixed
// chunk step from 513 to 470 us (warps of different roles run different loops at once, so the
// cache must hold all of them).
static __device__ __noinline__ bool mbar_wait_poll(uint64_t* bar, uint32_t parity, WaitCtx ctx) {
  const uint64_t t0 = global_timer_ns();
  for (uint32_t i = 1;; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((i & 63u) == 0 && global_timer_ns() - t0 > kWaitLimitNs) {
      *ctx.abort_flag = 1;
      atomicOr(ctx.status, FD_FLAG_WAIT_TIMEOUT);
      return false;
    }
  }
}
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, const WaitCtx& ctx) {
  if (mbar_try_wait(bar, parity)) return true;
  return mbar_wait_poll(bar, parity, ctx);
}

// Bounded wait used only while draining after an abort: never sets flags. Out of line, as the
// polling loop above.
static __device__ __noinline__ void mbar_drain(uint64_t* bar, uint32_t parity) {
  const uint64_t t0 = global_timer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (global_timer_ns() - t0 > kWaitLimitNs) return;
  }
}

// Called by one thread per CTA once the CTA has made its last claim on the work cursor `counter`:
// the CTA that arrives last puts the cursor and the arrival count back to zero, so every call
// starts from zero without a separate reset.
__device__ __forceinline__ void release_work_cursor(int32_t* counter, int32_t* exits) {
  __threadfence();
  if (atomicAdd(exits, 1) == static_cast<int>(gridDim.x) - 1) {
    atomicExch(counter, 0);
    atomicExch(exits, 0);
  }
}

// ---- named barriers (a subset of the CTA's warps) -----------------------------------------------

__device__ __forceinline__ void named_bar_sync(uint32_t id, uint32_t nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// Barrier over `nthreads` threads that also returns the OR of `pred` across them.
__device__ __forceinline__ bool named_bar_or(uint32_t id, uint32_t nthreads, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, %2, %3, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(pred ? 1u : 0u), "r"(id), "r"(nthreads)
      : "memory");
  return r != 0;
}

// ---- bulk and tensor copies (TMA) ---------------------------------------------------------------

// Contiguous global -> shared copy completing on `bar` (addresses 16 B aligned, size % 16 == 0).
// 4-byte asynchronous copy global -> shared (no register dependency on the loaded value).
__device__ __forceinline__ void cp_async_4(void* dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_u32(dst)), "l"(src)
               : "memory");
}
// Arrive on `bar` once every cp.async this thread issued so far has completed (the arrival is
// the barrier's expected one: .noinc).
__device__ __forceinline__ void cp_async_mbar_arrive(uint64_t* bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes,
                                          uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
          "r"(smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, uint64_t* bar,
                                            int32_t c0, int32_t c1, int32_t c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(smem_u32(dst)),
      "l"(map), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}

__device__ __forceinline__ void tma_load_4d(void* dst, const CUtensorMap* map, uint64_t* bar,
                                            int32_t c0, int32_t c1, int32_t c2, int32_t c3) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5, %6}], [%2];" ::"r"(smem_u32(dst)),
      "l"(map), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
      : "memory");
}

// L2 policy for data read exactly once (the K/V stream): evict it first, so that it does not
// push out the partial results and query rows that are read again soon.
__device__ __forceinline__ uint64_t l2_evict_first_policy() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}

__device__ __forceinline__ void bulk_load_stream(void* dst, const void* src, uint32_t bytes,
                                                 uint64_t* bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1], %2, [%3], %4;" ::"r"(smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}

__device__ __forceinline__ void tma_load_4d_stream(void* dst, const CUtensorMap* map,
                                                   uint64_t* bar, int32_t c0, int32_t c1,
                                                   int32_t c2, int32_t c3, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      ".L2::cache_hint [%0], [%1, {%3, %4, %5, %6}], [%2], %7;" ::"r"(smem_u32(dst)),
      "l"(map), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "l"(policy)
      : "memory");
}

__device__ __forceinline__ void prefetch_tensor_map(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(map) : "memory");
}

// Make this thread's generic-proxy shared-memory writes visible to the async proxy (tensor
// cores, TMA) before signalling the consumer.
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ---- tcgen05: tensor memory and UMMA --------------------------------------------------------------

__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// D(tmem) (+)= A(smem desc) · B(smem desc), kind::f16 (bf16 inputs, fp32 accumulator).
__device__ __forceinline__ void umma_bf16_ss(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                             uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// D(tmem) (+)= A(smem desc) · B(smem desc), kind::f8f6f4 (8-bit A/B, fp32 accumulator).
__device__ __forceinline__ void umma_f8_ss(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                           uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// D(tmem) (+)= A(tmem) · B(smem desc), kind::f16.
__device__ __forceinline__ void umma_bf16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc,
                                             uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrive on `bar` once every tcgen05 operation issued so far by this thread has completed.
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_u32(bar))
      : "memory");
}

// 32 lanes x 32 bit, 16 consecutive columns: thread t of the warp gets lane (32*(warp%4) + t).
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}

__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t (&r)[8]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
      : "memory");
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15])
      : "memory");
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]),
      "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]),
      "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}

__device__ __forceinline__ void tmem_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_wait_st() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// Shared-memory matrix descriptor (tcgen05 format): start, leading / stride byte offsets,
// version 1, layout (0 = no swizzle, 2 = 128-byte swizzle).
constexpr uint32_t kLayoutNone = 0;
constexpr uint32_t kLayoutSW128 = 2;

__device__ __forceinline__ uint64_t smem_desc(uint32_t saddr, uint32_t lbo_bytes,
                                              uint32_t sbo_bytes, uint32_t layout) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>((lbo_bytes >> 4) & 0x3FFFu) << 16;
  d |= static_cast<uint64_t>((sbo_bytes >> 4) & 0x3FFFu) << 32;
  d |= static_cast<uint64_t>(1) << 46;
  d |= static_cast<uint64_t>(layout & 7u) << 61;
  return d;
}

// Instruction descriptor for kind::f16 with bf16 A/B and fp32 D; a_mn / b_mn select MN-major.
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int M, int N, bool a_mn, bool b_mn) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((a_mn ? 1u : 0u) << 15) |
         ((b_mn ? 1u : 0u) << 16) | (static_cast<uint32_t>(N >> 3) << 17) |
         (static_cast<uint32_t>(M >> 4) << 24);
}

// The same with f16 A/B (format fields 0).
__host__ __device__ constexpr uint32_t idesc_f16_f32(int M, int N, bool a_mn, bool b_mn) {
  return (1u << 4) | ((a_mn ? 1u : 0u) << 15) | ((b_mn ? 1u : 0u) << 16) |
         (static_cast<uint32_t>(N >> 3) << 17) | (static_cast<uint32_t>(M >> 4) << 24);
}

// Instruction descriptor for kind::f8f6f4 with E4M3 A and B (format code 0), fp32 D, K-major.
__host__ __device__ constexpr uint32_t idesc_e4m3_f32(int M, int N) {
  return (1u << 4) | (0u << 7) | (0u << 10) | (static_cast<uint32_t>(N >> 3) << 17) |
         (static_cast<uint32_t>(M >> 4) << 24);
}

// ---- programmatic dependent launch ---------------------------------------------------------------

// Let the next kernel of the stream (launched with programmatic stream serialization) start.
__device__ __forceinline__ void pdl_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
// Wait until the previous kernel of the stream has completed and its writes are visible.
__device__ __forceinline__ void pdl_wait_prerequisites() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}

// ---- numerics -------------------------------------------------------------------------------

// 2^x with the hardware approximation (relative error ~2^-22); ex2(-inf) = 0.
__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ float warp_max_f32(float v) {
  float r;
  asm volatile("redux.sync.max.f32 %0, %1, 0xffffffff;" : "=f"(r) : "f"(v));
  return r;
}

__device__ __forceinline__ float warp_sum_f32(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

template <typename T>
__device__ __forceinline__ float to_f32(T x);
template <>
__device__ __forceinline__ float to_f32<float>(float x) {
  return x;
}
template <>
__device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 x) {
  return __bfloat162float(x);
}

template <typename T>
__device__ __forceinline__ T from_f32(float x);
template <>
__device__ __forceinline__ float from_f32<float>(float x) {
  return x;
}
template <>
__device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

// ---- in-kernel LSE merge of the splits of one (row, KV head) group ------------------------------

// Where split partials live and where merged results go.
struct MergeTarget {
  const float* part_o;   // [slots][G][D] fp32, the slots of one group consecutive
  const float* part_lse; // [slots][G] base-2 log-sum-exp
  int32_t* arrivals;     // [rows][Hkv] splits completed so far in this call
  void* out;             // [rows][Hq][D]
  int64_t o_sr, o_sh;
  float* lse;            // [rows][Hq] natural log
  int32_t hq, hkv, g, d;
};

constexpr int kMergeThreads = 128;  // the role group that writes partials and merges
constexpr int kMergeLseCap = 512;   // floats of shared memory holding one chunk of split LSEs

// Called by the kMergeThreads threads of named barrier `bar` right after they stored this CTA's
// partial (O_s, LSE_s) of one split of group (row, h). The split is counted on a device-scope
// arrival counter; the CTA that completes the group's last split merges all of its partials,
//   M = max_s LSE_s;  w_s = 2^(LSE_s - M);  O = sum_s w_s O_s / sum_s w_s;  LSE = M + log2 sum_s w_s
// (the merge of "大模型推理加速FlashDecoding算法原理与多GPU并行解码实战",
// "多GPU张量并行扩展下的FlashDecoding实现", with the per-split sums folded into w_s), in a fixed
// split order, while the partials are still in L2. Splits whose LSE is -inf weigh nothing; a group
// with no visible key gets O = 0 and LSE = -inf. EPT = elements of the G x D output per thread.
template <typename T, int EPT>
__device__ __forceinline__ void finish_split_and_merge(const MergeTarget& t, int row, int h,
                                                       int nsplit, int64_t slot0, int tid,
                                                       int bar, volatile int* s_flag,
                                                       float* s_lse) {
  __threadfence();  // this thread's partial stores, visible device-wide before the count
  named_bar_sync(bar, kMergeThreads);
  if (tid == 0) *s_flag = atomicAdd(&t.arrivals[row * t.hkv + h], 1);
  named_bar_sync(bar, kMergeThreads);
  if (*s_flag != nsplit - 1) return;  // the same value for every thread of the group
  __threadfence();
  const int G = t.g, D = t.d, GD = G * D;
  float acc[EPT], wsum[EPT], mx[EPT];
#pragma unroll
  for (int k = 0; k < EPT; ++k) { acc[k] = 0.f; wsum[k] = 0.f; mx[k] = -INFINITY; }
  const int chunk = kMergeLseCap / G;  // splits whose LSEs fit the shared buffer
  for (int c0 = 0; c0 < nsplit; c0 += chunk) {
    const int cn = min(chunk, nsplit - c0);
    const float* lsrc = t.part_lse + (slot0 + c0) * G;
    for (int i = tid; i < cn * G; i += kMergeThreads) s_lse[i] = __ldcg(lsrc + i);
    named_bar_sync(bar, kMergeThreads);
    // running maximum per element's head, rescaling what was accumulated so far
#pragma unroll
    for (int k = 0; k < EPT; ++k) {
      const int e = tid + k * kMergeThreads;
      if (e < GD) {
        const int g = e / D;
        float cm = -INFINITY;
        for (int s = 0; s < cn; ++s) cm = fmaxf(cm, s_lse[s * G + g]);
        const float nm = fmaxf(mx[k], cm);
        const float sc = (nm == -INFINITY) ? 1.f : fast_exp2(mx[k] - nm);
        acc[k] *= sc;
        wsum[k] *= sc;
        mx[k] = nm;
      }
    }
    // weighted sum, kB splits per round with all their loads (kB x EPT <= 32) in flight
    constexpr int kB = EPT >= 32 ? 1 : 32 / EPT;
    const float* osrc = t.part_o + (slot0 + c0) * static_cast<int64_t>(GD);
    for (int s0 = 0; s0 < cn; s0 += kB) {
      float x[kB][EPT];
#pragma unroll
      for (int j = 0; j < kB; ++j)
#pragma unroll
        for (int k = 0; k < EPT; ++k) {
          const int e = tid + k * kMergeThreads;
          x[j][k] = (s0 + j < cn && e < GD) ? __ldcg(osrc + static_cast<int64_t>(s0 + j) * GD + e) : 0.f;
        }
#pragma unroll
      for (int j = 0; j < kB; ++j)
#pragma unroll
        for (int k = 0; k < EPT; ++k) {
          const int e = tid + k * kMergeThreads;
          if (s0 + j < cn && e < GD && mx[k] != -INFINITY) {
            const float w = fast_exp2(s_lse[(s0 + j) * G + e / D] - mx[k]);
            acc[k] = fmaf(w, x[j][k], acc[k]);
            wsum[k] += w;
          }
        }
    }
    named_bar_sync(bar, kMergeThreads);  // s_lse is reused by the next chunk
  }
#pragma unroll
  for (int k = 0; k < EPT; ++k) {
    const int e = tid + k * kMergeThreads;
    if (e < GD) {
      const int g = e / D, d = e - g * D;
      const int hq = h * G + g;
      T* o = static_cast<T*>(t.out) + static_cast<int64_t>(row) * t.o_sr + static_cast<int64_t>(hq) * t.o_sh;
      o[d] = from_f32<T>(wsum[k] > 0.f ? acc[k] / wsum[k] : 0.f);
      if (d == 0)
        t.lse[static_cast<int64_t>(row) * t.hq + hq] =
            wsum[k] > 0.f ? (mx[k] + log2f(wsum[k])) * kLn2 : -INFINITY;
    }
  }
  if (tid == 0) t.arrivals[row * t.hkv + h] = 0;  // ready for the next call on this workspace
}

}  // namespace fd
