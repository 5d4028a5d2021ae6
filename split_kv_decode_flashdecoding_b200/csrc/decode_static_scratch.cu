// fd_decode_attention_static: the decode attention call for callers that cannot allocate device
// memory. It runs the same planner, split and combine kernels as fd_decode_attention, but its
// scratch (the split plan, the work items and the per-split partial results) lives in one
// file-scope device array of FD_STATIC_SCRATCH_BYTES instead of the library's per-stream
// workspace, so the call itself never allocates.
//
// Who needs this: serving engines that hand nearly all of a GPU's memory to their own KV-cache
// pool (a late cudaMalloc would fail or fragment that pool), plugin hosts that only let a plugin
// use buffers the host has already allocated, and latency-critical loops where the implicit
// device synchronisation of cudaMalloc / cudaFree is not acceptable.
//
// Rules for callers (also stated in include/fd.h):
//  - Every GPU that loads this library holds the array until the process exits.
//  - The first call on a device looks up the array's device address with cudaGetSymbolAddress,
//    with that device current; make that first call before any stream capture begins.
//  - All calls share the one array, which keeps the previous call's contents: calls that overlap
//    on the GPU (other streams, or other host threads without ordering between them) race on it.
//    Each call clears the header it needs zeroed (status word and work cursor) on its stream.
//  - A shape whose worst-case scratch exceeds FD_STATIC_SCRATCH_BYTES is rejected on the host with
//    FD_ERR_UNSUPPORTED before anything is enqueued.
//  - Device status flags raised by these kernels land in the array's header, which the next call
//    clears; fd_poll_status does not report them.
#include <cmath>
#include <map>
#include <mutex>

#include "abi_internal.h"
#include "common.cuh"
#include "internal.h"

using namespace fd;
using namespace fd_abi;

namespace {

// The scratch itself. In host code this name is only a stand-in for the symbol: its device
// address comes from cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_fd_static_scratch[FD_STATIC_SCRATCH_BYTES];

std::mutex g_static_mu;
std::map<int, void*> g_static_addr;  // device ordinal -> device address of g_fd_static_scratch

// Device address of the scratch on device `dev` (the current device), looked up once.
fd_status static_scratch_address(int dev, void** out) {
  std::lock_guard<std::mutex> lock(g_static_mu);
  auto it = g_static_addr.find(dev);
  if (it != g_static_addr.end()) {
    *out = it->second;
    return FD_OK;
  }
  void* ptr = nullptr;
  cudaError_t e = cudaGetSymbolAddress(&ptr, g_fd_static_scratch);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(static scratch)");
  if (!ptr) return fail(FD_ERR_CUDA, "cudaGetSymbolAddress returned a null static scratch address");
  g_static_addr[dev] = ptr;
  *out = ptr;
  return FD_OK;
}

}  // namespace

extern "C" fd_status fd_decode_attention_static(const fd_tensor* q, const fd_tensor* k_cache,
                                                const fd_tensor* v_cache,
                                                const int32_t* cache_lens, int32_t num_splits,
                                                fd_tensor* out, float* lse, void* stream_) {
  cudaStream_t stream = static_cast<cudaStream_t>(stream_);
  DecodeShape sh{};
  fd_status s = resolve_decode(q, k_cache, v_cache, out, &sh);
  if (s != FD_OK) return s;
  if (num_splits < 0) return fail(FD_ERR_INVALID_ARGUMENT, "num_splits must be >= 0");
  if (num_splits > 65536) return fail(FD_ERR_UNSUPPORTED, "num_splits above 65536");
  if (sh.B == 0) return FD_OK;
  if (!cache_lens) return fail(FD_ERR_INVALID_ARGUMENT, "cache_lens is NULL");
  if (!lse) return fail(FD_ERR_INVALID_ARGUMENT, "lse is NULL");
  int dev = 0;
  cudaError_t ce = cudaGetDevice(&dev);
  if (ce != cudaSuccess) return cuda_fail(ce, "cudaGetDevice");
  const int nctas = decode_ctas(dev, sh.use_tc);
  if (nctas < 1) return fail(FD_ERR_CUDA, "no multiprocessors reported for device %d", dev);

  const int64_t max_items = decode_max_items(sh.B, sh.hkv, sh.cap, num_splits, nctas);
  const int64_t max_slots = max_items;  // one partial slot (G heads) per split item
  const WsLayout L = ws_layout(max_items, 0, sh.B, max_slots, sh.hq, sh.d, sh.hkv);
  if (L.total > static_cast<size_t>(FD_STATIC_SCRATCH_BYTES))
    return fail(FD_ERR_UNSUPPORTED,
                "this decode shape needs up to %zu bytes of scratch, more than the %zu-byte static "
                "scratch of fd_decode_attention_static; use fd_decode_attention",
                L.total, static_cast<size_t>(FD_STATIC_SCRATCH_BYTES));

  void* ws = nullptr;
  if ((s = static_scratch_address(dev, &ws)) != FD_OK) return s;
  char* base = static_cast<char*>(ws);
  WsHeader* hdr = reinterpret_cast<WsHeader*>(base);
  DecodeItem* items = reinterpret_cast<DecodeItem*>(base + L.dec_items);
  int32_t* row_nsplit = reinterpret_cast<int32_t*>(base + L.row_nsplit);
  int32_t* row_base = reinterpret_cast<int32_t*>(base + L.row_base);
  float* part_o = reinterpret_cast<float*>(base + L.part_o);
  float* part_lse = reinterpret_cast<float*>(base + L.part_lse);
  int32_t* arrivals = reinterpret_cast<int32_t*>(base + L.arrivals);

  DecodeParams dp{};
  dp.q = q->data;
  dp.q_sr = q->stride[0];
  dp.q_sh = q->stride[1];
  dp.k = k_cache->data;
  dp.v = v_cache->data;
  dp.kv_sb = k_cache->stride[0];
  dp.kv_sh = k_cache->stride[1];
  dp.out = out->data;
  dp.o_sr = out->stride[0];
  dp.o_sh = out->stride[1];
  dp.lse = lse;
  dp.hq = sh.hq;
  dp.hkv = sh.hkv;
  dp.g = sh.g;
  dp.d = sh.d;
  dp.cap = sh.cap;
  dp.q_box_rows = sh.hq < 16 ? sh.hq : 16;
  dp.kv_box_rows = sh.cap < 128 ? sh.cap : 128;
  dp.scale_log2 = static_cast<float>(1.0 / std::sqrt(static_cast<double>(sh.d)) * 1.4426950408889634);
  dp.hdr = hdr;
  dp.items = items;
  dp.row_base = row_base;
  dp.part_o = part_o;
  dp.part_lse = part_lse;
  dp.arrivals = arrivals;

  CUtensorMap tq, tk, tv;
  if (sh.use_tc) {
    const uint64_t qd[3] = {static_cast<uint64_t>(sh.d), static_cast<uint64_t>(sh.hq), static_cast<uint64_t>(sh.B)};
    const uint64_t qs[2] = {static_cast<uint64_t>(q->stride[1]) * 2, static_cast<uint64_t>(q->stride[0]) * 2};
    const uint32_t qb[3] = {64, static_cast<uint32_t>(dp.q_box_rows), 1};
    if ((s = make_tmap(&tq, q->data, 3, qd, qs, qb, "q")) != FD_OK) return s;
    const uint64_t kd[4] = {static_cast<uint64_t>(sh.d), static_cast<uint64_t>(sh.cap),
                            static_cast<uint64_t>(sh.hkv), static_cast<uint64_t>(sh.B)};
    const uint64_t ks[3] = {static_cast<uint64_t>(k_cache->stride[2]) * 2,
                            static_cast<uint64_t>(k_cache->stride[1]) * 2,
                            static_cast<uint64_t>(k_cache->stride[0]) * 2};
    const uint32_t kb[4] = {64, static_cast<uint32_t>(dp.kv_box_rows), 1, 1};
    if ((s = make_tmap(&tk, k_cache->data, 4, kd, ks, kb, "k_cache")) != FD_OK) return s;
    if ((s = make_tmap(&tv, v_cache->data, 4, kd, ks, kb, "v_cache")) != FD_OK) return s;
  }

  PlanParams pp{};
  pp.lens = cache_lens;
  pp.B = sh.B;
  pp.hkv = sh.hkv;
  pp.hq = sh.hq;
  pp.cap = sh.cap;
  pp.fixed = num_splits;
  pp.nctas = nctas;
  pp.max_dec_items = max_items;
  pp.hdr = hdr;
  pp.items = items;
  pp.row_nsplit = row_nsplit;
  pp.row_base = row_base;
  pp.arrivals = arrivals;

  CombineParams cp{};
  cp.row_nsplit = row_nsplit;
  cp.row_base = row_base;
  cp.part_o = part_o;
  cp.part_lse = part_lse;
  cp.out = out->data;
  cp.o_sr = out->stride[0];
  cp.o_sh = out->stride[1];
  cp.lse = lse;
  cp.rows = sh.B;
  cp.hq = sh.hq;
  cp.hkv = sh.hkv;
  cp.g = sh.g;
  cp.d = sh.d;
  cp.dtype = sh.dtype;

  // the status word and the work cursor must start at zero; the previous call left its own
  ce = cudaMemsetAsync(hdr, 0, sizeof(WsHeader), stream);
  if (ce != cudaSuccess) return cuda_fail(ce, "clear static scratch header");
  ce = launch_plan_decode(pp, stream);
  if (ce != cudaSuccess) return cuda_fail(ce, "plan kernel launch");
  ce = sh.use_tc ? launch_decode_tc(dp, tq, tk, tv, nctas, stream)
                 : launch_decode_simt(dp, sh.dtype, nctas, stream);
  if (ce != cudaSuccess) return cuda_fail(ce, "split kernel launch");
  if (sh.use_tc) {
    ce = launch_combine(cp, stream);
    if (ce != cudaSuccess) return cuda_fail(ce, "combine kernel launch");
  }
  return FD_OK;
}
