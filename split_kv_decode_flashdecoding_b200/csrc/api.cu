// C ABI of the library (include/fd.h): argument validation, the per-(device, stream) workspace,
// tensor-map construction, kernel dispatch and optional per-launch timing.
#include <algorithm>
#include <cfloat>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstddef>
#include <cstring>
#include <map>
#include <mutex>
#include <string>
#include <utility>
#include <vector>

#include "abi_internal.h"
#include "common.cuh"
#include "internal.h"

using namespace fd;

// Helpers shared with the other C-ABI source files of the library (abi_internal.h).
namespace fd_abi {

// ---------------------------------------------------------------------------- errors ---------
thread_local std::string g_last_error;

fd_status fail(fd_status s, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return s;
}

fd_status cuda_fail(cudaError_t e, const char* what) {
  return fail(FD_ERR_CUDA, "%s: %s (%s)", what, cudaGetErrorName(e), cudaGetErrorString(e));
}

#define FD_CUDA(call, what)                       \
  do {                                            \
    cudaError_t e_ = (call);                      \
    if (e_ != cudaSuccess) return cuda_fail(e_, what); \
  } while (0)

// ---------------------------------------------------------------------------- workspace ------
// Per (device, stream): the grow-only device buffer, plus the side stream and the two events a
// chunked-prefill call forks its decode rows onto and joins back with. They are created with the
// first buffer, so a call under graph capture (which must find the buffer reserved) never
// creates them.
struct Workspace {
  void* ptr = nullptr;
  size_t bytes = 0;
  cudaStream_t side = nullptr;
  cudaEvent_t fork = nullptr, join = nullptr;
};
std::mutex g_mu;
std::map<std::pair<int, uintptr_t>, Workspace> g_ws;

fd_status get_workspace(cudaStream_t stream, size_t need, void** out, Workspace* view = nullptr) {
  int dev = 0;
  FD_CUDA(cudaGetDevice(&dev), "cudaGetDevice");
  std::lock_guard<std::mutex> lock(g_mu);
  Workspace& w = g_ws[{dev, reinterpret_cast<uintptr_t>(stream)}];
  if (w.ptr && w.bytes >= need) {
    *out = w.ptr;
    if (view) *view = w;
    return FD_OK;
  }
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  FD_CUDA(cudaStreamIsCapturing(stream, &cs), "cudaStreamIsCapturing");
  if (cs != cudaStreamCaptureStatusNone)
    return fail(FD_ERR_WORKSPACE,
                "workspace of this stream holds %zu bytes but the call needs %zu; reserve it with "
                "fd_reserve_workspace before capturing",
                w.bytes, need);
  uint32_t old_status = 0;
  if (w.ptr) {
    FD_CUDA(cudaStreamSynchronize(stream), "cudaStreamSynchronize");
    FD_CUDA(cudaMemcpy(&old_status, w.ptr, sizeof(uint32_t), cudaMemcpyDeviceToHost), "read status");
    FD_CUDA(cudaFree(w.ptr), "cudaFree(workspace)");
    w.ptr = nullptr;
    w.bytes = 0;
  }
  size_t nb = std::max(need, static_cast<size_t>(1) << 20);
  nb = (nb + (2u << 20) - 1) / (2u << 20) * (2u << 20);
  void* p = nullptr;
  cudaError_t e = cudaMalloc(&p, nb);
  if (e != cudaSuccess) {
    (void)cudaGetLastError();
    return fail(FD_ERR_WORKSPACE, "cudaMalloc of %zu workspace bytes failed: %s", nb,
                cudaGetErrorString(e));
  }
  WsHeader h;
  std::memset(&h, 0, sizeof(h));
  h.status = old_status;
  FD_CUDA(cudaMemcpyAsync(p, &h, sizeof(h), cudaMemcpyHostToDevice, stream), "init workspace");
  FD_CUDA(cudaStreamSynchronize(stream), "cudaStreamSynchronize");
  w.ptr = p;
  w.bytes = nb;
  if (!w.side) {
    int prio_lo = 0, prio_hi = 0;
    FD_CUDA(cudaDeviceGetStreamPriorityRange(&prio_lo, &prio_hi), "cudaDeviceGetStreamPriorityRange");
    FD_CUDA(cudaStreamCreateWithPriority(&w.side, cudaStreamNonBlocking, prio_lo), "create side stream");
    FD_CUDA(cudaEventCreateWithFlags(&w.fork, cudaEventDisableTiming), "create fork event");
    FD_CUDA(cudaEventCreateWithFlags(&w.join, cudaEventDisableTiming), "create join event");
  }
  *out = p;
  if (view) *view = w;
  return FD_OK;
}

// ---------------------------------------------------------------------------- devices --------
int sm_count(int dev) {
  static std::mutex mu;
  static std::map<int, int> cache;
  std::lock_guard<std::mutex> lock(mu);
  auto it = cache.find(dev);
  if (it != cache.end()) return it->second;
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) n = 0;
  cache[dev] = n;
  return n;
}

// ---------------------------------------------------------------------------- tensor maps ----
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static std::once_flag once;
  static EncodeTiledFn fn = nullptr;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &f, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(f);
  });
  return fn;
}

// Tensor map with 128-byte swizzle (rank <= 5); dims/strides innermost first. Returns the
// driver's result (CUDA_ERROR_NOT_SUPPORTED when the encoder is missing).
CUresult encode_tmap(CUtensorMap* map, const void* base, int rank, const uint64_t* dims,
                     const uint64_t* strides_bytes, const uint32_t* box, CUtensorMapDataType dtype) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return CUDA_ERROR_NOT_SUPPORTED;
  cuuint64_t d[5], s[4];
  cuuint32_t b[5], es[5];
  for (int i = 0; i < rank; ++i) {
    d[i] = dims[i];
    b[i] = box[i];
    es[i] = 1;
    if (i > 0) s[i - 1] = strides_bytes[i - 1];
  }
  return fn(map, dtype, rank, const_cast<void*>(base), d, s, b,
            es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
}

// The same, failing the call with a message.
fd_status make_tmap(CUtensorMap* map, const void* base, int rank, const uint64_t* dims,
                    const uint64_t* strides_bytes, const uint32_t* box, const char* what,
                    CUtensorMapDataType dtype) {
  if (!encode_fn()) return fail(FD_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  const CUresult r = encode_tmap(map, base, rank, dims, strides_bytes, box, dtype);
  if (r != CUDA_SUCCESS) return fail(FD_ERR_CUDA, "cuTensorMapEncodeTiled(%s) failed: %d", what, (int)r);
  return FD_OK;
}

// ---------------------------------------------------------------------------- profiling ------
// Per profiled call: a start and an end event around each of the planner, the decode split
// kernel, the chunk tile kernel and the combine kernel (both at the same point for a launch the
// call does not make). A chunked-prefill call records its split kernel's pair on its side stream.
constexpr int kProfSegments = 4;
constexpr int kProfEvents = 2 * kProfSegments;
enum ProfSeg { kSegPlan = 0, kSegSplit = 1, kSegTiles = 2, kSegCombine = 3 };
struct Profiler {
  std::mutex mu;
  std::vector<cudaEvent_t> ev;  // kProfEvents per call
  int max_calls = 0;
  int calls = 0;
  bool active = false;
} g_prof;

// Returns the events of the next profiled call, or nullptr.
cudaEvent_t* prof_next() {
  std::lock_guard<std::mutex> lock(g_prof.mu);
  if (!g_prof.active || g_prof.calls >= g_prof.max_calls) return nullptr;
  return &g_prof.ev[kProfEvents * static_cast<size_t>(g_prof.calls++)];
}

// ---------------------------------------------------------------------------- validation -----
size_t elem_size(int dtype) { return dtype == FD_F32 ? 4 : (dtype == FD_E4M3 ? 1 : 2); }

fd_status check_tensor(const fd_tensor* t, const char* name, int ndim) {
  if (!t) return fail(FD_ERR_INVALID_ARGUMENT, "%s is NULL", name);
  if (t->ndim != ndim) return fail(FD_ERR_INVALID_ARGUMENT, "%s must have %d dimensions, got %d", name, ndim, t->ndim);
  if (t->dtype != FD_F32 && t->dtype != FD_BF16 && t->dtype != FD_E4M3)
    return fail(FD_ERR_UNSUPPORTED, "%s: dtype %d is not FD_F32, FD_BF16 or FD_E4M3", name, t->dtype);
  for (int i = 0; i < ndim; ++i) {
    if (t->shape[i] < 0) return fail(FD_ERR_INVALID_ARGUMENT, "%s: negative shape[%d]", name, i);
    if (t->shape[i] > INT32_MAX) return fail(FD_ERR_UNSUPPORTED, "%s: shape[%d] exceeds int32", name, i);
    if (t->stride[i] < 0) return fail(FD_ERR_UNSUPPORTED, "%s: negative stride[%d]", name, i);
  }
  if (t->stride[ndim - 1] != 1)
    return fail(FD_ERR_UNSUPPORTED, "%s: the last dimension must be contiguous (stride 1)", name);
  return FD_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool stride16(int64_t stride_elems, int dtype) { return (stride_elems * static_cast<int64_t>(elem_size(dtype))) % 16 == 0; }

fd_status check_kv(const fd_tensor* k, const fd_tensor* v, int dtype, int B, int d) {
  fd_status s;
  if ((s = check_tensor(k, "k_cache", 4)) != FD_OK) return s;
  if ((s = check_tensor(v, "v_cache", 4)) != FD_OK) return s;
  if (k->dtype != dtype || v->dtype != dtype)
    return fail(FD_ERR_INVALID_ARGUMENT, dtype == FD_E4M3 ? "k_cache / v_cache must be FD_E4M3"
                                                           : "k_cache / v_cache dtype differs from q");
  for (int i = 0; i < 4; ++i) {
    if (k->shape[i] != v->shape[i]) return fail(FD_ERR_INVALID_ARGUMENT, "k_cache and v_cache shapes differ");
    if (k->stride[i] != v->stride[i]) return fail(FD_ERR_UNSUPPORTED, "k_cache and v_cache must share strides");
  }
  if (k->shape[0] != B) return fail(FD_ERR_INVALID_ARGUMENT, "k_cache batch %lld != %d", (long long)k->shape[0], B);
  if (k->shape[3] != d) return fail(FD_ERR_INVALID_ARGUMENT, "k_cache head_dim %lld != q head_dim %d", (long long)k->shape[3], d);
  if (k->shape[1] < 1) return fail(FD_ERR_INVALID_ARGUMENT, "k_cache needs at least one KV head");
  if (k->shape[2] < 1) return fail(FD_ERR_INVALID_ARGUMENT, "k_cache capacity (dim 2) must be >= 1");
  if (k->stride[2] != d) return fail(FD_ERR_UNSUPPORTED, "token rows of the cache must be contiguous (stride[2] == head_dim)");
  if (B > 0 && (!k->data || !v->data)) return fail(FD_ERR_INVALID_ARGUMENT, "k_cache / v_cache data is NULL");
  if (!aligned16(k->data) || !aligned16(v->data) || !stride16(k->stride[0], dtype) || !stride16(k->stride[1], dtype))
    return fail(FD_ERR_UNSUPPORTED, "cache data and strides must be 16-byte aligned");
  return FD_OK;
}

fd_status check_q_out(const fd_tensor* q, const fd_tensor* out, const char* qn) {
  fd_status s;
  if ((s = check_tensor(q, qn, 3)) != FD_OK) return s;
  if ((s = check_tensor(out, "out", 3)) != FD_OK) return s;
  if (q->dtype == FD_E4M3) return fail(FD_ERR_UNSUPPORTED, "%s: FD_E4M3 is a cache dtype only", qn);
  if (out->dtype != q->dtype) return fail(FD_ERR_INVALID_ARGUMENT, "out dtype differs from %s", qn);
  for (int i = 0; i < 3; ++i)
    if (out->shape[i] != q->shape[i]) return fail(FD_ERR_INVALID_ARGUMENT, "out shape differs from %s", qn);
  if (q->shape[0] > 0 && (!q->data || !out->data)) return fail(FD_ERR_INVALID_ARGUMENT, "%s / out data is NULL", qn);
  if (!aligned16(q->data) || !stride16(q->stride[0], q->dtype) || !stride16(q->stride[1], q->dtype))
    return fail(FD_ERR_UNSUPPORTED, "%s data and strides must be 16-byte aligned", qn);
  return FD_OK;
}

// The split kernel of a call: tensor cores for bf16 groups of 2..16 with D 128 (and for every
// group of <= 8 heads over an E4M3 cache), CUDA cores otherwise.
fd_status choose_kernel(DecodeShape* sh) {
  if (sh->kv_fp8) {
    sh->use_tc = sh->d == 128 && sh->g <= 8;
    if (!sh->use_tc)
      return fail(FD_ERR_UNSUPPORTED, "an FP8 cache needs head_dim 128 and group size <= 8 (got %d, %d)",
                  sh->d, sh->g);
    return FD_OK;
  }
  sh->use_tc = sh->dtype == FD_BF16 && sh->d == 128 && sh->g >= 2 && sh->g <= 16;
  if (!sh->use_tc && sh->g > 8)
    return fail(FD_ERR_UNSUPPORTED, "group size %d needs bf16 with head_dim 128 (tensor-core kernel)", sh->g);
  return FD_OK;
}

fd_status check_quant(const fd_tensor* q, const KvQuant* quant) {
  if (!quant) return FD_OK;
  if (q->dtype != FD_BF16) return fail(FD_ERR_UNSUPPORTED, "an FP8 cache needs bf16 q and out");
  const float ks = quant->k_scale, vs = quant->v_scale;
  if (!(ks > 0.f && ks <= FLT_MAX) || !(vs > 0.f && vs <= FLT_MAX))
    return fail(FD_ERR_INVALID_ARGUMENT, "k_scale and v_scale must be finite and > 0");
  return FD_OK;
}

fd_status resolve_decode(const fd_tensor* q, const fd_tensor* k, const fd_tensor* v,
                         const fd_tensor* out, DecodeShape* sh, const KvQuant* quant) {
  fd_status s;
  if ((s = check_q_out(q, out, "q")) != FD_OK) return s;
  if ((s = check_quant(q, quant)) != FD_OK) return s;
  sh->B = static_cast<int>(q->shape[0]);
  sh->hq = static_cast<int>(q->shape[1]);
  sh->d = static_cast<int>(q->shape[2]);
  sh->dtype = q->dtype;
  sh->kv_fp8 = quant != nullptr;
  if (sh->d != 64 && sh->d != 128) return fail(FD_ERR_UNSUPPORTED, "head_dim %d: only 64 and 128 are supported", sh->d);
  if ((s = check_kv(k, v, sh->kv_fp8 ? FD_E4M3 : sh->dtype, sh->B, sh->d)) != FD_OK) return s;
  sh->hkv = static_cast<int>(k->shape[1]);
  sh->cap = static_cast<int>(k->shape[2]);
  if (sh->hq < 1 || sh->hq % sh->hkv != 0)
    return fail(FD_ERR_INVALID_ARGUMENT, "q heads (%d) must be a positive multiple of KV heads (%d)", sh->hq, sh->hkv);
  sh->g = sh->hq / sh->hkv;
  if (sh->B > kMaxPlanBatch) return fail(FD_ERR_UNSUPPORTED, "batch %d exceeds %d", sh->B, kMaxPlanBatch);
  return choose_kernel(sh);
}

fd_status resolve_paged(const fd_tensor* q, const fd_tensor* k, const fd_tensor* v,
                        PagedCache& pg, const fd_tensor* out, DecodeShape* sh,
                        const KvQuant* quant) {
  fd_status s;
  if ((s = check_q_out(q, out, "q")) != FD_OK) return s;
  if ((s = check_quant(q, quant)) != FD_OK) return s;
  sh->B = static_cast<int>(q->shape[0]);
  sh->hq = static_cast<int>(q->shape[1]);
  sh->d = static_cast<int>(q->shape[2]);
  sh->dtype = q->dtype;
  sh->kv_fp8 = quant != nullptr;
  const int kvt = sh->kv_fp8 ? FD_E4M3 : sh->dtype;
  if (sh->d != 64 && sh->d != 128) return fail(FD_ERR_UNSUPPORTED, "head_dim %d: only 64 and 128 are supported", sh->d);
  if ((s = check_tensor(k, "k_pages", 4)) != FD_OK) return s;
  if ((s = check_tensor(v, "v_pages", 4)) != FD_OK) return s;
  if (k->dtype != kvt || v->dtype != kvt)
    return fail(FD_ERR_INVALID_ARGUMENT, sh->kv_fp8 ? "k_pages / v_pages must be FD_E4M3"
                                                    : "k_pages / v_pages dtype differs from q");
  for (int i = 0; i < 4; ++i) {
    if (k->shape[i] != v->shape[i]) return fail(FD_ERR_INVALID_ARGUMENT, "k_pages and v_pages shapes differ");
    if (k->stride[i] != v->stride[i]) return fail(FD_ERR_UNSUPPORTED, "k_pages and v_pages must share strides");
  }
  if (k->shape[0] < 1) return fail(FD_ERR_INVALID_ARGUMENT, "the page pool needs at least one page");
  if (k->shape[1] < 1) return fail(FD_ERR_INVALID_ARGUMENT, "k_pages needs at least one KV head");
  if (k->shape[3] != sh->d) return fail(FD_ERR_INVALID_ARGUMENT, "k_pages head_dim %lld != q head_dim %d", (long long)k->shape[3], sh->d);
  const int64_t psz = k->shape[2];
  if (!(psz == 8 || psz == 16 || psz == 32 || psz == 64 || (psz >= 128 && psz % 128 == 0)))
    return fail(FD_ERR_UNSUPPORTED, "page size %lld: must be 8, 16, 32, 64 or a multiple of 128", (long long)psz);
  if (k->stride[2] != sh->d) return fail(FD_ERR_UNSUPPORTED, "token rows of a page must be contiguous (stride[2] == head_dim)");
  if (sh->B > 0 && (!k->data || !v->data)) return fail(FD_ERR_INVALID_ARGUMENT, "k_pages / v_pages data is NULL");
  if (!aligned16(k->data) || !aligned16(v->data) || !stride16(k->stride[0], kvt) || !stride16(k->stride[1], kvt))
    return fail(FD_ERR_UNSUPPORTED, "page data and strides must be 16-byte aligned");
  if (sh->B > 0 && !pg.block_table) return fail(FD_ERR_INVALID_ARGUMENT, "block_table is NULL");
  if (pg.pages_per_seq < 1) return fail(FD_ERR_INVALID_ARGUMENT, "pages_per_seq must be >= 1");
  if (static_cast<int64_t>(pg.pages_per_seq) * psz > INT32_MAX)
    return fail(FD_ERR_UNSUPPORTED, "pages_per_seq * page_size exceeds 2^31 keys");
  pg.page_size = static_cast<int32_t>(psz);
  sh->hkv = static_cast<int>(k->shape[1]);
  sh->cap = pg.pages_per_seq * pg.page_size;
  if (sh->hq < 1 || sh->hq % sh->hkv != 0)
    return fail(FD_ERR_INVALID_ARGUMENT, "q heads (%d) must be a positive multiple of KV heads (%d)", sh->hq, sh->hkv);
  sh->g = sh->hq / sh->hkv;
  if (sh->B > kMaxPlanBatch) return fail(FD_ERR_UNSUPPORTED, "batch %d exceeds %d", sh->B, kMaxPlanBatch);
  return choose_kernel(sh);
}

int decode_ctas(int dev, bool use_tc) {
  const int n = sm_count(dev);
  return use_tc ? n : n * simt_ctas_per_sm();
}

size_t decode_ws_bytes(int B, int hq, int hkv, int cap, int d, int fixed, int nctas) {
  const int64_t items = decode_max_items(B, hkv, cap, fixed, nctas);
  return ws_layout(items, 0, B, items, hq, d, hkv).total;
}

// ---------------------------------------------------------------------------- host planner ---
struct HostPlan {
  int32_t chunk = 0;
  std::vector<int32_t> lens, nsplit, order;
  int64_t total_items = 0;
};

void host_plan(const int32_t* lens_in, int B, int hkv, int cap, int fixed, int nctas, HostPlan* hp) {
  hp->lens.resize(B);
  hp->nsplit.resize(B);
  int64_t total = 0;
  for (int b = 0; b < B; ++b) {
    hp->lens[b] = clamp_len(lens_in[b], cap);
    total += hp->lens[b];
  }
  hp->chunk = 0;
  if (fixed <= 0) {
    int32_t chunks[kPlanWaveChoices];
    int64_t sums[kPlanWaveChoices];
    for (int i = 0; i < kPlanWaveChoices; ++i) {
      chunks[i] = plan_chunk_for_waves(total, hkv, nctas, plan_waves(i));
      sums[i] = 0;
      for (int b = 0; b < B; ++b) sums[i] += plan_num_splits(hp->lens[b], chunks[i], 0);
    }
    hp->chunk = plan_pick_chunk(chunks, sums, hkv, nctas);
  }
  std::vector<int32_t> key(B);
  hp->total_items = 0;
  for (int b = 0; b < B; ++b) {
    hp->nsplit[b] = plan_num_splits(hp->lens[b], hp->chunk, fixed);
    key[b] = plan_sort_key(hp->lens[b], hp->nsplit[b]);
    hp->total_items += static_cast<int64_t>(hp->nsplit[b]) * hkv;
  }
  hp->order.resize(B);
  for (int b = 0; b < B; ++b) hp->order[b] = b;
  std::stable_sort(hp->order.begin(), hp->order.end(), [&](int a, int c) { return key[a] > key[c]; });
}

void prof_start(cudaEvent_t* ev, int seg, cudaStream_t stream) {
  if (ev) cudaEventRecord(ev[2 * seg], stream);
}
void prof_end(cudaEvent_t* ev, int seg, cudaStream_t stream) {
  if (ev) cudaEventRecord(ev[2 * seg + 1], stream);
}
// a segment the call does not launch: both events at this point of the stream
void prof_empty(cudaEvent_t* ev, int seg, cudaStream_t stream) {
  prof_start(ev, seg, stream);
  prof_end(ev, seg, stream);
}

}  // namespace fd_abi

using namespace fd_abi;

// ================================================================================ ABI ========
extern "C" {

const char* fd_status_string(fd_status s) {
  switch (s) {
    case FD_OK: return "FD_OK";
    case FD_ERR_INVALID_ARGUMENT: return "FD_ERR_INVALID_ARGUMENT";
    case FD_ERR_UNSUPPORTED: return "FD_ERR_UNSUPPORTED";
    case FD_ERR_CUDA: return "FD_ERR_CUDA";
    case FD_ERR_WORKSPACE: return "FD_ERR_WORKSPACE";
  }
  return "FD_UNKNOWN_STATUS";
}

const char* fd_last_error_message(void) { return g_last_error.c_str(); }

int32_t fd_decode_num_ctas(int32_t device, int32_t dtype, int32_t group_size, int32_t head_dim) {
  const bool tc = (dtype == FD_BF16 && head_dim == 128 && group_size >= 2 && group_size <= 16) ||
                  (dtype == FD_E4M3 && head_dim == 128 && group_size >= 1 && group_size <= 8);
  return decode_ctas(device, tc);
}

size_t fd_decode_workspace_bytes(int32_t batch, int32_t num_q_heads, int32_t num_kv_heads,
                                 int32_t cache_capacity, int32_t head_dim, int32_t num_splits,
                                 int32_t num_ctas) {
  if (batch < 0 || num_q_heads < 1 || num_kv_heads < 1 || cache_capacity < 0 || head_dim < 1 || num_splits < 0)
    return 0;
  return decode_ws_bytes(batch, num_q_heads, num_kv_heads, cache_capacity, head_dim, num_splits,
                         num_ctas);
}

fd_status fd_split_plan(const int32_t* cache_lens_host, int32_t batch, int32_t num_kv_heads,
                        int32_t cache_capacity, int32_t num_splits, int32_t num_ctas,
                        int32_t key_align, int32_t* splits_per_seq_host, int32_t* items_host,
                        int32_t items_capacity, fd_plan_info* info) {
  if (!info) return fail(FD_ERR_INVALID_ARGUMENT, "info is NULL");
  if (batch < 0) return fail(FD_ERR_INVALID_ARGUMENT, "batch must be >= 0");
  if (batch > 0 && !cache_lens_host) return fail(FD_ERR_INVALID_ARGUMENT, "cache_lens_host is NULL");
  if (num_kv_heads < 1) return fail(FD_ERR_INVALID_ARGUMENT, "num_kv_heads must be >= 1");
  if (cache_capacity < 0) return fail(FD_ERR_INVALID_ARGUMENT, "cache_capacity must be >= 0");
  if (num_splits < 0) return fail(FD_ERR_INVALID_ARGUMENT, "num_splits must be >= 0");
  if (num_ctas < 1) return fail(FD_ERR_INVALID_ARGUMENT, "num_ctas must be >= 1");
  if (key_align < 1) return fail(FD_ERR_INVALID_ARGUMENT, "key_align must be >= 1");
  if (items_host && items_capacity < 0) return fail(FD_ERR_INVALID_ARGUMENT, "items_capacity must be >= 0");
  HostPlan hp;
  host_plan(cache_lens_host, batch, num_kv_heads, cache_capacity, num_splits, num_ctas, &hp);
  if (hp.total_items > INT32_MAX) return fail(FD_ERR_UNSUPPORTED, "plan has more than 2^31 items");
  int32_t maxs = 0;
  for (int b = 0; b < batch; ++b) {
    if (splits_per_seq_host) splits_per_seq_host[b] = hp.nsplit[b];
    maxs = std::max(maxs, hp.nsplit[b]);
  }
  if (items_host) {
    int64_t i = 0;
    for (int r = 0; r < batch && i < items_capacity; ++r) {
      const int b = hp.order[r];
      const int n = hp.nsplit[b];
      for (int h = 0; h < num_kv_heads && i < items_capacity; ++h)
        for (int s = 0; s < n && i < items_capacity; ++s, ++i) {
          int32_t t0, t1;
          plan_split_range(hp.lens[b], n, s, num_splits, key_align, &t0, &t1);
          int32_t* o = items_host + 5 * i;
          o[0] = b; o[1] = h; o[2] = s; o[3] = t0; o[4] = t1;
        }
    }
  }
  info->chunk_tokens = hp.chunk;
  info->total_items = static_cast<int32_t>(hp.total_items);
  info->max_splits_per_seq = maxs;
  info->num_ctas = num_ctas;
  // plan tables only: header, items and the per-row split tables
  info->workspace_bytes = ws_layout(hp.total_items, 0, batch, 0, 1, 1).total;
  return FD_OK;
}

fd_status fd_split_plan_device(const int32_t* cache_lens, int32_t batch, int32_t num_kv_heads,
                               int32_t cache_capacity, int32_t num_splits, int32_t num_ctas,
                               int32_t key_align, int32_t* splits_per_seq_dev, int32_t* items_dev,
                               int32_t items_capacity, int32_t* total_items_dev, void* stream_) {
  cudaStream_t stream = static_cast<cudaStream_t>(stream_);
  if (batch < 0 || batch > kMaxPlanBatch) return fail(FD_ERR_INVALID_ARGUMENT, "batch must be in [0, %d]", kMaxPlanBatch);
  if (batch > 0 && (!cache_lens || !splits_per_seq_dev)) return fail(FD_ERR_INVALID_ARGUMENT, "NULL device pointer");
  if (!total_items_dev) return fail(FD_ERR_INVALID_ARGUMENT, "total_items_dev is NULL");
  if (num_kv_heads < 1 || cache_capacity < 0 || num_splits < 0 || num_ctas < 1 || key_align < 1)
    return fail(FD_ERR_INVALID_ARGUMENT, "bad plan arguments");
  if (items_dev && items_capacity < 0) return fail(FD_ERR_INVALID_ARGUMENT, "items_capacity must be >= 0");
  const int64_t items = decode_max_items(batch, num_kv_heads, cache_capacity, num_splits, num_ctas);
  const WsLayout L = ws_layout(items, 0, batch, 0, 1, 1, num_kv_heads);
  void* ws = nullptr;
  fd_status s = get_workspace(stream, L.total, &ws);
  if (s != FD_OK) return s;
  char* base = static_cast<char*>(ws);
  PlanParams pp{};
  pp.lens = cache_lens;
  pp.B = batch;
  pp.hkv = num_kv_heads;
  pp.hq = num_kv_heads;
  pp.cap = cache_capacity;
  pp.fixed = num_splits;
  pp.nctas = num_ctas;
  pp.align = key_align;
  pp.max_dec_items = items;
  pp.hdr = reinterpret_cast<WsHeader*>(base);
  pp.items = reinterpret_cast<DecodeItem*>(base + L.dec_items);
  pp.row_nsplit = reinterpret_cast<int32_t*>(base + L.row_nsplit);
  pp.row_base = reinterpret_cast<int32_t*>(base + L.row_base);
  pp.arrivals = reinterpret_cast<int32_t*>(base + L.arrivals);
  pp.out_splits = splits_per_seq_dev;
  pp.out_items = items_dev;
  pp.out_cap = items_dev ? items_capacity : 0;
  pp.out_total = total_items_dev;
  FD_CUDA(launch_plan_decode(pp, stream), "plan kernel launch");
  return FD_OK;
}

}  // extern "C"

namespace fd_abi {

// The decode call of both entry points: a contiguous cache (pg == nullptr) or a paged one.
fd_status decode_call(const fd_tensor* q, const fd_tensor* k_cache, const fd_tensor* v_cache,
                      const int32_t* cache_lens, int32_t num_splits, fd_tensor* out, float* lse,
                      cudaStream_t stream, PagedCache* pg, const KvQuant* quant,
                      const PresetScratch* preset) {
  DecodeShape sh{};
  fd_status s = pg ? resolve_paged(q, k_cache, v_cache, *pg, out, &sh, quant)
                   : resolve_decode(q, k_cache, v_cache, out, &sh, quant);
  if (s != FD_OK) return s;
  if (num_splits < 0) return fail(FD_ERR_INVALID_ARGUMENT, "num_splits must be >= 0");
  if (num_splits > 65536) return fail(FD_ERR_UNSUPPORTED, "num_splits above 65536");
  if (sh.B == 0) return FD_OK;
  if (!cache_lens) return fail(FD_ERR_INVALID_ARGUMENT, "cache_lens is NULL");
  if (!lse) return fail(FD_ERR_INVALID_ARGUMENT, "lse is NULL");
  int dev = 0;
  FD_CUDA(cudaGetDevice(&dev), "cudaGetDevice");
  const int nctas = decode_ctas(dev, sh.use_tc);
  if (nctas < 1) return fail(FD_ERR_CUDA, "no multiprocessors reported for device %d", dev);

  const int64_t max_items = decode_max_items(sh.B, sh.hkv, sh.cap, num_splits, nctas);
  const int64_t max_slots = max_items;  // one partial slot (G heads) per split item
  const WsLayout L = ws_layout(max_items, 0, sh.B, max_slots, sh.hq, sh.d, sh.hkv);
  void* ws = nullptr;
  if (preset) {
    if (L.total > preset->bytes)
      return fail(FD_ERR_UNSUPPORTED,
                  "this decode shape needs up to %zu bytes of scratch, more than the %zu bytes of "
                  "the %s; use fd_decode_attention",
                  L.total, preset->bytes, preset->name);
    ws = preset->base;
  } else if ((s = get_workspace(stream, L.total, &ws)) != FD_OK) {
    return s;
  }
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
  dp.q_box_rows = std::min(16, sh.hq);
  dp.kv_box_rows = std::min(128, pg ? pg->page_size : sh.cap);
  if (pg) {
    dp.block_table = pg->block_table;
    dp.pages_per_seq = pg->pages_per_seq;
    dp.page_size = pg->page_size;
    dp.num_pages = static_cast<int32_t>(std::min<int64_t>(k_cache->shape[0], INT32_MAX));
    dp.align = kPagedKeyAlign;
  } else {
    // the tensor-core kernel reads whole 128-key tiles: with a bf16 cache, splits that end on a
    // tile boundary (no partly used tile in the middle of a sequence) run ~2% faster at the
    // 70B-like shape; an E4M3 cache runs ~2% slower that way (225 vs 230 us, measured A/B; 20%
    // before the wait loop went out of line), so it keeps unaligned splits
    dp.align = (sh.use_tc && !sh.kv_fp8) ? kTcKeyAlign : 1;
  }
  // an E4M3 cache: k_scale multiplies every score, v_scale every output (both linear)
  dp.scale_log2 = static_cast<float>(1.0 / std::sqrt(static_cast<double>(sh.d)) * 1.4426950408889634 *
                                     (quant ? static_cast<double>(quant->k_scale) : 1.0));
  dp.v_scale = quant ? quant->v_scale : 1.f;
  dp.kv_fp8 = sh.kv_fp8 ? 1 : 0;
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
    // contiguous: (D, S_cap, Hkv, B); paged: (D, page_size, Hkv, num_pages)
    const uint64_t rows = pg ? static_cast<uint64_t>(pg->page_size) : static_cast<uint64_t>(sh.cap);
    const uint64_t outer = static_cast<uint64_t>(k_cache->shape[0]);
    // bf16: boxes of 64 elements (one 128-byte swizzle row), two per tile row; E4M3: one box of
    // 128 one-byte codes per tile row
    const uint64_t es = sh.kv_fp8 ? 1 : 2;
    const uint64_t kd[4] = {static_cast<uint64_t>(sh.d), rows, static_cast<uint64_t>(sh.hkv), outer};
    const uint64_t ks[3] = {static_cast<uint64_t>(k_cache->stride[2]) * es, static_cast<uint64_t>(k_cache->stride[1]) * es,
                            static_cast<uint64_t>(k_cache->stride[0]) * es};
    const uint32_t kb[4] = {sh.kv_fp8 ? 128u : 64u, static_cast<uint32_t>(dp.kv_box_rows), 1, 1};
    const CUtensorMapDataType kt = sh.kv_fp8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    // bf16 pages of < 128 keys with their KV heads one after another: 5-D maps (64 columns,
    // 8 rows 256 bytes apart, 2 halves 128 bytes apart, Hkv * page_size / 8 row groups 2048
    // bytes apart, pages) whose box is a whole page, laid out as the tensor-core kernel's
    // interleaved tile (one copy per page instead of two). Where the driver rejects a map of
    // such strides, the 4-D maps below serve.
    if (pg && !sh.kv_fp8 && pg->page_size < 128 &&
        k_cache->stride[1] == static_cast<int64_t>(pg->page_size) * sh.d) {
      const uint64_t groups = static_cast<uint64_t>(pg->page_size / 8) * static_cast<uint64_t>(sh.hkv);
      const uint64_t id[5] = {64, 8, 2, groups, outer};
      const uint64_t is[4] = {256, 128, 2048, static_cast<uint64_t>(k_cache->stride[0]) * 2};
      const uint32_t ib[5] = {64, 8, 2, static_cast<uint32_t>(pg->page_size / 8), 1};
      if (encode_tmap(&tk, k_cache->data, 5, id, is, ib, kt) == CUDA_SUCCESS &&
          encode_tmap(&tv, v_cache->data, 5, id, is, ib, kt) == CUDA_SUCCESS)
        dp.pg_interleave = 1;
    }
    if (!dp.pg_interleave) {
      if ((s = make_tmap(&tk, k_cache->data, 4, kd, ks, kb, "k_cache", kt)) != FD_OK) return s;
      if ((s = make_tmap(&tv, v_cache->data, 4, kd, ks, kb, "v_cache", kt)) != FD_OK) return s;
    }
  }

  PlanParams pp{};
  pp.lens = cache_lens;
  pp.B = sh.B;
  pp.hkv = sh.hkv;
  pp.hq = sh.hq;
  pp.cap = sh.cap;
  pp.fixed = num_splits;
  pp.nctas = nctas;
  pp.align = dp.align;
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


  // The tensor-core kernel plans small batches itself (every CTA computes the plan in shared
  // memory, CTA 0 writes the combine's row tables): no planner launch, no items in memory.
  const bool fused_plan = sh.use_tc && sh.B <= kFusedPlanMaxBatch;
  if (fused_plan) {
    dp.items = nullptr;
    dp.lens = cache_lens;
    dp.B = sh.B;
    dp.fixed = num_splits;
    dp.plan_ctas = nctas;
    dp.max_items = static_cast<int32_t>(std::min<int64_t>(max_items, INT32_MAX));
    dp.row_nsplit_out = row_nsplit;
    dp.row_base_out = row_base;
  }

  if (preset) {
    // scratch shared with other calls: the cursors must start at zero whatever the last call
    // left; the status word (offset 0) is kept until it is polled
    static_assert(offsetof(WsHeader, status) == 0, "status word first");
    FD_CUDA(cudaMemsetAsync(base + sizeof(uint32_t), 0, sizeof(WsHeader) - sizeof(uint32_t), stream),
            "clear scratch header");
  }

  cudaEvent_t* ev = prof_next();
  prof_start(ev, kSegPlan, stream);
  if (!fused_plan) FD_CUDA(launch_plan_decode(pp, stream), "plan kernel launch");
  prof_end(ev, kSegPlan, stream);
  prof_start(ev, kSegSplit, stream);
  if (sh.use_tc) {
    FD_CUDA(launch_decode_tc(dp, tq, tk, tv, nctas, stream), "tensor-core split kernel launch");
  } else {
    FD_CUDA(launch_decode_simt(dp, sh.dtype, nctas, stream), "split kernel launch");
  }
  prof_end(ev, kSegSplit, stream);
  prof_empty(ev, kSegTiles, stream);  // no chunk tiles in a decode call
  // the CUDA-core kernel merges each group's partials itself; the tensor-core kernel leaves them
  // to the combine kernel
  prof_start(ev, kSegCombine, stream);
  if (sh.use_tc) FD_CUDA(launch_combine(cp, stream), "combine kernel launch");
  prof_end(ev, kSegCombine, stream);
  return FD_OK;
}

}  // namespace fd_abi

extern "C" {

fd_status fd_decode_attention(const fd_tensor* q, const fd_tensor* k_cache,
                              const fd_tensor* v_cache, const int32_t* cache_lens,
                              int32_t num_splits, fd_tensor* out, float* lse, void* stream) {
  return decode_call(q, k_cache, v_cache, cache_lens, num_splits, out, lse,
                     static_cast<cudaStream_t>(stream), nullptr);
}

fd_status fd_decode_attention_paged(const fd_tensor* q, const fd_tensor* k_pages,
                                    const fd_tensor* v_pages, const int32_t* block_table,
                                    int32_t pages_per_seq, const int32_t* cache_lens,
                                    int32_t num_splits, fd_tensor* out, float* lse,
                                    void* stream) {
  PagedCache pg{};
  pg.block_table = block_table;
  pg.pages_per_seq = pages_per_seq;
  return decode_call(q, k_pages, v_pages, cache_lens, num_splits, out, lse,
                     static_cast<cudaStream_t>(stream), &pg);
}

fd_status fd_decode_attention_fp8(const fd_tensor* q, const fd_tensor* k_cache,
                                  const fd_tensor* v_cache, float k_scale, float v_scale,
                                  const int32_t* cache_lens, int32_t num_splits, fd_tensor* out,
                                  float* lse, void* stream) {
  const KvQuant quant{k_scale, v_scale};
  return decode_call(q, k_cache, v_cache, cache_lens, num_splits, out, lse,
                     static_cast<cudaStream_t>(stream), nullptr, &quant);
}

fd_status fd_decode_attention_paged_fp8(const fd_tensor* q, const fd_tensor* k_pages,
                                        const fd_tensor* v_pages, float k_scale, float v_scale,
                                        const int32_t* block_table, int32_t pages_per_seq,
                                        const int32_t* cache_lens, int32_t num_splits,
                                        fd_tensor* out, float* lse, void* stream) {
  const KvQuant quant{k_scale, v_scale};
  PagedCache pg{};
  pg.block_table = block_table;
  pg.pages_per_seq = pages_per_seq;
  return decode_call(q, k_pages, v_pages, cache_lens, num_splits, out, lse,
                     static_cast<cudaStream_t>(stream), &pg, &quant);
}

fd_status fd_chunk_prefill_attention(const fd_tensor* q_chunk, const fd_tensor* k_cache,
                                     const fd_tensor* v_cache, const int32_t* prefix_lens,
                                     const int32_t* chunk_lens, fd_tensor* out, float* lse,
                                     void* stream_) {
  cudaStream_t stream = static_cast<cudaStream_t>(stream_);
  fd_status s;
  if ((s = check_q_out(q_chunk, out, "q_chunk")) != FD_OK) return s;
  const int T = static_cast<int>(q_chunk->shape[0]);
  const int hq = static_cast<int>(q_chunk->shape[1]);
  const int d = static_cast<int>(q_chunk->shape[2]);
  if (q_chunk->dtype != FD_BF16) return fail(FD_ERR_UNSUPPORTED, "chunked prefill needs bf16 tensors");
  if (d != 64 && d != 128) return fail(FD_ERR_UNSUPPORTED, "chunked prefill supports head_dim 64 and 128, got %d", d);
  if (!k_cache) return fail(FD_ERR_INVALID_ARGUMENT, "k_cache is NULL");
  const int B = static_cast<int>(k_cache->shape[0]);
  if ((s = check_kv(k_cache, v_cache, FD_BF16, B, d)) != FD_OK) return s;
  const int hkv = static_cast<int>(k_cache->shape[1]);
  const int cap = static_cast<int>(k_cache->shape[2]);
  if (hq < 1 || hq % hkv != 0)
    return fail(FD_ERR_INVALID_ARGUMENT, "q heads (%d) must be a positive multiple of KV heads (%d)", hq, hkv);
  const int g = hq / hkv;
  if (g > 16) return fail(FD_ERR_UNSUPPORTED, "group size %d above 16", g);
  if (d == 64 && g > 8)
    return fail(FD_ERR_UNSUPPORTED, "group size %d above 8 needs head_dim 128 (its decode rows run on tensor cores)", g);
  if (B > kMaxPlanBatch) return fail(FD_ERR_UNSUPPORTED, "batch %d exceeds %d", B, kMaxPlanBatch);
  if (T == 0) return FD_OK;
  if (B == 0) return fail(FD_ERR_INVALID_ARGUMENT, "q_chunk has %d rows but the cache has no request", T);
  if (!prefix_lens || !chunk_lens) return fail(FD_ERR_INVALID_ARGUMENT, "prefix_lens / chunk_lens is NULL");
  if (!lse) return fail(FD_ERR_INVALID_ARGUMENT, "lse is NULL");
  int dev = 0;
  FD_CUDA(cudaGetDevice(&dev), "cudaGetDevice");
  // decode rows with head_dim 128 use the tensor-core decode kernel (for G = 1 too: beside the
  // tile kernel it streams more per multiprocessor than the CUDA-core kernel, 611 against 635 µs
  // per call at workload 5), the others the CUDA-core one
  const bool dec_tc = d == 128;
  const int dec_ctas = decode_ctas(dev, dec_tc);
  const int tile_ctas = sm_count(dev);
  if (dec_ctas < 1 || tile_ctas < 1) return fail(FD_ERR_CUDA, "no multiprocessors reported for device %d", dev);

  const int64_t max_dec = decode_max_items(B, hkv, cap, 0, dec_ctas);
  const int64_t max_tiles = chunk_max_tile_items(B, T, hq, cap);
  const int64_t max_slots = chunk_max_slots(B, T, hkv, cap, dec_ctas);
  const WsLayout L = ws_layout(max_dec, max_tiles, static_cast<int64_t>(T) + 1, max_slots, hq, d, hkv);
  void* ws = nullptr;
  Workspace wv;
  if ((s = get_workspace(stream, L.total, &ws, &wv)) != FD_OK) return s;
  char* base = static_cast<char*>(ws);
  WsHeader* hdr = reinterpret_cast<WsHeader*>(base);
  DecodeItem* items = reinterpret_cast<DecodeItem*>(base + L.dec_items);
  TileItem* tiles = reinterpret_cast<TileItem*>(base + L.tile_items);
  int32_t* row_nsplit = reinterpret_cast<int32_t*>(base + L.row_nsplit);
  int32_t* row_base = reinterpret_cast<int32_t*>(base + L.row_base);
  int32_t* arrivals = reinterpret_cast<int32_t*>(base + L.arrivals);
  float* part_o = reinterpret_cast<float*>(base + L.part_o);
  float* part_lse = reinterpret_cast<float*>(base + L.part_lse);
  const float scale_log2 = static_cast<float>(1.0 / std::sqrt(static_cast<double>(d)) * 1.4426950408889634);

  PlanParams pp{};
  pp.lens = prefix_lens;
  pp.chunk_lens = chunk_lens;
  pp.B = B;
  pp.hkv = hkv;
  pp.hq = hq;
  pp.cap = cap;
  pp.nctas = dec_ctas;
  pp.max_dec_items = max_dec;
  pp.max_tile_items = max_tiles;
  pp.hdr = hdr;
  pp.items = items;
  pp.tiles = tiles;
  pp.row_nsplit = row_nsplit;
  pp.row_base = row_base;
  pp.arrivals = arrivals;
  pp.total_rows = T;
  pp.decode_merged_in_kernel = dec_tc ? 0 : 1;
  pp.align = dec_tc ? kTcKeyAlign : 1;  // decode rows' split boundaries
  pp.tile_sms = tile_ctas;
  pp.kv_key_bytes = 2ll * hkv * d * 2;

  DecodeParams dp{};
  dp.q = q_chunk->data;
  dp.q_sr = q_chunk->stride[0];
  dp.q_sh = q_chunk->stride[1];
  dp.k = k_cache->data;
  dp.v = v_cache->data;
  dp.kv_sb = k_cache->stride[0];
  dp.kv_sh = k_cache->stride[1];
  dp.out = out->data;
  dp.o_sr = out->stride[0];
  dp.o_sh = out->stride[1];
  dp.lse = lse;
  dp.hq = hq;
  dp.hkv = hkv;
  dp.g = g;
  dp.d = d;
  dp.cap = cap;
  dp.q_box_rows = std::min(16, hq);
  dp.kv_box_rows = std::min(128, cap);
  dp.scale_log2 = scale_log2;
  dp.hdr = hdr;
  dp.items = items;
  dp.row_base = row_base;
  dp.part_o = part_o;
  dp.part_lse = part_lse;
  dp.arrivals = arrivals;

  TileParams tp{};
  tp.q = q_chunk->data;
  tp.q_sr = q_chunk->stride[0];
  tp.q_sh = q_chunk->stride[1];
  tp.out = out->data;
  tp.o_sr = out->stride[0];
  tp.o_sh = out->stride[1];
  tp.lse = lse;
  tp.hq = hq;
  tp.hkv = hkv;
  tp.g = g;
  tp.d = d;
  tp.cap = cap;
  tp.q_box_rows = std::min(128, T);
  tp.qp_box_rows = std::min(kQTile / g, T);
  tp.quad_rows = g >= 2 ? 32 / g : 0;
  tp.qq_box_rows = std::min(std::max(tp.quad_rows, 1), T);
  tp.g_recip16 = (65536 + g - 1) / g;
  tp.kv_box_rows = std::min(128, cap);
  tp.scale_log2 = scale_log2;
  tp.hdr = hdr;
  tp.tiles = tiles;
  tp.part_o = part_o;
  tp.part_lse = part_lse;

  CombineParams cp{};
  cp.row_nsplit = row_nsplit;
  cp.row_base = row_base;
  cp.part_o = part_o;
  cp.part_lse = part_lse;
  cp.out = out->data;
  cp.o_sr = out->stride[0];
  cp.o_sh = out->stride[1];
  cp.lse = lse;
  cp.rows = T;
  cp.hq = hq;
  cp.hkv = hkv;
  cp.g = g;
  cp.d = d;
  cp.dtype = FD_BF16;

  // tensor maps: q as (D, Hq, T); caches as (D, S_cap, Hkv, B)
  CUtensorMap tq_dec, tq_tile, tk, tv;
  const uint64_t qd[3] = {static_cast<uint64_t>(d), static_cast<uint64_t>(hq), static_cast<uint64_t>(T)};
  const uint64_t qs[2] = {static_cast<uint64_t>(q_chunk->stride[1]) * 2, static_cast<uint64_t>(q_chunk->stride[0]) * 2};
  const uint32_t qb_dec[3] = {64, static_cast<uint32_t>(dp.q_box_rows), 1};
  const uint32_t qb_tile[3] = {64, 1, static_cast<uint32_t>(tp.q_box_rows)};
  if ((s = make_tmap(&tq_tile, q_chunk->data, 3, qd, qs, qb_tile, "q_chunk")) != FD_OK) return s;
  // head-packed tiles (groups >= 2): G heads x 128 / G rows per box
  CUtensorMap tq_packed = tq_tile;
  const uint32_t qb_packed[3] = {64, static_cast<uint32_t>(g), static_cast<uint32_t>(tp.qp_box_rows)};
  if (g >= 2 && (s = make_tmap(&tq_packed, q_chunk->data, 3, qd, qs, qb_packed, "q_chunk (head-packed)")) != FD_OK)
    return s;
  // quarter items (head-packed requests of <= 32 / G rows): G heads x 32 / G rows per box
  CUtensorMap tq_quarter = tq_tile;
  const uint32_t qb_quarter[3] = {64, static_cast<uint32_t>(g), static_cast<uint32_t>(tp.qq_box_rows)};
  if (tp.quad_rows > 0 &&
      (s = make_tmap(&tq_quarter, q_chunk->data, 3, qd, qs, qb_quarter, "q_chunk (quarter items)")) != FD_OK)
    return s;
  const uint64_t kd[4] = {static_cast<uint64_t>(d), static_cast<uint64_t>(cap), static_cast<uint64_t>(hkv), static_cast<uint64_t>(B)};
  const uint64_t ks[3] = {static_cast<uint64_t>(k_cache->stride[2]) * 2, static_cast<uint64_t>(k_cache->stride[1]) * 2,
                          static_cast<uint64_t>(k_cache->stride[0]) * 2};
  const uint32_t kb[4] = {64, static_cast<uint32_t>(dp.kv_box_rows), 1, 1};
  if ((s = make_tmap(&tk, k_cache->data, 4, kd, ks, kb, "k_cache")) != FD_OK) return s;
  if ((s = make_tmap(&tv, v_cache->data, 4, kd, ks, kb, "v_cache")) != FD_OK) return s;
  if (dec_tc && (s = make_tmap(&tq_dec, q_chunk->data, 3, qd, qs, qb_dec, "q_chunk (decode rows)")) != FD_OK) return s;

  // The planner, then the tile kernel on this stream beside the decode-row split kernel on the
  // side stream (forked after the planner, joined before the combine): the planner keeps
  // hdr->tile_ctas of the tile kernel's CTAs (the rest leave at once) so that the decode rows,
  // bound by HBM, stream on the other multiprocessors while the tiles, bound by the tensor
  // cores, run ("大语言模型长序列推理优化：ChunkedPrefill与FlashDecoding技术解析" §2.2: chunks
  // scheduled together with decode requests).
  cudaEvent_t* ev = prof_next();
  prof_start(ev, kSegPlan, stream);
  FD_CUDA(launch_plan_chunk(pp, stream), "chunk plan kernel launch");
  prof_end(ev, kSegPlan, stream);
  FD_CUDA(cudaEventRecord(wv.fork, stream), "record fork event");
  prof_start(ev, kSegTiles, stream);
  FD_CUDA(launch_chunk_tc(tp, tq_tile, tq_packed, tq_quarter, tk, tv, tile_ctas, stream),
          "chunk tile kernel launch");
  prof_end(ev, kSegTiles, stream);
  FD_CUDA(cudaStreamWaitEvent(wv.side, wv.fork, 0), "side stream waits for the planner");
  prof_start(ev, kSegSplit, wv.side);
  if (dec_tc) {
    FD_CUDA(launch_decode_tc(dp, tq_dec, tk, tv, dec_ctas, wv.side), "decode-row split kernel launch");
  } else {
    FD_CUDA(launch_decode_simt(dp, FD_BF16, dec_ctas, wv.side), "decode-row split kernel launch");
  }
  prof_end(ev, kSegSplit, wv.side);
  FD_CUDA(cudaEventRecord(wv.join, wv.side), "record join event");
  FD_CUDA(cudaStreamWaitEvent(stream, wv.join, 0), "stream waits for the decode rows");
  prof_start(ev, kSegCombine, stream);
  FD_CUDA(launch_combine(cp, stream), "combine kernel launch");
  prof_end(ev, kSegCombine, stream);
  return FD_OK;
}

size_t fd_chunk_workspace_bytes(int32_t batch, int32_t total_rows, int32_t num_q_heads,
                                int32_t num_kv_heads, int32_t cache_capacity, int32_t head_dim,
                                int32_t num_ctas) {
  if (batch < 0 || total_rows < 0 || num_q_heads < 1 || num_kv_heads < 1 || cache_capacity < 0 ||
      head_dim < 1 || num_ctas < 1)
    return 0;
  const int64_t max_dec = decode_max_items(batch, num_kv_heads, cache_capacity, 0, num_ctas);
  const int64_t max_tiles = chunk_max_tile_items(batch, total_rows, num_q_heads, cache_capacity);
  const int64_t max_slots = chunk_max_slots(batch, total_rows, num_kv_heads, cache_capacity, num_ctas);
  return ws_layout(max_dec, max_tiles, static_cast<int64_t>(total_rows) + 1, max_slots,
                   num_q_heads, head_dim, num_kv_heads).total;
}

fd_status fd_reserve_workspace(size_t bytes, void* stream_) {
  void* ws = nullptr;
  return get_workspace(static_cast<cudaStream_t>(stream_), std::max(bytes, sizeof(WsHeader)), &ws);
}

fd_status fd_poll_status(void* stream_, uint32_t* flags) {
  if (!flags) return fail(FD_ERR_INVALID_ARGUMENT, "flags is NULL");
  cudaStream_t stream = static_cast<cudaStream_t>(stream_);
  *flags = 0;
  int dev = 0;
  FD_CUDA(cudaGetDevice(&dev), "cudaGetDevice");
  FD_CUDA(cudaStreamSynchronize(stream), "cudaStreamSynchronize");
  void* ptr = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_mu);
    auto it = g_ws.find({dev, reinterpret_cast<uintptr_t>(stream)});
    if (it != g_ws.end()) ptr = it->second.ptr;
  }
  uint32_t v = 0;
  if (ptr) {
    FD_CUDA(cudaMemcpy(&v, ptr, sizeof(v), cudaMemcpyDeviceToHost), "read status");
    const uint32_t zero = 0;
    FD_CUDA(cudaMemcpy(ptr, &zero, sizeof(zero), cudaMemcpyHostToDevice), "clear status");
  }
  // the status bits of fd_decode_attention_static calls on this device
  uint32_t st = 0;
  fd_status s = static_scratch_take_status(&st);
  if (s != FD_OK) return s;
  *flags = v | st;
  return FD_OK;
}

fd_status fd_profile_begin(int32_t max_calls) {
  if (max_calls < 1) return fail(FD_ERR_INVALID_ARGUMENT, "max_calls must be >= 1");
  std::lock_guard<std::mutex> lock(g_prof.mu);
  for (cudaEvent_t e : g_prof.ev) cudaEventDestroy(e);
  g_prof.ev.assign(kProfEvents * static_cast<size_t>(max_calls), nullptr);
  for (auto& e : g_prof.ev) FD_CUDA(cudaEventCreate(&e), "cudaEventCreate");
  g_prof.max_calls = max_calls;
  g_prof.calls = 0;
  g_prof.active = true;
  return FD_OK;
}

fd_status fd_profile_end(float* ms, int32_t max_calls, int32_t* n_calls) {
  if (!ms || !n_calls) return fail(FD_ERR_INVALID_ARGUMENT, "NULL output");
  std::lock_guard<std::mutex> lock(g_prof.mu);
  if (!g_prof.active) return fail(FD_ERR_INVALID_ARGUMENT, "profiling was not started");
  const int n = std::min(g_prof.calls, max_calls);
  for (int i = 0; i < n; ++i) {
    cudaEvent_t* e = &g_prof.ev[kProfEvents * static_cast<size_t>(i)];
    for (int j = 0; j < kProfSegments; ++j) {
      FD_CUDA(cudaEventSynchronize(e[2 * j + 1]), "cudaEventSynchronize");
      FD_CUDA(cudaEventElapsedTime(&ms[kProfSegments * i + j], e[2 * j], e[2 * j + 1]), "cudaEventElapsedTime");
    }
  }
  *n_calls = n;
  for (cudaEvent_t e : g_prof.ev) cudaEventDestroy(e);
  g_prof.ev.clear();
  g_prof.active = false;
  g_prof.calls = 0;
  return FD_OK;
}

void fd_shutdown(void) {
  {
    std::lock_guard<std::mutex> lock(g_mu);
    for (auto& kv : g_ws) {
      int cur = 0;
      cudaGetDevice(&cur);
      cudaSetDevice(kv.first.first);
      cudaDeviceSynchronize();
      if (kv.second.ptr) cudaFree(kv.second.ptr);
      if (kv.second.side) cudaStreamDestroy(kv.second.side);
      if (kv.second.fork) cudaEventDestroy(kv.second.fork);
      if (kv.second.join) cudaEventDestroy(kv.second.join);
      cudaSetDevice(cur);
    }
    g_ws.clear();
  }
  std::lock_guard<std::mutex> lock(g_prof.mu);
  for (cudaEvent_t e : g_prof.ev) cudaEventDestroy(e);
  g_prof.ev.clear();
  g_prof.active = false;
}

}  // extern "C"
