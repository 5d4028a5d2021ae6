// fd_decode_attention_static: the decode attention call for callers that cannot allocate device
// memory. It is fd_decode_attention itself (the same argument checks, split plan, kernels and
// launch sequence, in fd_abi::decode_call), except that its scratch (the split plan, the work
// items and the per-split partial results) lives in one file-scope device array of
// FD_STATIC_SCRATCH_BYTES instead of the library's per-stream workspace, so the call itself never
// allocates.
//
// Who needs this: serving engines that hand nearly all of a GPU's memory to their own KV-cache
// pool (a late cudaMalloc would fail or fragment that pool), plugin hosts that only let a plugin
// use buffers the host has already allocated, and latency-critical loops where the implicit
// device synchronisation of cudaMalloc / cudaFree is not acceptable.
//
// Rules for callers (also stated in include/fd.h):
//  - Every GPU that loads this library holds the array until the process exits.
//  - The first call on a device looks up the array's device address with cudaGetSymbolAddress,
//    with that device current; make that first call before any stream capture begins. The
//    lookup is repeated when the device's current context changes (after a device reset).
//  - All calls share the one array, which keeps the previous call's contents: calls that overlap
//    on the GPU (other streams, or other host threads without ordering between them) race on it.
//    Each call clears, on its stream, the header fields that must start at zero.
//  - A shape whose worst-case scratch exceeds FD_STATIC_SCRATCH_BYTES is rejected on the host with
//    FD_ERR_UNSUPPORTED before anything is enqueued.
//  - Device status flags raised by these kernels stay in the array's header until fd_poll_status
//    reads and clears them.
#include <cuda.h>

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

struct StaticAddr {
  void* ptr;
  CUcontext ctx;  // the context the address belongs to
};
std::mutex g_static_mu;
std::map<int, StaticAddr> g_static_addr;  // device ordinal -> device address of the array

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);

// The driver's cuCtxGetCurrent (the runtime is linked statically; the driver entry point is
// fetched at run time, like cuTensorMapEncodeTiled).
CtxGetCurrentFn ctx_get_current_fn() {
  static std::once_flag once;
  static CtxGetCurrentFn fn = nullptr;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &f, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<CtxGetCurrentFn>(f);
  });
  return fn;
}

// The context current on the calling thread (nullptr when it cannot be read).
CUcontext current_context() {
  CtxGetCurrentFn fn = ctx_get_current_fn();
  CUcontext c = nullptr;
  if (!fn || fn(&c) != CUDA_SUCCESS) return nullptr;
  return c;
}

// True when `ctx` (the calling thread's current context, or nullptr if none is bound yet) may be
// the context an address was taken in: only two known contexts that differ rule it out.
bool same_context(CUcontext stored, CUcontext ctx) {
  return stored == nullptr || ctx == nullptr || stored == ctx;
}

// Device address of the array on device `dev` (the current device): looked up once per device,
// and again when the device's context is no longer the one the address was taken in (a device
// reset destroys that context).
fd_status static_scratch_address(int dev, void** out) {
  const CUcontext ctx = current_context();
  std::lock_guard<std::mutex> lock(g_static_mu);
  auto it = g_static_addr.find(dev);
  if (it != g_static_addr.end() && same_context(it->second.ctx, ctx)) {
    *out = it->second.ptr;
    return FD_OK;
  }
  void* ptr = nullptr;
  cudaError_t e = cudaGetSymbolAddress(&ptr, g_fd_static_scratch);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(static scratch)");
  if (!ptr) return fail(FD_ERR_CUDA, "cudaGetSymbolAddress returned a null static scratch address");
  // the runtime call above has made the device's primary context current on this thread
  g_static_addr[dev] = StaticAddr{ptr, current_context()};
  *out = ptr;
  return FD_OK;
}

}  // namespace

namespace fd_abi {

fd_status static_scratch_take_status(uint32_t* flags) {
  *flags = 0;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  void* ptr = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_static_mu);
    auto it = g_static_addr.find(dev);
    if (it == g_static_addr.end() || !same_context(it->second.ctx, current_context())) return FD_OK;
    ptr = it->second.ptr;
  }
  uint32_t v = 0;
  e = cudaMemcpy(&v, ptr, sizeof(v), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e, "read static scratch status");
  const uint32_t zero = 0;
  e = cudaMemcpy(ptr, &zero, sizeof(zero), cudaMemcpyHostToDevice);
  if (e != cudaSuccess) return cuda_fail(e, "clear static scratch status");
  *flags = v;
  return FD_OK;
}

}  // namespace fd_abi

extern "C" fd_status fd_decode_attention_static(const fd_tensor* q, const fd_tensor* k_cache,
                                                const fd_tensor* v_cache,
                                                const int32_t* cache_lens, int32_t num_splits,
                                                fd_tensor* out, float* lse, void* stream) {
  // shapes that are rejected or need no launch never touch the array
  DecodeShape sh{};
  fd_status s = resolve_decode(q, k_cache, v_cache, out, &sh);
  if (s != FD_OK) return s;
  PresetScratch scratch{nullptr, static_cast<size_t>(FD_STATIC_SCRATCH_BYTES),
                        "static scratch of fd_decode_attention_static"};
  if (sh.B > 0 && num_splits >= 0 && cache_lens && lse) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    if ((s = static_scratch_address(dev, &scratch.base)) != FD_OK) return s;
  }
  return decode_call(q, k_cache, v_cache, cache_lens, num_splits, out, lse,
                     static_cast<cudaStream_t>(stream), nullptr, nullptr, &scratch);
}
