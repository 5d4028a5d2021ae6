// Host-side helpers of the C ABI shared by its source files: error reporting, decode-call
// validation, tensor maps and launch geometry (defined in api.cu).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/fd.h"

namespace fd_abi {

// Record a formatted message for fd_last_error_message() and return `s`.
fd_status fail(fd_status s, const char* fmt, ...);
fd_status cuda_fail(cudaError_t e, const char* what);

struct DecodeShape {
  int B, hq, hkv, g, d, cap, dtype;
  bool use_tc;
  bool kv_fp8;  // the cache holds E4M3 codes (dtype is q's)
  int nctas;
};

// Scales of an FP8 (E4M3) cache: the cached value of code c is e4m3(c) * scale.
struct KvQuant {
  float k_scale, v_scale;
};

// Validate a decode call's tensors and choose its split kernel; `quant` != nullptr: the cache
// is E4M3 with those scales.
fd_status resolve_decode(const fd_tensor* q, const fd_tensor* k, const fd_tensor* v,
                         const fd_tensor* out, DecodeShape* sh, const KvQuant* quant = nullptr);

// A paged cache: K/V pages [num_pages, Hkv, page_size, D] read through a block table
// [B, pages_per_seq]. page_size is filled in by resolve_paged.
struct PagedCache {
  const int32_t* block_table;
  int32_t pages_per_seq;
  int32_t page_size;
};

// Validate a paged decode call (S_cap becomes pages_per_seq * page_size).
fd_status resolve_paged(const fd_tensor* q, const fd_tensor* k, const fd_tensor* v,
                        PagedCache& pg, const fd_tensor* out, DecodeShape* sh,
                        const KvQuant* quant = nullptr);

// Scratch memory a decode call uses instead of the library's per-stream workspace: `base` (256-byte
// aligned device memory of `bytes` bytes) holds the same layout. A shape whose worst-case
// scratch exceeds `bytes` is rejected with FD_ERR_UNSUPPORTED before anything is enqueued. The
// call clears the header's cursors on its stream first and keeps its status word.
struct PresetScratch {
  void* base;
  size_t bytes;
  const char* name;  // for the error message
};

// The decode call of fd_decode_attention (pg == nullptr) and fd_decode_attention_paged, and of
// their FP8 forms (quant != nullptr); with `preset`, in that scratch.
fd_status decode_call(const fd_tensor* q, const fd_tensor* k_cache, const fd_tensor* v_cache,
                      const int32_t* cache_lens, int32_t num_splits, fd_tensor* out, float* lse,
                      cudaStream_t stream, PagedCache* pg, const KvQuant* quant = nullptr,
                      const PresetScratch* preset = nullptr);

// The status word of the allocation-free entry point's scratch on the current device, read and
// cleared (0 when that scratch has not been set up on the device). The caller synchronises.
fd_status static_scratch_take_status(uint32_t* flags);

// Persistent CTAs of the split kernel on device `dev`.
int decode_ctas(int dev, bool use_tc);

// Tensor map with 128-byte swizzle (bf16 elements, or bytes for an E4M3 cache); dims / strides
// innermost first.
fd_status make_tmap(CUtensorMap* map, const void* base, int rank, const uint64_t* dims,
                    const uint64_t* strides_bytes, const uint32_t* box, const char* what,
                    CUtensorMapDataType dtype = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16);

}  // namespace fd_abi
