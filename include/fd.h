/*
 * fd.h — C ABI of the split-KV FlashDecoding attention library for NVIDIA B200 (sm_100a).
 *
 * The library computes attention of new query tokens against a KV cache:
 *
 *   out[b,h,:] = sum_j softmax_j(q[b,h,:]·k[b,kv,j,:] / sqrt(D)) · v[b,kv,j,:],  kv = h / (Hq/Hkv)
 *   lse[b,h]   = ln sum_j exp(q[b,h,:]·k[b,kv,j,:] / sqrt(D))                (natural log)
 *
 * over the keys j < cache_lens[b] (decode), or, for a query chunk, over the keys
 * j <= prefix_lens[b] + i for chunk row i (chunked prefill).
 *
 * Sources (web pages, cited by title and section):
 *  - "大语言模型长序列推理优化：ChunkedPrefill与FlashDecoding技术解析"
 *    (ChunkedPrefill and FlashDecoding), §2.1 chunk attention with the causal mask,
 *    §3.1 KV tiling (256-1024 tokens) and online-softmax reduction.
 *  - "大模型推理加速FlashDecoding算法原理与多GPU并行解码实战"
 *    (FlashDecoding algorithm and multi-GPU decoding): the Q/K/V shapes and split pass in
 *    "FlashDecoding算法原理与标准注意力机制对比", the cache_lens mask and the max/sum merge in
 *    "多GPU张量并行扩展下的FlashDecoding实现", the variable-length allocator in
 *    "Variable-Length序列动态切分策略", the contiguous KV layout, fp32 reduction and
 *    GQA-by-KV-head grouping in "部署落地的工程细节".
 *  - "Chunked-Prefills分块预填充机制：破解大模型推理的吞吐与延迟困局" §三.2 (a chunk attends to a
 *    reused prefix).
 *
 * Conventions shared by every entry point
 *  - Pointers named *_host are host memory; every other data pointer is device memory on the
 *    current CUDA device. The caller owns all tensors; the library never frees them.
 *  - `stream` is a cudaStream_t passed as void* (NULL = the legacy default stream). All
 *    attention calls are asynchronous on it: no host synchronisation and, once the workspace is
 *    reserved (fd_reserve_workspace), no allocation, so they may be captured in a CUDA graph.
 *  - The library owns one grow-only device workspace per (device, stream) for its split plan and
 *    partial results, freed by fd_shutdown(). A call whose workspace must grow synchronises that
 *    stream once before reallocating.
 *  - Errors: argument errors return before any launch (FD_ERR_INVALID_ARGUMENT /
 *    FD_ERR_UNSUPPORTED). CUDA errors map to FD_ERR_CUDA. fd_last_error_message() gives the
 *    detail for the calling thread. Nothing aborts or throws across the ABI.
 *  - Bad device data cannot be checked on the host: a cache length outside [0, S_cap] is clamped
 *    into that range on the device and raises FD_FLAG_LEN_CLAMPED in the device status word read
 *    by fd_poll_status(). Kernel waits are bounded; a wait that runs out raises
 *    FD_FLAG_WAIT_TIMEOUT instead of hanging.
 *  - Results are deterministic: a fixed merge order and no floating-point atomics.
 */
#ifndef FD_H_
#define FD_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  FD_OK = 0,
  FD_ERR_INVALID_ARGUMENT = 1, /* null pointer, inconsistent shapes, negative sizes         */
  FD_ERR_UNSUPPORTED = 2,      /* legal but not implemented: dtype, head_dim, layout         */
  FD_ERR_CUDA = 3,             /* a CUDA runtime / driver call failed                        */
  FD_ERR_WORKSPACE = 4         /* workspace allocation failed or is too small under capture  */
} fd_status;

/* FD_E4M3: one-byte OCP FP8 E4M3 codes (4 exponent bits, bias 7, 3 mantissa bits, no
 * infinities); a KV-cache dtype only, for the *_fp8 entry points. */
typedef enum { FD_F32 = 0, FD_BF16 = 1, FD_E4M3 = 2 } fd_dtype;

/* A strided device tensor. `stride` is in elements; the last dimension must be contiguous
 * (stride[ndim-1] == 1). Unused trailing shape/stride entries are ignored. */
typedef struct {
  void* data;
  int32_t dtype; /* fd_dtype */
  int32_t ndim;
  int64_t shape[4];
  int64_t stride[4];
} fd_tensor;

/* Summary of a split plan (fd_split_plan). */
typedef struct {
  int32_t chunk_tokens;       /* planner chunk (0 when num_splits > 0 fixes the split count)   */
  int32_t total_items;        /* work items = Hkv * sum of splits per sequence                 */
  int32_t max_splits_per_seq; /* largest split count of any sequence                           */
  int32_t num_ctas;           /* persistent CTAs the plan was made for                         */
  size_t workspace_bytes;     /* device workspace a decode call with this plan needs           */
} fd_plan_info;

/* Device status word bits (fd_poll_status). */
#define FD_FLAG_LEN_CLAMPED 0x1u  /* some cache/prefix/chunk length was outside [0, S_cap]     */
#define FD_FLAG_WAIT_TIMEOUT 0x2u /* a kernel wait gave up; the call's results are invalid     */
#define FD_FLAG_PLAN_OVERFLOW 0x4u /* the device plan exceeded the workspace bound (a bug)     */
#define FD_FLAG_BAD_PAGE 0x8u      /* a block-table entry of a used page was outside the pool   */

/*
 * fd_decode_attention — split-KV FlashDecoding decode attention (one query token per sequence).
 *
 * FlashDecoding page, "FlashDecoding算法原理与标准注意力机制对比": the cache of each sequence is
 * cut along the sequence axis into splits; every split yields a partial output and its
 * log-sum-exp under an online softmax (ChunkedPrefill page §3.1); a second pass merges the
 * splits by log-sum-exp ("多GPU张量并行扩展下的FlashDecoding实现", merge read with the per-split
 * sum of exponentials). One work item serves all Hq/Hkv query heads of a KV head, so K/V are
 * read once ("部署落地的工程细节", item 3).
 *
 *  q          [B, Hq, D]          dtype FD_F32 or FD_BF16; D in {64, 128}.
 *  k_cache    [B, Hkv, S_cap, D]  same dtype as q; Hq % Hkv == 0. Token rows of one (b, kv)
 *  v_cache    [B, Hkv, S_cap, D]  must be contiguous (stride[2] == D); all strides must be
 *                                 multiples of 16 bytes and data 16-byte aligned.
 *  cache_lens [B] int32 (device): keys j < cache_lens[b] are attended; 0 gives out = 0 and
 *                                 lse = -inf; values outside [0, S_cap] are clamped (status flag).
 *  num_splits > 0: every sequence gets exactly num_splits splits of ceil(len/num_splits) keys
 *             (trailing splits may be empty); 0: the variable-length planner chooses (see
 *             fd_split_plan); negative is an error.
 *  out        [B, Hq, D]          same dtype as q (written).
 *  lse        [B, Hq] float32 (device, contiguous, written): natural-log log-sum-exp of the
 *                                 scaled scores.
 *  stream     cudaStream_t.
 * B == 0 is a no-op. Returns FD_OK once all kernels are enqueued.
 */
fd_status fd_decode_attention(const fd_tensor* q, const fd_tensor* k_cache,
                              const fd_tensor* v_cache, const int32_t* cache_lens,
                              int32_t num_splits, fd_tensor* out, float* lse, void* stream);

/*
 * fd_decode_attention_paged — fd_decode_attention over a paged KV cache.
 *
 * The FlashDecoding page ("部署落地的工程细节") pairs split-KV decoding with a paged KV cache;
 * the pages give no layout, so this one is read as the usual block-table form: the cache of
 * sequence b is the sequence of pages block_table[b][0], block_table[b][1], ...; token t of
 * sequence b is row t % page_size of page block_table[b][t / page_size]. The result is exactly
 * fd_decode_attention's on the gathered contiguous cache. Splits are planned as in
 * fd_split_plan with key_align = 128, so no key tile crosses a page.
 *
 *  q            [B, Hq, D]                      as in fd_decode_attention.
 *  k_pages      [num_pages, Hkv, page_size, D]  the page pool (same dtype as q). page_size is
 *  v_pages      [num_pages, Hkv, page_size, D]  8, 16, 32, 64 or a multiple of 128. The rows of
 *                                               one (page, head) must be contiguous
 *                                               (stride[2] == D); strides multiples of 16 bytes,
 *                                               data 16-byte aligned; k and v share strides.
 *                                               Any page stride is accepted; bf16 pages of < 128
 *                                               keys whose heads are consecutive (stride[1] ==
 *                                               page_size * D) are read with one copy per page,
 *                                               other head strides with two.
 *  block_table  [B, pages_per_seq] int32 (device, contiguous rows): physical page of each
 *               logical page. Entries past a sequence's last page are never dereferenced as
 *               memory addresses (they may hold any value, e.g. -1).
 *  pages_per_seq >= 1: the table's row length; a sequence holds at most pages_per_seq *
 *               page_size keys, and longer cache_lens are clamped to that (status flag).
 *  cache_lens, num_splits, out, lse, stream: as in fd_decode_attention.
 * Table entries of pages a sequence uses must be valid page indices (0 <= id < num_pages). An
 * out-of-range index there is never dereferenced: that page's keys are not read (their contents
 * in the result are unspecified) and FD_FLAG_BAD_PAGE is raised.
 */
fd_status fd_decode_attention_paged(const fd_tensor* q, const fd_tensor* k_pages,
                                    const fd_tensor* v_pages, const int32_t* block_table,
                                    int32_t pages_per_seq, const int32_t* cache_lens,
                                    int32_t num_splits, fd_tensor* out, float* lse,
                                    void* stream);

/*
 * fd_decode_attention_fp8 — fd_decode_attention over an FP8 (E4M3) KV cache.
 *
 * The FlashDecoding page, section "与其他推理加速方案的组合使用" (combining FlashDecoding with
 * other speed-ups), item "Quantization + FlashDecoding", pairs split-KV decoding with an INT8/
 * FP8 cache whose values are dequantized to bf16 for the score computation. Format and scale
 * granularity are not given there; they are read as: E4M3 codes, one scale for all of K and one
 * for all of V, the cached value of code c being e4m3(c) * scale. Every E4M3 value is exact in
 * bf16 and in f16, so the kernel expands the codes without rounding (K to bf16, V to f16), folds
 * k_scale into the score scale and applies v_scale to the output: the result is the attention of
 * fd_decode_attention over the exact values e4m3(c) * scale, up to fp32 rounding. The NaN codes
 * (0x7F, 0xFF) must not occur among a sequence's valid keys (a quantized cache holds none); the
 * result is unspecified where they do.
 *
 *  q          [B, Hq, D]          FD_BF16; D == 128; group size Hq / Hkv <= 8.
 *  k_cache    [B, Hkv, S_cap, D]  FD_E4M3 (one byte per element); layout and alignment rules
 *  v_cache    [B, Hkv, S_cap, D]  as in fd_decode_attention (strides in bytes, multiples of 16).
 *  k_scale, v_scale               finite, > 0.
 *  cache_lens, num_splits, out (FD_BF16), lse, stream: as in fd_decode_attention.
 * Other dtypes, head sizes or group sizes return FD_ERR_UNSUPPORTED.
 */
fd_status fd_decode_attention_fp8(const fd_tensor* q, const fd_tensor* k_cache,
                                  const fd_tensor* v_cache, float k_scale, float v_scale,
                                  const int32_t* cache_lens, int32_t num_splits, fd_tensor* out,
                                  float* lse, void* stream);

/*
 * fd_decode_attention_paged_fp8 — fd_decode_attention_paged over FP8 (E4M3) pages, with the
 * scales of fd_decode_attention_fp8. k_pages / v_pages are FD_E4M3 [num_pages, Hkv, page_size,
 * D]; every other argument is as in those two calls.
 */
fd_status fd_decode_attention_paged_fp8(const fd_tensor* q, const fd_tensor* k_pages,
                                        const fd_tensor* v_pages, float k_scale, float v_scale,
                                        const int32_t* block_table, int32_t pages_per_seq,
                                        const int32_t* cache_lens, int32_t num_splits,
                                        fd_tensor* out, float* lse, void* stream);

/*
 * fd_split_plan — the variable-length split planner, on the host (no CUDA call).
 *
 * FlashDecoding page, "Variable-Length序列动态切分策略" (allocator with min_chunk 128 and
 * max_chunk 1024), read for persistent CTAs on one GPU. For W = 8, 4, 2, 1 waves of items,
 * chunk_W = clamp(ceil(sum(len) * Hkv / (W * num_ctas)), 256, 1024) tokens ("性能压测与瓶颈分析":
 * pieces under ~256 tokens lose to launch overhead); the chunk is the chunk_W of least
 * ceil(items_W / num_ctas) * (ceil(chunk_W / 128) + 2), items_W = Hkv * sum_b max(1,
 * ceil(len_b / chunk_W)), ties to the larger W (a work item's fixed cost is taken as two 128-key
 * tiles). Sequence b gets n_b = max(1, ceil(len_b / chunk)) equal splits
 * [floor(s*len_b/n_b), floor((s+1)*len_b/n_b)); items are ordered longest split first
 * (sequences by their longest split, descending, ties by index), then KV head, then split.
 * num_splits > 0 instead fixes n_b = num_splits with ceil(len_b/num_splits)-key splits.
 * key_align = A > 1 puts every split boundary on a multiple of A keys: planner splits cut the
 * ceil(len_b/A) units equally, [min(len_b, A*floor(s*U/n_b)), min(len_b, A*floor((s+1)*U/n_b))),
 * and a fixed count rounds its split size up to a multiple of A; split counts and order do not
 * change. The decode calls build this plan on the device with A = 128 for a paged cache (no key
 * tile crosses a page) and for a contiguous bf16 cache on the tensor-core kernel (groups of
 * 2..16 query heads per KV head: a split then ends on a key-tile boundary), and with A = 1 for a
 * contiguous E4M3 cache and on the CUDA-core kernel (MHA, fp32).
 *
 *  cache_lens_host    [batch] int32 (host); clamped into [0, cache_capacity].
 *  num_ctas           persistent CTAs to plan for (>= 1); fd_decode_num_ctas() gives the count a
 *                     decode call on a device uses.
 *  key_align          >= 1 (see above).
 *  splits_per_seq_host [batch] int32 (host, written) or NULL.
 *  items_host         [items_capacity][5] int32 (host, written) or NULL: per item
 *                     (b, kv_head, split, start, end) in execution order. Items beyond
 *                     items_capacity are not written (info->total_items still reports all).
 *  info               written (required).
 */
fd_status fd_split_plan(const int32_t* cache_lens_host, int32_t batch, int32_t num_kv_heads,
                        int32_t cache_capacity, int32_t num_splits, int32_t num_ctas,
                        int32_t key_align, int32_t* splits_per_seq_host, int32_t* items_host,
                        int32_t items_capacity, fd_plan_info* info);

/*
 * fd_split_plan_device — run the device planner kernel that fd_decode_attention launches, on
 * device lengths, and copy its result out (used to check host and device plans are identical).
 *
 *  cache_lens          [batch] int32 (device).
 *  splits_per_seq_dev  [batch] int32 (device, written).
 *  items_dev           [items_capacity][5] int32 (device, written), same format as fd_split_plan.
 *  total_items_dev     [1] int32 (device, written).
 * Asynchronous on `stream`; uses the library workspace of that stream.
 */
fd_status fd_split_plan_device(const int32_t* cache_lens, int32_t batch, int32_t num_kv_heads,
                               int32_t cache_capacity, int32_t num_splits, int32_t num_ctas,
                               int32_t key_align, int32_t* splits_per_seq_dev, int32_t* items_dev,
                               int32_t items_capacity, int32_t* total_items_dev, void* stream);

/*
 * fd_chunk_prefill_attention — causal attention of packed query chunks against their cached
 * prefix plus themselves (chunked prefill), merged with decode rows in one call.
 *
 * ChunkedPrefill page §2.1: a chunk's K/V are appended to the cache, then its queries attend to
 * the whole cache under a causal mask; Chunked-Prefills page §三.2: the prefix may be a reused
 * cache. Reading: row i of request b sees keys j <= prefix_lens[b] + i (bottom-right aligned).
 * A request with chunk_len == 1 is a decode row and runs through the split-KV decode kernels;
 * longer chunks run through tensor-core tiles of 128 query rows, split along the keys; one
 * combine pass merges every row. Multi-token verification (FlashDecoding page, "与其他推理加速
 * 方案的组合使用", item "Speculative Decoding + FlashDecoding": k speculative tokens checked in
 * one pass) is this call with chunk_lens[b] = k: a request of 2 <= k <= 128 / G rows (G = Hq /
 * Hkv >= 2) runs as head-packed tiles, all G query heads of a KV head in one tile, so its keys
 * are read once per KV head.
 *
 *  q_chunk     [T, Hq, D] with T = sum(chunk_lens), packed request by request; D == 128, bf16.
 *  k_cache,    [B, Hkv, S_cap, D] bf16, holding each request's keys/values at
 *  v_cache     [0, prefix_lens[b] + chunk_lens[b]). Same layout rules as fd_decode_attention.
 *  prefix_lens [B] int32 (device), chunk_lens [B] int32 (device, each >= 0, summing to T).
 *              prefix + chunk is clamped to S_cap on the device (status flag). If the chunk
 *              lengths do not sum to T nothing is computed, `out` / `lse` are left unchanged and
 *              FD_FLAG_LEN_CLAMPED is raised.
 *  out         [T, Hq, D] bf16 (written); lse [T, Hq] float32 (device, written, natural log).
 */
fd_status fd_chunk_prefill_attention(const fd_tensor* q_chunk, const fd_tensor* k_cache,
                                     const fd_tensor* v_cache, const int32_t* prefix_lens,
                                     const int32_t* chunk_lens, fd_tensor* out, float* lse,
                                     void* stream);

/* Size of the device array that holds the scratch of fd_decode_attention_static (64 MiB). */
#define FD_STATIC_SCRATCH_BYTES (64u * 1024u * 1024u)

/*
 * fd_decode_attention_static — fd_decode_attention for callers that cannot allocate device memory.
 *
 * The pages have no counterpart: this is a deployment variant of the same call. Some callers
 * cannot call cudaMalloc when they attend: serving engines that hand nearly all HBM to their own
 * KV-cache pool (a late allocation would fail or fragment it), plugin hosts that only give a
 * plugin buffers they allocated themselves, and latency-critical loops that cannot afford the
 * implicit device synchronisation of cudaMalloc / cudaFree. This entry point takes the same
 * arguments and computes the same result with the same kernels, but keeps its scratch (split plan,
 * work items, per-split partials, merge counters) in one file-scope device array of FD_STATIC_SCRATCH_BYTES and
 * allocates nothing; the caller still passes every input and output.
 *  - Every GPU that loads the library holds that array until the process exits.
 *  - The first call on a device looks up the array's device address (cudaGetSymbolAddress) with
 *    that device current; make that first call before any stream capture begins. The lookup is
 *    repeated when the device's context has changed (after a device reset), so after a reset the
 *    first call must again come before any capture.
 *  - All calls share the array and it keeps the last call's contents: calls that overlap on the GPU
 *    (different streams, or host threads without ordering between their calls) race on it and give
 *    wrong results. Each call clears, on its stream, the header fields that must start at zero
 *    (work cursors), and keeps the status word.
 *  - A shape whose worst-case scratch (fd_decode_workspace_bytes) exceeds FD_STATIC_SCRATCH_BYTES
 *    returns FD_ERR_UNSUPPORTED before anything is enqueued.
 *  - Device status flags these calls raise (FD_FLAG_*) collect in the array's status word until
 *    fd_poll_status, called on the stream the calls used, returns and clears them.
 */
fd_status fd_decode_attention_static(const fd_tensor* q, const fd_tensor* k_cache,
                                     const fd_tensor* v_cache, const int32_t* cache_lens,
                                     int32_t num_splits, fd_tensor* out, float* lse,
                                     void* stream);

/* Human-readable name of a status code (static string). */
const char* fd_status_string(fd_status s);

/* Detail of the last error returned on the calling thread (thread-local, static storage). */
const char* fd_last_error_message(void);

/* Number of persistent CTAs a decode call with this dtype / group size uses on `device`
 * (the num_ctas its planner uses). dtype is the cache's: FD_E4M3 for the *_fp8 calls. Returns
 * 0 on error. */
int32_t fd_decode_num_ctas(int32_t device, int32_t dtype, int32_t group_size, int32_t head_dim);

/* Device workspace bytes a decode call of this shape needs (any cache_lens). */
size_t fd_decode_workspace_bytes(int32_t batch, int32_t num_q_heads, int32_t num_kv_heads,
                                 int32_t cache_capacity, int32_t head_dim, int32_t num_splits,
                                 int32_t num_ctas);

/* Device workspace bytes a chunked-prefill call of this shape needs (any lengths). */
size_t fd_chunk_workspace_bytes(int32_t batch, int32_t total_rows, int32_t num_q_heads,
                                int32_t num_kv_heads, int32_t cache_capacity,
                                int32_t head_dim, int32_t num_ctas);

/* Grow the workspace of (current device, stream) to at least `bytes`, so later calls on that
 * stream allocate nothing (required before CUDA-graph capture). Synchronises `stream`. */
fd_status fd_reserve_workspace(size_t bytes, void* stream);

/* Synchronise `stream`, return the device status word bits (FD_FLAG_*) raised since the last
 * poll on that stream's workspace, together with those raised by fd_decode_attention_static calls
 * on the current device since the last poll, and clear them. */
fd_status fd_poll_status(void* stream, uint32_t* flags);

/* Kernel timing for measurement. fd_profile_begin(n) makes the next n attention calls record a
 * CUDA event before and after each of their kernel launches; fd_profile_end synchronises and
 * writes, per profiled call, the milliseconds of its [planner, decode split kernel, chunk tile
 * kernel, combine] launches into ms[4*i + 0..3] (ms has room for 4*max_calls floats; a segment
 * a call does not launch reads about 0) and the call count into *n_calls. Profiling adds event
 * records between launches, which also keeps them from overlapping; it is off by default. */
fd_status fd_profile_begin(int32_t max_calls);
fd_status fd_profile_end(float* ms, int32_t max_calls, int32_t* n_calls);

/* Free every workspace and profiling resource (all devices). Safe to call more than once. */
void fd_shutdown(void);

#ifdef __cplusplus
}
#endif

#endif /* FD_H_ */
