"""Python binding of the split-KV FlashDecoding C ABI (include/fd.h).

Argument marshalling only: every step of the attention path runs in the CUDA kernels of
libfd.so. PyTorch supplies device memory and streams. Importing this package fails loudly when
libfd.so has not been built (``python split_kv_decode_flashdecoding_b200/build.py``); there is no
CPU fallback.

Functions keep the C names:

* ``fd_decode_attention(q, k_cache, v_cache, cache_lens, num_splits=0, out=None, lse=None)``
* ``fd_chunk_prefill_attention(q_chunk, k_cache, v_cache, prefix_lens, chunk_lens, out=None, lse=None)``
* ``fd_split_plan(cache_lens, num_kv_heads, cache_capacity, num_splits=0, num_ctas=148)``
* ``fd_split_plan_device(cache_lens, num_kv_heads, cache_capacity, num_splits=0, num_ctas=148)``
* status, workspace and profiling helpers.
"""

from __future__ import annotations

import ctypes
import os
from typing import List, Optional, Sequence, Tuple

import torch

__all__ = [
    "FdError", "LIB_PATH", "lib", "fd_decode_attention", "fd_decode_attention_paged",
    "fd_decode_attention_static", "fd_decode_attention_fp8", "fd_decode_attention_paged_fp8",
    "fd_chunk_prefill_attention",
    "fd_split_plan", "fd_split_plan_device", "fd_decode_num_ctas", "fd_decode_workspace_bytes",
    "fd_chunk_workspace_bytes", "fd_reserve_workspace", "fd_poll_status", "fd_profile_begin",
    "fd_profile_end", "fd_shutdown", "fd_status_string", "FD_F32", "FD_BF16", "FD_E4M3",
    "FD_FLAG_LEN_CLAMPED", "FD_FLAG_WAIT_TIMEOUT", "FD_FLAG_PLAN_OVERFLOW", "FD_FLAG_BAD_PAGE",
    "ABI_FUNCTIONS",
]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libfd.so")

FD_OK, FD_ERR_INVALID_ARGUMENT, FD_ERR_UNSUPPORTED, FD_ERR_CUDA, FD_ERR_WORKSPACE = range(5)
FD_F32, FD_BF16, FD_E4M3 = 0, 1, 2
FD_FLAG_LEN_CLAMPED = 0x1
FD_FLAG_WAIT_TIMEOUT = 0x2
FD_FLAG_PLAN_OVERFLOW = 0x4
FD_FLAG_BAD_PAGE = 0x8

c_i32, c_i64, c_size, c_vp, c_f32p = (ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t,
                                      ctypes.c_void_p, ctypes.POINTER(ctypes.c_float))
c_i32p = ctypes.POINTER(ctypes.c_int32)


class FdTensor(ctypes.Structure):
    _fields_ = [("data", c_vp), ("dtype", c_i32), ("ndim", c_i32),
                ("shape", c_i64 * 4), ("stride", c_i64 * 4)]


class FdPlanInfo(ctypes.Structure):
    _fields_ = [("chunk_tokens", c_i32), ("total_items", c_i32), ("max_splits_per_seq", c_i32),
                ("num_ctas", c_i32), ("workspace_bytes", c_size)]


class FdError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(message)
        self.status = status


if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python split_kv_decode_flashdecoding_b200/build.py`"
        " (there is no fallback implementation)")

lib = ctypes.CDLL(LIB_PATH)

_TP = ctypes.POINTER(FdTensor)
# name -> (restype, argtypes); the same names as include/fd.h
ABI_FUNCTIONS = {
    "fd_decode_attention": (c_i32, [_TP, _TP, _TP, c_i32p, c_i32, _TP, c_f32p, c_vp]),
    "fd_decode_attention_static": (c_i32, [_TP, _TP, _TP, c_i32p, c_i32, _TP, c_f32p, c_vp]),
    "fd_split_plan": (c_i32, [c_i32p, c_i32, c_i32, c_i32, c_i32, c_i32, c_i32, c_i32p, c_i32p,
                              c_i32, ctypes.POINTER(FdPlanInfo)]),
    "fd_split_plan_device": (c_i32, [c_i32p, c_i32, c_i32, c_i32, c_i32, c_i32, c_i32, c_i32p,
                                     c_i32p, c_i32, c_i32p, c_vp]),
    "fd_chunk_prefill_attention": (c_i32, [_TP, _TP, _TP, c_i32p, c_i32p, _TP, c_f32p, c_vp]),
    "fd_decode_attention_paged": (c_i32, [_TP, _TP, _TP, c_i32p, c_i32, c_i32p, c_i32, _TP, c_f32p,
                                          c_vp]),
    "fd_decode_attention_fp8": (c_i32, [_TP, _TP, _TP, ctypes.c_float, ctypes.c_float, c_i32p,
                                        c_i32, _TP, c_f32p, c_vp]),
    "fd_decode_attention_paged_fp8": (c_i32, [_TP, _TP, _TP, ctypes.c_float, ctypes.c_float,
                                              c_i32p, c_i32, c_i32p, c_i32, _TP, c_f32p, c_vp]),
    "fd_status_string": (ctypes.c_char_p, [c_i32]),
    "fd_last_error_message": (ctypes.c_char_p, []),
    "fd_decode_num_ctas": (c_i32, [c_i32, c_i32, c_i32, c_i32]),
    "fd_decode_workspace_bytes": (c_size, [c_i32, c_i32, c_i32, c_i32, c_i32, c_i32, c_i32]),
    "fd_chunk_workspace_bytes": (c_size, [c_i32, c_i32, c_i32, c_i32, c_i32, c_i32, c_i32]),
    "fd_reserve_workspace": (c_i32, [c_size, c_vp]),
    "fd_poll_status": (c_i32, [c_vp, ctypes.POINTER(ctypes.c_uint32)]),
    "fd_profile_begin": (c_i32, [c_i32]),
    "fd_profile_end": (c_i32, [c_f32p, c_i32, c_i32p]),
    "fd_shutdown": (None, []),
}
for _name, (_res, _args) in ABI_FUNCTIONS.items():
    _f = getattr(lib, _name)
    _f.restype = _res
    _f.argtypes = _args


def fd_status_string(status: int) -> str:
    return lib.fd_status_string(status).decode()


def _check(status: int, what: str) -> None:
    if status != FD_OK:
        raise FdError(status, f"{what}: {fd_status_string(status)}: "
                              f"{lib.fd_last_error_message().decode()}")


# an E4M3 cache may be passed as torch.float8_e4m3fn or as its uint8 codes
_DTYPES = {torch.float32: FD_F32, torch.bfloat16: FD_BF16, torch.float8_e4m3fn: FD_E4M3,
           torch.uint8: FD_E4M3}


def _tensor(t: torch.Tensor) -> FdTensor:
    n = t.dim()
    if n > 4:
        raise ValueError("at most 4 dimensions")
    ft = FdTensor(t.data_ptr() if t.numel() > 0 else None, _DTYPES.get(t.dtype, -1), n)
    ft.shape[:n] = t.shape
    ft.stride[:n] = t.stride()
    return ft


def _ptr(t: Optional[torch.Tensor], ctype):
    if t is None:
        return None
    return ctypes.cast(ctypes.c_void_p(t.data_ptr()), ctypes.POINTER(ctype))


def _stream(stream, device) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream(device)
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def fd_decode_attention(q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
                        cache_lens: torch.Tensor, num_splits: int = 0,
                        out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
                        stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """Split-KV decode attention. q [B,Hq,D]; caches [B,Hkv,S_cap,D]; cache_lens int32 [B].

    Returns (out [B,Hq,D] in q's dtype, lse float32 [B,Hq], natural log). Asynchronous on
    ``stream`` (default: the current stream of q's device)."""
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty(q.shape[:2], dtype=torch.float32, device=q.device)
    with torch.cuda.device(q.device):
        st = lib.fd_decode_attention(ctypes.byref(_tensor(q)), ctypes.byref(_tensor(k_cache)),
                                     ctypes.byref(_tensor(v_cache)), _ptr(cache_lens, c_i32),
                                     int(num_splits), ctypes.byref(_tensor(out)),
                                     _ptr(lse, ctypes.c_float), _stream(stream, q.device))
    _check(st, "fd_decode_attention")
    return out, lse


def fd_decode_attention_paged(q: torch.Tensor, k_pages: torch.Tensor, v_pages: torch.Tensor,
                              block_table: torch.Tensor, cache_lens: torch.Tensor,
                              num_splits: int = 0, out: Optional[torch.Tensor] = None,
                              lse: Optional[torch.Tensor] = None,
                              stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """Split-KV decode attention over a paged cache. k_pages / v_pages [num_pages, Hkv,
    page_size, D]; block_table int32 [B, pages_per_seq] (contiguous rows); token t of sequence b
    is row t % page_size of page block_table[b, t // page_size]."""
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty(q.shape[:2], dtype=torch.float32, device=q.device)
    if block_table.dim() != 2 or block_table.stride(1) != 1 or block_table.stride(0) != block_table.shape[1]:
        raise ValueError("block_table must be a contiguous [B, pages_per_seq] int32 tensor")
    with torch.cuda.device(q.device):
        st = lib.fd_decode_attention_paged(
            ctypes.byref(_tensor(q)), ctypes.byref(_tensor(k_pages)),
            ctypes.byref(_tensor(v_pages)), _ptr(block_table, c_i32), int(block_table.shape[1]),
            _ptr(cache_lens, c_i32), int(num_splits), ctypes.byref(_tensor(out)),
            _ptr(lse, ctypes.c_float), _stream(stream, q.device))
    _check(st, "fd_decode_attention_paged")
    return out, lse


def fd_decode_attention_fp8(q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
                            k_scale: float, v_scale: float, cache_lens: torch.Tensor,
                            num_splits: int = 0, out: Optional[torch.Tensor] = None,
                            lse: Optional[torch.Tensor] = None,
                            stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """Decode attention over an E4M3 cache (torch.float8_e4m3fn or uint8 codes, [B,Hkv,S_cap,D]);
    the cached value of code c is e4m3(c) * scale. q / out bf16."""
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty(q.shape[:2], dtype=torch.float32, device=q.device)
    with torch.cuda.device(q.device):
        st = lib.fd_decode_attention_fp8(
            ctypes.byref(_tensor(q)), ctypes.byref(_tensor(k_cache)), ctypes.byref(_tensor(v_cache)),
            float(k_scale), float(v_scale), _ptr(cache_lens, c_i32), int(num_splits),
            ctypes.byref(_tensor(out)), _ptr(lse, ctypes.c_float), _stream(stream, q.device))
    _check(st, "fd_decode_attention_fp8")
    return out, lse


def fd_decode_attention_paged_fp8(q: torch.Tensor, k_pages: torch.Tensor, v_pages: torch.Tensor,
                                  k_scale: float, v_scale: float, block_table: torch.Tensor,
                                  cache_lens: torch.Tensor, num_splits: int = 0,
                                  out: Optional[torch.Tensor] = None,
                                  lse: Optional[torch.Tensor] = None,
                                  stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """fd_decode_attention_paged over E4M3 pages, with the scales of fd_decode_attention_fp8."""
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty(q.shape[:2], dtype=torch.float32, device=q.device)
    if block_table.dim() != 2 or block_table.stride(1) != 1 or block_table.stride(0) != block_table.shape[1]:
        raise ValueError("block_table must be a contiguous [B, pages_per_seq] int32 tensor")
    with torch.cuda.device(q.device):
        st = lib.fd_decode_attention_paged_fp8(
            ctypes.byref(_tensor(q)), ctypes.byref(_tensor(k_pages)), ctypes.byref(_tensor(v_pages)),
            float(k_scale), float(v_scale), _ptr(block_table, c_i32), int(block_table.shape[1]),
            _ptr(cache_lens, c_i32), int(num_splits), ctypes.byref(_tensor(out)),
            _ptr(lse, ctypes.c_float), _stream(stream, q.device))
    _check(st, "fd_decode_attention_paged_fp8")
    return out, lse


def fd_decode_attention_static(q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
                               cache_lens: torch.Tensor, num_splits: int, out: torch.Tensor,
                               lse: torch.Tensor, stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """Same as fd_decode_attention, for callers that cannot allocate device memory: the library
    keeps this call's scratch in a fixed device array (FD_STATIC_SCRATCH_BYTES) and allocates
    nothing, so `out` and `lse` must be passed in. Calls that overlap on the GPU share that array
    and race; the first call on a device should come before any stream capture."""
    with torch.cuda.device(q.device):
        st = lib.fd_decode_attention_static(
            ctypes.byref(_tensor(q)), ctypes.byref(_tensor(k_cache)), ctypes.byref(_tensor(v_cache)),
            _ptr(cache_lens, c_i32), int(num_splits), ctypes.byref(_tensor(out)),
            _ptr(lse, ctypes.c_float), _stream(stream, q.device))
    _check(st, "fd_decode_attention_static")
    return out, lse


def fd_chunk_prefill_attention(q_chunk: torch.Tensor, k_cache: torch.Tensor,
                               v_cache: torch.Tensor, prefix_lens: torch.Tensor,
                               chunk_lens: torch.Tensor, out: Optional[torch.Tensor] = None,
                               lse: Optional[torch.Tensor] = None,
                               stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """Causal attention of packed query chunks [T,Hq,D] against their cached prefix + self.
    chunk_lens[b] = 1 is a decode row; chunk_lens[b] = k speculative tokens is a verification
    step (head-packed tiles when 2 <= k <= 128 / (Hq / Hkv))."""
    if out is None:
        out = torch.empty_like(q_chunk)
    if lse is None:
        lse = torch.empty(q_chunk.shape[:2], dtype=torch.float32, device=q_chunk.device)
    with torch.cuda.device(q_chunk.device):
        st = lib.fd_chunk_prefill_attention(
            ctypes.byref(_tensor(q_chunk)), ctypes.byref(_tensor(k_cache)),
            ctypes.byref(_tensor(v_cache)), _ptr(prefix_lens, c_i32), _ptr(chunk_lens, c_i32),
            ctypes.byref(_tensor(out)), _ptr(lse, ctypes.c_float),
            _stream(stream, q_chunk.device))
    _check(st, "fd_chunk_prefill_attention")
    return out, lse


def fd_split_plan(cache_lens: Sequence[int], num_kv_heads: int, cache_capacity: int,
                  num_splits: int = 0, num_ctas: int = 148, with_items: bool = True,
                  key_align: int = 1):
    """Host planner. Returns (info dict, splits per sequence, items [(b,h,split,start,end)])."""
    B = len(cache_lens)
    lens = (c_i32 * max(1, B))(*[int(x) for x in cache_lens])
    splits = (c_i32 * max(1, B))()
    info = FdPlanInfo()
    _check(lib.fd_split_plan(lens, B, num_kv_heads, cache_capacity, num_splits, num_ctas,
                             key_align, splits, None, 0, ctypes.byref(info)), "fd_split_plan")
    items: List[Tuple[int, int, int, int, int]] = []
    if with_items and info.total_items > 0:
        buf = (c_i32 * (5 * info.total_items))()
        _check(lib.fd_split_plan(lens, B, num_kv_heads, cache_capacity, num_splits, num_ctas,
                                 key_align, splits, buf, info.total_items, ctypes.byref(info)),
               "fd_split_plan")
        items = [tuple(buf[5 * i:5 * i + 5]) for i in range(info.total_items)]
    d = {f: getattr(info, f) for f, _ in FdPlanInfo._fields_}
    return d, [splits[i] for i in range(B)], items


def fd_split_plan_device(cache_lens: torch.Tensor, num_kv_heads: int, cache_capacity: int,
                         num_splits: int = 0, num_ctas: int = 148, items_capacity: int = 0,
                         stream=None, key_align: int = 1):
    """Run the device planner on device lengths. Returns (total_items, splits, items) tensors."""
    dev = cache_lens.device
    B = cache_lens.numel()
    splits = torch.zeros(max(1, B), dtype=torch.int32, device=dev)
    total = torch.zeros(1, dtype=torch.int32, device=dev)
    items = torch.zeros((max(1, items_capacity), 5), dtype=torch.int32, device=dev)
    with torch.cuda.device(dev):
        st = lib.fd_split_plan_device(_ptr(cache_lens, c_i32), B, num_kv_heads, cache_capacity,
                                      num_splits, num_ctas, key_align, _ptr(splits, c_i32),
                                      _ptr(items, c_i32) if items_capacity > 0 else None,
                                      items_capacity, _ptr(total, c_i32), _stream(stream, dev))
    _check(st, "fd_split_plan_device")
    return total, splits[:B], items[:items_capacity]


def fd_decode_num_ctas(device: int, dtype: torch.dtype, group_size: int, head_dim: int) -> int:
    return int(lib.fd_decode_num_ctas(device, _DTYPES[dtype], group_size, head_dim))


def fd_decode_workspace_bytes(batch, num_q_heads, num_kv_heads, cache_capacity, head_dim,
                              num_splits, num_ctas) -> int:
    return int(lib.fd_decode_workspace_bytes(batch, num_q_heads, num_kv_heads, cache_capacity,
                                             head_dim, num_splits, num_ctas))


def fd_chunk_workspace_bytes(batch, total_rows, num_q_heads, num_kv_heads, cache_capacity,
                             head_dim, num_ctas) -> int:
    return int(lib.fd_chunk_workspace_bytes(batch, total_rows, num_q_heads, num_kv_heads,
                                            cache_capacity, head_dim, num_ctas))


def fd_reserve_workspace(nbytes: int, stream=None, device=None) -> None:
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else device
    with torch.cuda.device(dev):
        _check(lib.fd_reserve_workspace(int(nbytes), _stream(stream, dev)), "fd_reserve_workspace")


def fd_poll_status(stream=None, device=None) -> int:
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else device
    flags = ctypes.c_uint32(0)
    with torch.cuda.device(dev):
        _check(lib.fd_poll_status(_stream(stream, dev), ctypes.byref(flags)), "fd_poll_status")
    return int(flags.value)


def fd_profile_begin(max_calls: int) -> None:
    _check(lib.fd_profile_begin(int(max_calls)), "fd_profile_begin")


def fd_profile_end(max_calls: int) -> List[Tuple[float, float, float, float]]:
    """Per profiled call: (planner ms, decode split ms, chunk tile ms, combine ms)."""
    ms = (ctypes.c_float * (4 * max_calls))()
    n = c_i32(0)
    _check(lib.fd_profile_end(ms, int(max_calls), ctypes.byref(n)), "fd_profile_end")
    return [tuple(ms[4 * i + j] for j in range(4)) for i in range(n.value)]


def fd_shutdown() -> None:
    lib.fd_shutdown()
