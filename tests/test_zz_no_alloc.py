"""The allocation-free decode entry point against the regular one, through the C ABI.

fd_decode_attention_static exists for callers that cannot allocate device memory when they
attend (engines whose KV-cache pool owns nearly all HBM, plugin hosts that only hand out their own
buffers, loops that cannot take cudaMalloc's implicit synchronisation). It keeps its scratch in a
fixed device array instead of the library's workspace. This file is collected last so a run that
stops at the first failure has already run every other test; it also passes alone in a fresh
process, where its first call is also the first use of the device array.
"""

import ctypes

import pytest
import torch

from parity import check_lse, check_out, to_f64
from workloads import make_decode_inputs

pytestmark = pytest.mark.gpu

NAN = float("nan")


def _c_call(fd, name, q, k, v, lens, num_splits, out, lse):
    """Call an fd_decode_attention-shaped C entry point directly through ctypes."""
    f = getattr(fd.lib, name)
    st = f(ctypes.byref(fd._tensor(q)), ctypes.byref(fd._tensor(k)), ctypes.byref(fd._tensor(v)),
           ctypes.cast(ctypes.c_void_p(lens.data_ptr()), ctypes.POINTER(ctypes.c_int32)),
           int(num_splits), ctypes.byref(fd._tensor(out)),
           ctypes.cast(ctypes.c_void_p(lse.data_ptr()), ctypes.POINTER(ctypes.c_float)),
           ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    return st


def test_static_scratch_matches_regular_entry_point_twice_in_a_row():
    import split_kv_decode_flashdecoding_b200 as fd
    dev = torch.device("cuda", 0)
    cases = [
        # GQA on the tensor-core kernel, ragged lengths, planner splits
        dict(args=(4, 64, 8, 128, 4096, [4096, 17, 2500, 1000], torch.bfloat16), seed=501, ns=0),
        # MHA on the CUDA-core kernel with fixed splits: a different plan reuses the same array
        dict(args=(3, 8, 8, 128, 3000, [3000, 1, 129], torch.bfloat16), seed=502, ns=5),
    ]
    for c in cases:
        inp = make_decode_inputs(*c["args"], seed=c["seed"], pad_fill=NAN)
        q, k, v = inp.q.to(dev), inp.k_cache.to(dev), inp.v_cache.to(dev)
        lens = inp.cache_lens.to(dev)
        B, hq, d = q.shape
        ref_o = torch.empty_like(q)
        ref_l = torch.empty((B, hq), dtype=torch.float32, device=dev)
        st_o = torch.full_like(q, 7.0)
        st_l = torch.full((B, hq), 7.0, dtype=torch.float32, device=dev)
        assert _c_call(fd, "fd_decode_attention", q, k, v, lens, c["ns"], ref_o, ref_l) == fd.FD_OK
        assert _c_call(fd, "fd_decode_attention_static", q, k, v, lens, c["ns"], st_o, st_l) == fd.FD_OK
        torch.cuda.synchronize()
        check_out(st_o, to_f64(ref_o), "static-scratch out")
        check_lse(st_l, to_f64(ref_l), "static-scratch lse")


def test_static_scratch_rejects_oversized_shapes():
    import split_kv_decode_flashdecoding_b200 as fd
    dev = torch.device("cuda", 0)
    # 64 sequences x 8 KV heads x 65536 keys of capacity: the worst-case partials exceed the array
    B, hq, hkv, cap, d = 64, 64, 8, 65536, 128
    q = torch.zeros((B, hq, d), dtype=torch.bfloat16, device=dev)
    k = torch.zeros((1, hkv, 1, d), dtype=torch.bfloat16, device=dev).expand(B, hkv, cap, d)
    lens = torch.ones(B, dtype=torch.int32, device=dev)
    out = torch.empty_like(q)
    lse = torch.empty((B, hq), dtype=torch.float32, device=dev)
    need = fd.fd_decode_workspace_bytes(B, hq, hkv, cap, d, 0, fd.fd_decode_num_ctas(0, torch.bfloat16, 8, d))
    assert need > 64 * 1024 * 1024
    kt = fd._tensor(k)
    for i, st in enumerate((hkv * cap * d, cap * d, d, 1)):   # a valid layout; never read
        kt.stride[i] = st
    kt.data = k.data_ptr()
    st = fd.lib.fd_decode_attention_static(
        ctypes.byref(fd._tensor(q)), ctypes.byref(kt), ctypes.byref(kt),
        ctypes.cast(ctypes.c_void_p(lens.data_ptr()), ctypes.POINTER(ctypes.c_int32)), 0,
        ctypes.byref(fd._tensor(out)),
        ctypes.cast(ctypes.c_void_p(lse.data_ptr()), ctypes.POINTER(ctypes.c_float)), None)
    assert st == fd.FD_ERR_UNSUPPORTED
    assert "static scratch" in fd.lib.fd_last_error_message().decode()
