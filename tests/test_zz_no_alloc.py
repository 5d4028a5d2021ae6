"""The allocation-free decode entry point against the regular one, through the C ABI.

fd_decode_attention_static exists for callers that cannot allocate device memory when they
attend (engines whose KV-cache pool owns nearly all HBM, plugin hosts that only hand out their own
buffers, loops that cannot take cudaMalloc's implicit synchronisation). It keeps its scratch in a
fixed device array instead of the library's workspace. Every case below runs twice in a row on
one stream, so the second call reuses the array exactly as the first left it. This file is
collected last so a run that stops at the first failure has already run every other test; it
also passes alone in a fresh process, where its first call is also the first use of the array.
"""

import ctypes

import pytest
import torch

from oracle import attention as oracle
from parity import check_lse, check_out, to_f64
from workloads import make_decode_inputs, to_numpy_exact, workload

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


CASES = [
    # GQA on the tensor-core kernel (it plans the call itself), ragged lengths, planner splits
    dict(args=(4, 64, 8, 128, 4096, [4096, 17, 2500, 1000], torch.bfloat16), seed=501, ns=0),
    # MHA on the CUDA-core kernel with fixed splits: a different plan reuses the same array
    dict(args=(3, 8, 8, 128, 3000, [3000, 1, 129], torch.bfloat16), seed=502, ns=5),
    # the fp32 decode shape of the benchmarks (MHA, D 64, 4 fixed splits, in-kernel merge)
    dict(args=(1, 8, 8, 64, 1024, [1024], torch.float32), seed=503, ns=4),
    # the tensor-core kernel again, above 256 sequences (the planner kernel plans it)
    dict(args=(300, 16, 2, 128, 256, [(37 * i) % 257 for i in range(300)], torch.bfloat16),
         seed=504, ns=0),
]


def _inputs(c):
    dev = torch.device("cuda", 0)
    inp = make_decode_inputs(*c["args"], seed=c["seed"], pad_fill=NAN)
    return inp, inp.q.to(dev), inp.k_cache.to(dev), inp.v_cache.to(dev), inp.cache_lens.to(dev)


@pytest.mark.parametrize("case", range(len(CASES)))
def test_static_scratch_matches_regular_entry_point_twice_in_a_row(case):
    import split_kv_decode_flashdecoding_b200 as fd
    c = CASES[case]
    inp, q, k, v, lens = _inputs(c)
    B, hq, d = q.shape
    ref_o = torch.empty_like(q)
    ref_l = torch.empty((B, hq), dtype=torch.float32, device=q.device)
    assert _c_call(fd, "fd_decode_attention", q, k, v, lens, c["ns"], ref_o, ref_l) == fd.FD_OK
    outs = []
    for _ in range(2):
        st_o = torch.full_like(q, 7.0)
        st_l = torch.full((B, hq), 7.0, dtype=torch.float32, device=q.device)
        assert _c_call(fd, "fd_decode_attention_static", q, k, v, lens, c["ns"], st_o, st_l) == fd.FD_OK
        outs.append((st_o, st_l))
    torch.cuda.synchronize()
    assert fd.fd_poll_status() == 0
    for i, (st_o, st_l) in enumerate(outs):
        check_out(st_o, to_f64(ref_o), f"static call {i} vs regular out")
        check_lse(st_l, to_f64(ref_l), f"static call {i} vs regular lse")
    # the same results as the regular call, and the oracle's
    ro, rl = oracle.decode_attention(to_numpy_exact(inp.q), to_numpy_exact(inp.k_cache),
                                     to_numpy_exact(inp.v_cache), inp.cache_lens.tolist())
    check_out(outs[1][0], ro, "static call vs oracle out")
    check_lse(outs[1][1], rl, "static call vs oracle lse")


def test_static_scratch_after_a_clamped_call():
    # a call whose lengths are clamped raises FD_FLAG_LEN_CLAMPED in the array's status word,
    # which fd_poll_status reports and clears; the calls after it are unaffected
    import split_kv_decode_flashdecoding_b200 as fd
    c = CASES[0]
    inp, q, k, v, lens = _inputs(c)
    B, hq, d = q.shape
    cap = k.shape[2]
    fd.fd_poll_status()
    ref_o = torch.empty_like(q)
    ref_l = torch.empty((B, hq), dtype=torch.float32, device=q.device)
    assert _c_call(fd, "fd_decode_attention", q, k, v, lens, 0, ref_o, ref_l) == fd.FD_OK
    bad = torch.tensor([cap + 100, -3, 2500, 1000], dtype=torch.int32, device=q.device)
    o = torch.empty_like(q)
    l = torch.empty((B, hq), dtype=torch.float32, device=q.device)
    # (the clamped rows read only keys below the capacity: row 0 all of them, row 1 none)
    assert _c_call(fd, "fd_decode_attention_static", q, k, v, bad, 0, o, l) == fd.FD_OK
    flags = fd.fd_poll_status()
    assert flags & fd.FD_FLAG_LEN_CLAMPED, hex(flags)
    assert flags & fd.FD_FLAG_WAIT_TIMEOUT == 0, hex(flags)
    assert fd.fd_poll_status() == 0, "polling clears the flags"
    assert bool((o[1].float() == 0).all()) and bool(torch.isneginf(l[1]).all())
    for _ in range(2):
        o2 = torch.full_like(q, 7.0)
        l2 = torch.full((B, hq), 7.0, dtype=torch.float32, device=q.device)
        assert _c_call(fd, "fd_decode_attention_static", q, k, v, lens, 0, o2, l2) == fd.FD_OK
        torch.cuda.synchronize()
        check_out(o2, to_f64(ref_o), "static call after a clamped call out")
        check_lse(l2, to_f64(ref_l), "static call after a clamped call lse")
    assert fd.fd_poll_status() == 0


def test_static_scratch_full_workload_3():
    # the 70B-like decode workload at full size fits the array (its worst case is about 35 MB)
    import split_kv_decode_flashdecoding_b200 as fd
    inp = workload(3)
    dev = torch.device("cuda", 0)
    q, k, v, lens = inp.q.to(dev), inp.k_cache.to(dev), inp.v_cache.to(dev), inp.cache_lens.to(dev)
    ref_o = torch.empty_like(q)
    ref_l = torch.empty(q.shape[:2], dtype=torch.float32, device=dev)
    st_o = torch.empty_like(q)
    st_l = torch.empty(q.shape[:2], dtype=torch.float32, device=dev)
    assert _c_call(fd, "fd_decode_attention", q, k, v, lens, 0, ref_o, ref_l) == fd.FD_OK
    assert _c_call(fd, "fd_decode_attention_static", q, k, v, lens, 0, st_o, st_l) == fd.FD_OK
    torch.cuda.synchronize()
    assert fd.fd_poll_status() == 0
    assert torch.equal(st_o, ref_o) and torch.equal(st_l, ref_l), "same kernels, same plan"


def test_static_scratch_rejects_oversized_shapes():
    import split_kv_decode_flashdecoding_b200 as fd
    dev = torch.device("cuda", 0)
    # 64 sequences x 8 KV heads x 65536 keys of capacity: the worst-case partials exceed the array.
    # The tensors only describe that layout over a small allocation and every length is 0, so no
    # kernel could form a cache address even if the host-side check were missing.
    B, hq, hkv, cap, d = 64, 64, 8, 65536, 128
    q = torch.zeros((B, hq, d), dtype=torch.bfloat16, device=dev)
    k = torch.zeros((1, hkv, 1, d), dtype=torch.bfloat16, device=dev).expand(B, hkv, cap, d)
    lens = torch.zeros(B, dtype=torch.int32, device=dev)
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
