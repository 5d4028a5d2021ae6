"""CPU checks of the C ABI: the library loads, exports every function include/fd.h declares, its
host planner equals the planner oracle integer for integer, and bad arguments are rejected on
the host before anything touches a GPU. No test here runs a kernel."""

import ctypes
import os
import random
import re

import pytest

import split_kv_decode_flashdecoding_b200 as fd
from oracle import planner as P

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    with open(os.path.join(ROOT, "include", "fd.h")) as f:
        src = f.read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(fd_[a-z_0-9]+)\s*\(", src)))


def test_every_declared_symbol_is_exported_and_bound():
    names = _declared()
    assert "fd_decode_attention" in names and "fd_split_plan" in names
    assert "fd_chunk_prefill_attention" in names
    for n in names:
        assert hasattr(fd.lib, n), f"{n} not exported by libfd.so"
        assert n in fd.ABI_FUNCTIONS, f"{n} has no binding"


def test_status_strings():
    for s, name in enumerate(["FD_OK", "FD_ERR_INVALID_ARGUMENT", "FD_ERR_UNSUPPORTED",
                              "FD_ERR_CUDA", "FD_ERR_WORKSPACE"]):
        assert fd.fd_status_string(s) == name
    assert fd.fd_status_string(99) == "FD_UNKNOWN_STATUS"


@pytest.mark.parametrize("seed", range(60))
def test_host_plan_equals_oracle(seed):
    rng = random.Random(1000 + seed)
    B = rng.choice([1, 2, 3, 5, 32, 64, 200])
    hkv = rng.choice([1, 2, 8, 40])
    cap = rng.choice([1, 16, 63, 64, 65, 257, 1024, 16384, 32768])
    ctas = rng.choice([1, 7, 148, 296])
    fixed = rng.choice([0, 0, 0, 1, 4, 9])
    lens = [rng.choice([0, 1, cap - 1, cap, cap + 5, -2, rng.randint(0, cap)]) for _ in range(B)]
    align = rng.choice([1, 1, 128, 16])
    info, splits, items = fd.fd_split_plan(lens, hkv, cap, fixed, ctas, key_align=align)
    ref = P.decode_plan(lens, hkv, cap, ctas, fixed, align=align)
    assert info["chunk_tokens"] == ref.chunk_tokens
    assert splits == ref.splits_per_seq
    assert info["total_items"] == ref.total_items
    assert info["max_splits_per_seq"] == ref.max_splits_per_seq
    assert [tuple(x) for x in items] == ref.items


def test_host_plan_workload_shapes():
    from workloads import uniform_lens
    lens = uniform_lens(1103, 32, 1024, 32768)
    info, splits, items = fd.fd_split_plan(lens, 8, 32768, 0, 148)
    ref = P.decode_plan(lens, 8, 32768, 148, 0)
    assert info["chunk_tokens"] == 1024 == ref.chunk_tokens
    assert [tuple(x) for x in items] == ref.items
    assert info["total_items"] <= P.MAX_CHUNK * 0 + 8 * 32 + max(8 * 148, 8 * 32 * 32)


def test_plan_rejects_bad_arguments():
    info = fd.FdPlanInfo()
    lens = (ctypes.c_int32 * 2)(5, 6)
    assert fd.lib.fd_split_plan(lens, -1, 1, 8, 0, 1, 1, None, None, 0, ctypes.byref(info)) == 1
    assert fd.lib.fd_split_plan(lens, 2, 0, 8, 0, 1, 1, None, None, 0, ctypes.byref(info)) == 1
    assert fd.lib.fd_split_plan(lens, 2, 1, 8, -1, 1, 1, None, None, 0, ctypes.byref(info)) == 1
    assert fd.lib.fd_split_plan(lens, 2, 1, 8, 0, 0, 1, None, None, 0, ctypes.byref(info)) == 1
    assert fd.lib.fd_split_plan(None, 2, 1, 8, 0, 1, 1, None, None, 0, ctypes.byref(info)) == 1
    assert fd.lib.fd_split_plan(lens, 2, 1, 8, 0, 1, 0, None, None, 0, ctypes.byref(info)) == 1
    assert fd.lib.fd_split_plan(lens, 2, 1, 8, 0, 1, 1, None, None, 0, None) == 1
    assert "info" in fd.lib.fd_last_error_message().decode()


def _fake(shape, dtype=fd.FD_BF16, strides=None, ptr=0x100000):
    t = fd.FdTensor()
    t.data = ptr
    t.dtype = dtype
    t.ndim = len(shape)
    if strides is None:
        strides, s = [], 1
        for n in reversed(shape):
            strides.insert(0, s)
            s *= n
    for i, (n, st) in enumerate(zip(shape, strides)):
        t.shape[i] = n
        t.stride[i] = st
    return t


def _decode(q, k, v, out, lens=0x200000, lse=0x300000, splits=0):
    lp = ctypes.cast(ctypes.c_void_p(lens), ctypes.POINTER(ctypes.c_int32)) if lens else None
    sp = ctypes.cast(ctypes.c_void_p(lse), ctypes.POINTER(ctypes.c_float)) if lse else None
    return fd.lib.fd_decode_attention(ctypes.byref(q) if q else None, ctypes.byref(k),
                                      ctypes.byref(v), lp, splits,
                                      ctypes.byref(out) if out else None, sp, None)


def test_decode_rejects_bad_arguments_on_host():
    B, Hq, Hkv, S, D = 2, 8, 2, 64, 128
    q, o = _fake([B, Hq, D]), _fake([B, Hq, D])
    k, v = _fake([B, Hkv, S, D]), _fake([B, Hkv, S, D])
    assert _decode(None, k, v, o) == fd.FD_ERR_INVALID_ARGUMENT
    assert _decode(q, k, v, None) == fd.FD_ERR_INVALID_ARGUMENT
    assert _decode(q, k, v, o, lens=0) == fd.FD_ERR_INVALID_ARGUMENT
    assert _decode(q, k, v, o, lse=0) == fd.FD_ERR_INVALID_ARGUMENT
    assert _decode(q, k, v, o, splits=-1) == fd.FD_ERR_INVALID_ARGUMENT
    # Hq not a multiple of Hkv
    q3, o3 = _fake([B, 6, D]), _fake([B, 6, D])
    k4, v4 = _fake([B, 4, S, D]), _fake([B, 4, S, D])
    assert _decode(q3, k4, v4, o3) == fd.FD_ERR_INVALID_ARGUMENT
    # head_dim 96 unsupported
    q96, o96 = _fake([B, Hq, 96]), _fake([B, Hq, 96])
    k96, v96 = _fake([B, Hkv, S, 96]), _fake([B, Hkv, S, 96])
    assert _decode(q96, k96, v96, o96) == fd.FD_ERR_UNSUPPORTED
    # mismatched dtype, mismatched strides, non-contiguous token rows
    assert _decode(q, _fake([B, Hkv, S, D], fd.FD_F32), _fake([B, Hkv, S, D], fd.FD_F32), o) == 1
    kt = _fake([B, Hkv, S, D], strides=[Hkv * S * D, S * D, D, 1])
    vt = _fake([B, Hkv, S, D], strides=[Hkv * S * D * 2, S * D, D, 1])
    assert _decode(q, kt, vt, o) == fd.FD_ERR_UNSUPPORTED
    kr = _fake([B, Hkv, S, D], strides=[Hkv * S * 2 * D, S * 2 * D, 2 * D, 1])
    assert _decode(q, kr, kr, o) == fd.FD_ERR_UNSUPPORTED
    # last dim not contiguous
    qs = _fake([B, Hq, D], strides=[Hq * D * 2, D * 2, 2])
    assert _decode(qs, k, v, o) == fd.FD_ERR_UNSUPPORTED
    # unaligned data pointer
    assert _decode(_fake([B, Hq, D], ptr=0x100002), k, v, o) == fd.FD_ERR_UNSUPPORTED
    # unknown dtype
    assert _decode(_fake([B, Hq, D], dtype=7), k, v, o) == fd.FD_ERR_UNSUPPORTED
    # out shape differs
    assert _decode(q, k, v, _fake([B, Hq + 1, D])) == fd.FD_ERR_INVALID_ARGUMENT
    # group size above 16 is unsupported
    q32, o32 = _fake([B, 32, D]), _fake([B, 32, D])
    k1, v1 = _fake([B, 1, S, D]), _fake([B, 1, S, D])
    assert _decode(q32, k1, v1, o32) == fd.FD_ERR_UNSUPPORTED
    # batch 0 is a no-op, before any device work
    q0, o0 = _fake([0, Hq, D]), _fake([0, Hq, D])
    k0, v0 = _fake([0, Hkv, S, D]), _fake([0, Hkv, S, D])
    assert _decode(q0, k0, v0, o0) == fd.FD_OK


def test_workspace_bound_covers_plan():
    for B, hkv, cap, fixed, ctas in [(32, 8, 32768, 0, 148), (1, 8, 32768, 0, 148),
                                     (4, 40, 16384, 0, 296), (1, 8, 1024, 4, 296),
                                     (3, 2, 100, 0, 1)]:
        ws = fd.fd_decode_workspace_bytes(B, hkv * 8, hkv, cap, 128, fixed, ctas)
        assert ws > 0
        for lens in ([cap] * B, [0] * B, [1] * B, [cap // 3 + 1] * B):
            ref = P.decode_plan(lens, hkv, cap, ctas, fixed)
            # every item's slot and the item list fit the sizes the workspace was laid out for
            items_bound = (hkv * B * fixed if fixed else
                           hkv * B + max(P.WAVES * ctas, -(-hkv * B * cap // P.MAX_CHUNK)))
            assert ref.total_items <= items_bound


def _decode_fp8(q, k, v, out, ks=1.0, vs=1.0, lens=0x200000, lse=0x300000, splits=0):
    lp = ctypes.cast(ctypes.c_void_p(lens), ctypes.POINTER(ctypes.c_int32)) if lens else None
    sp = ctypes.cast(ctypes.c_void_p(lse), ctypes.POINTER(ctypes.c_float)) if lse else None
    return fd.lib.fd_decode_attention_fp8(ctypes.byref(q), ctypes.byref(k), ctypes.byref(v), ks, vs,
                                          lp, splits, ctypes.byref(out), sp, None)


def test_fp8_decode_rejects_bad_arguments_on_host():
    B, Hq, Hkv, S, D = 2, 8, 1, 64, 128
    q, o = _fake([B, Hq, D]), _fake([B, Hq, D])
    k, v = _fake([B, Hkv, S, D], fd.FD_E4M3), _fake([B, Hkv, S, D], fd.FD_E4M3)
    for ks, vs in ((0.0, 1.0), (1.0, -2.0), (float("inf"), 1.0), (1.0, float("nan"))):
        assert _decode_fp8(q, k, v, o, ks, vs) == fd.FD_ERR_INVALID_ARGUMENT, (ks, vs)
    # bf16 caches through the FP8 call, and E4M3 caches through the bf16 call
    kb, vb = _fake([B, Hkv, S, D]), _fake([B, Hkv, S, D])
    assert _decode_fp8(q, kb, vb, o) == fd.FD_ERR_INVALID_ARGUMENT
    assert _decode(q, k, v, o) == fd.FD_ERR_INVALID_ARGUMENT
    # E4M3 is a cache dtype only; fp32 q is not served with an FP8 cache
    assert _decode_fp8(_fake([B, Hq, D], fd.FD_E4M3), k, v, _fake([B, Hq, D], fd.FD_E4M3)) == \
        fd.FD_ERR_UNSUPPORTED
    assert _decode_fp8(_fake([B, Hq, D], fd.FD_F32), k, v, _fake([B, Hq, D], fd.FD_F32)) == \
        fd.FD_ERR_UNSUPPORTED
    # head_dim 64 and groups above 8 are not served with an FP8 cache
    assert _decode_fp8(_fake([B, Hq, 64]), _fake([B, Hkv, S, 64], fd.FD_E4M3),
                       _fake([B, Hkv, S, 64], fd.FD_E4M3), _fake([B, Hq, 64])) == fd.FD_ERR_UNSUPPORTED
    assert _decode_fp8(_fake([B, 16, D]), k, v, _fake([B, 16, D])) == fd.FD_ERR_UNSUPPORTED
    # a row stride of the codes that is not a multiple of 16 bytes
    kr = _fake([B, Hkv, S, D], fd.FD_E4M3, strides=[Hkv * S * D + 8, S * D, D, 1])
    assert _decode_fp8(q, kr, kr, o) == fd.FD_ERR_UNSUPPORTED
    # batch 0 is a no-op
    q0, o0 = _fake([0, Hq, D]), _fake([0, Hq, D])
    k0, v0 = _fake([0, Hkv, S, D], fd.FD_E4M3), _fake([0, Hkv, S, D], fd.FD_E4M3)
    assert _decode_fp8(q0, k0, v0, o0) == fd.FD_OK


def _paged_fp8(q, kp, vp, ks=1.0, vs=1.0, table=0x400000, pps=4, lens=0x200000, lse=0x300000):
    tp = ctypes.cast(ctypes.c_void_p(table), ctypes.POINTER(ctypes.c_int32)) if table else None
    lp = ctypes.cast(ctypes.c_void_p(lens), ctypes.POINTER(ctypes.c_int32)) if lens else None
    sp = ctypes.cast(ctypes.c_void_p(lse), ctypes.POINTER(ctypes.c_float)) if lse else None
    out = _fake([q.shape[0], q.shape[1], q.shape[2]])
    return fd.lib.fd_decode_attention_paged_fp8(ctypes.byref(q), ctypes.byref(kp), ctypes.byref(vp),
                                                ks, vs, tp, pps, lp, 0, ctypes.byref(out), sp, None)


def test_fp8_paged_rejects_bad_arguments_on_host():
    B, Hq, Hkv, P, D = 2, 16, 2, 16, 128
    q = _fake([B, Hq, D])
    kp, vp = _fake([8, Hkv, P, D], fd.FD_E4M3), _fake([8, Hkv, P, D], fd.FD_E4M3)
    assert _paged_fp8(q, kp, vp, ks=-1.0) == fd.FD_ERR_INVALID_ARGUMENT
    assert _paged_fp8(q, kp, vp, table=0) == fd.FD_ERR_INVALID_ARGUMENT
    assert _paged_fp8(q, kp, vp, pps=0) == fd.FD_ERR_INVALID_ARGUMENT
    # bf16 pages through the FP8 call
    assert _paged_fp8(q, _fake([8, Hkv, P, D]), _fake([8, Hkv, P, D])) == fd.FD_ERR_INVALID_ARGUMENT
    # page size 48 is not a divisor or multiple of the 128-key tile
    k48, v48 = _fake([8, Hkv, 48, D], fd.FD_E4M3), _fake([8, Hkv, 48, D], fd.FD_E4M3)
    assert _paged_fp8(q, k48, v48) == fd.FD_ERR_UNSUPPORTED
    # a page stride that is not a multiple of 16 bytes
    kr = _fake([8, Hkv, P, D], fd.FD_E4M3, strides=[Hkv * P * D + 8, P * D, D, 1])
    assert _paged_fp8(q, kr, kr) == fd.FD_ERR_UNSUPPORTED
    # groups above 8 are not served with an FP8 cache
    q16 = _fake([B, 16, D])
    k1, v1 = _fake([8, 1, P, D], fd.FD_E4M3), _fake([8, 1, P, D], fd.FD_E4M3)
    assert _paged_fp8(q16, k1, v1) == fd.FD_ERR_UNSUPPORTED
    assert "group size" in fd.lib.fd_last_error_message().decode()


def _chunk(q, k, v, out, prefix=0x200000, chunk=0x200100, lse=0x300000):
    ip = lambda a: ctypes.cast(ctypes.c_void_p(a), ctypes.POINTER(ctypes.c_int32)) if a else None
    sp = ctypes.cast(ctypes.c_void_p(lse), ctypes.POINTER(ctypes.c_float)) if lse else None
    return fd.lib.fd_chunk_prefill_attention(ctypes.byref(q), ctypes.byref(k), ctypes.byref(v),
                                             ip(prefix), ip(chunk), ctypes.byref(out), sp, None)


def test_chunk_rejects_bad_arguments_on_host():
    B, T, S = 2, 5, 64
    # head_dim 96 and fp32 are unsupported; head_dim 64 with a group above 8 too (its decode rows
    # would need the CUDA-core kernel, which serves groups up to 8)
    for D, hq, hkv, dt in [(96, 8, 2, fd.FD_BF16), (128, 8, 2, fd.FD_F32), (64, 32, 2, fd.FD_BF16)]:
        q, o = _fake([T, hq, D], dt), _fake([T, hq, D], dt)
        k, v = _fake([B, hkv, S, D], dt), _fake([B, hkv, S, D], dt)
        assert _chunk(q, k, v, o) == fd.FD_ERR_UNSUPPORTED, (D, hq, hkv, dt)
    # missing lengths or lse
    q, o = _fake([T, 8, 64]), _fake([T, 8, 64])
    k, v = _fake([B, 2, S, 64]), _fake([B, 2, S, 64])
    assert _chunk(q, k, v, o, prefix=0) == fd.FD_ERR_INVALID_ARGUMENT
    assert _chunk(q, k, v, o, lse=0) == fd.FD_ERR_INVALID_ARGUMENT
