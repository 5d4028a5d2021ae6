"""GPU parity of the E4M3-cache calls (fd_decode_attention_fp8, fd_decode_attention_paged_fp8)
against the float64 oracle, through the C ABI.

The oracle dequantizes the same codes (e4m3(c) * scale) and applies the plain definition. Rows
past each sequence's length hold NaN codes, so a read past the end poisons the result. Two cases
check the expansion of the codes itself: a one-hot key makes the output one V row, which must
then equal every code's value exactly, and keys made only of subnormal codes make the scores
depend on those codes alone.
"""

import numpy as np
import pytest
import torch

from oracle import attention as oracle
from parity import check_lse, check_out
from workloads import make_decode_inputs, make_fp8, make_paged, to_numpy_exact, workload

pytestmark = pytest.mark.gpu

NAN = float("nan")


def _fd():
    import split_kv_decode_flashdecoding_b200 as fd
    return fd


def _dev():
    return torch.device("cuda", 0)


def _run(q, kc, vc, ks, vs, lens, num_splits=0):
    fd = _fd()
    dev = _dev()
    q = q.to(dev)
    B, Hq, D = q.shape
    big = torch.full((B + 2, Hq, D), 12345.0, dtype=q.dtype, device=dev)
    out = big[1:B + 1]
    lse = torch.empty((B, Hq), dtype=torch.float32, device=dev)
    fd.fd_decode_attention_fp8(q, kc.to(dev), vc.to(dev), ks, vs, lens.to(dev), num_splits,
                               out=out, lse=lse)
    torch.cuda.synchronize()
    assert bool((big[0] == 12345.0).all()) and bool((big[B + 1] == 12345.0).all()), "guard band"
    return out, lse


def _oracle(q, kc, vc, ks, vs, lens, rows=None):
    return oracle.decode_attention_fp8(to_numpy_exact(q), kc.numpy(), vc.numpy(), ks, vs,
                                       [int(x) for x in lens], rows=rows)


CASES = [
    # (B, Hq, Hkv, lens, cap)
    (4, 64, 8, [300, 1, 0, 129], 320),          # G = 8 (the 70B shape), ragged tiles
    (3, 32, 8, [1000, 128, 257], 1024),          # G = 4
    (3, 16, 8, [700, 5, 33], 704),               # G = 2
    (2, 8, 8, [1500, 129], 1536),                # MHA (G = 1)
    (1, 8, 1, [5000], 5120),                     # one KV head, long
    (2, 8, 2, [100, 37], 100),                   # capacity below one 128-key tile
]


@pytest.mark.parametrize("case", range(len(CASES)))
@pytest.mark.parametrize("num_splits", [0, 3])
def test_fp8_small(case, num_splits):
    B, hq, hkv, lens, cap = CASES[case]
    inp = make_decode_inputs(B, hq, hkv, 128, cap, lens, torch.bfloat16, seed=600 + case,
                             pad_fill=NAN)
    f8 = make_fp8(inp.k_cache, inp.v_cache)
    out, lse = _run(inp.q, f8.k_codes, f8.v_codes, f8.k_scale, f8.v_scale, inp.cache_lens,
                    num_splits)
    ro, rl = _oracle(inp.q, f8.k_codes, f8.v_codes, f8.k_scale, f8.v_scale, inp.cache_lens)
    check_out(out, ro, "fp8 out")
    check_lse(lse, rl, "fp8 lse")
    assert _fd().fd_poll_status() == 0


def test_fp8_every_value_code_expands_exactly():
    # key 37 holds code 0x7E (448) everywhere, the others 0: with q = 1 its weight is 1 to fp32
    # precision, so O = v_scale * V[37]; sequence b's row 37 holds codes 128 b .. 128 b + 127
    # (the NaN codes replaced by 0), every value exactly representable in bf16
    B, hq, hkv, S, D = 2, 8, 1, 200, 128
    kc = torch.zeros((B, hkv, S, D), dtype=torch.uint8)
    kc[:, :, 37] = 0x7E
    vc = torch.randint(0, 0x7E, (B, hkv, S, D), dtype=torch.uint8,
                       generator=torch.Generator().manual_seed(7))
    codes = torch.arange(256, dtype=torch.int32)
    codes[(codes == 0x7F) | (codes == 0xFF)] = 0
    for b in range(B):
        vc[b, :, 37] = codes[128 * b:128 * (b + 1)].to(torch.uint8)
    q = torch.ones((B, hq, D), dtype=torch.bfloat16)
    lens = torch.tensor([S, S], dtype=torch.int32)
    for vs in (1.0, 0.5):
        out, lse = _run(q, kc, vc, 1.0, vs, lens)
        ro, rl = _oracle(q, kc, vc, 1.0, vs, lens)
        assert np.array_equal(out.float().cpu().numpy(), ro.astype(np.float32)), "V codes"
        check_lse(lse, rl, "one-hot lse")


def test_fp8_subnormal_key_codes():
    # keys made of the subnormal codes (+-1..7 x 2^-9) and zeros only, a large q: the scores are
    # spread by several units, so flushing a subnormal (or misplacing its bits) changes them
    B, hq, hkv, S, D = 2, 16, 2, 300, 128
    g = torch.Generator().manual_seed(11)
    mag = torch.randint(0, 8, (B, hkv, S, D), dtype=torch.uint8, generator=g)
    sign = torch.randint(0, 2, (B, hkv, S, D), dtype=torch.uint8, generator=g) << 7
    kc = mag | sign
    vc = torch.randint(0, 0x7E, (B, hkv, S, D), dtype=torch.uint8, generator=g)
    q = (torch.randn((B, hq, D), generator=g) * 1024.0).to(torch.bfloat16)
    lens = torch.tensor([S, 123], dtype=torch.int32)
    out, lse = _run(q, kc, vc, 1.0, 0.25, lens)
    ro, rl = _oracle(q, kc, vc, 1.0, 0.25, lens)
    # the scores really depend on the subnormal codes: their spread is several units
    assert float(np.ptp(rl)) > 0.5
    check_out(out, ro, "subnormal keys out")
    check_lse(lse, rl, "subnormal keys lse")


def test_fp8_equals_bf16_call_on_exact_values():
    # a bf16 cache holding exactly e4m3(c) * 2^k gives (to rounding) the bf16 call's result
    fd = _fd()
    dev = _dev()
    inp = make_decode_inputs(3, 64, 8, 128, 2048, [2048, 77, 1500], torch.bfloat16, seed=620)
    f8 = make_fp8(inp.k_cache, inp.v_cache, k_scale=0.0078125, v_scale=0.00390625)
    kb = torch.from_numpy(oracle.dequant_e4m3(f8.k_codes.numpy(), f8.k_scale)).to(torch.bfloat16)
    vb = torch.from_numpy(oracle.dequant_e4m3(f8.v_codes.numpy(), f8.v_scale)).to(torch.bfloat16)
    o1, l1 = _run(inp.q, f8.k_codes, f8.v_codes, f8.k_scale, f8.v_scale, inp.cache_lens)
    o2, l2 = fd.fd_decode_attention(inp.q.to(dev), kb.to(dev), vb.to(dev), inp.cache_lens.to(dev))
    torch.cuda.synchronize()
    check_out(o1, o2.float().cpu().numpy().astype(np.float64), "fp8 vs bf16 call")
    check_lse(l1, l2.cpu().numpy().astype(np.float64), "fp8 vs bf16 call lse")


def test_fp8_accepts_float8_tensors():
    fd = _fd()
    inp = make_decode_inputs(2, 16, 2, 128, 256, [256, 40], torch.bfloat16, seed=630)
    f8 = make_fp8(inp.k_cache, inp.v_cache)
    o1, l1 = _run(inp.q, f8.k_codes, f8.v_codes, f8.k_scale, f8.v_scale, inp.cache_lens)
    o2, l2 = _run(inp.q, f8.k_codes.view(torch.float8_e4m3fn), f8.v_codes.view(torch.float8_e4m3fn),
                  f8.k_scale, f8.v_scale, inp.cache_lens)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
    assert fd.fd_poll_status() == 0


PAGED = [
    # (B, Hq, Hkv, page_size, lens, cap)
    (4, 64, 8, 16, [300, 1, 0, 129], 320),
    (2, 64, 8, 8, [77, 200], 200),               # 8-key pages: 16 boxes per key tile
    (3, 64, 8, 128, [1000, 128, 257], 1024),
    (2, 32, 4, 256, [2000, 255], 2048),
    (2, 8, 8, 64, [513, 64], 576),
]


@pytest.mark.parametrize("case", range(len(PAGED)))
def test_fp8_paged(case):
    fd = _fd()
    dev = _dev()
    B, hq, hkv, psz, lens, cap = PAGED[case]
    inp = make_decode_inputs(B, hq, hkv, 128, cap, lens, torch.bfloat16, seed=640 + case,
                             pad_fill=NAN)
    f8 = make_fp8(inp.k_cache, inp.v_cache)
    # the pages of the codes, at shuffled positions; unused pages hold the NaN code
    pk = make_paged(f8.k_codes.view(torch.float8_e4m3fn).float(), f8.v_codes.view(torch.float8_e4m3fn).float(),
                    lens, psz, seed=650 + case)
    kp = pk.k_pages.to(torch.float8_e4m3fn).view(torch.uint8)
    vp = pk.v_pages.to(torch.float8_e4m3fn).view(torch.uint8)
    q = inp.q.to(dev)
    out = torch.empty_like(q)
    lse = torch.empty((B, hq), dtype=torch.float32, device=dev)
    fd.fd_decode_attention_paged_fp8(q, kp.to(dev), vp.to(dev), f8.k_scale, f8.v_scale,
                                     pk.block_table.to(dev), inp.cache_lens.to(dev), out=out, lse=lse)
    torch.cuda.synchronize()
    ro, rl = _oracle(inp.q, f8.k_codes, f8.v_codes, f8.k_scale, f8.v_scale, inp.cache_lens)
    check_out(out, ro, "paged fp8 out")
    check_lse(lse, rl, "paged fp8 lse")
    assert fd.fd_poll_status() == 0


def test_fp8_rejections_on_device():
    fd = _fd()
    dev = _dev()
    q = torch.zeros((1, 8, 64), dtype=torch.bfloat16, device=dev)
    kc = torch.zeros((1, 8, 16, 64), dtype=torch.uint8, device=dev)
    lens = torch.tensor([10], dtype=torch.int32, device=dev)
    with pytest.raises(fd.FdError):          # head_dim 64
        fd.fd_decode_attention_fp8(q, kc, kc, 1.0, 1.0, lens)
    q = torch.zeros((1, 16, 128), dtype=torch.bfloat16, device=dev)
    kc = torch.zeros((1, 1, 16, 128), dtype=torch.uint8, device=dev)
    with pytest.raises(fd.FdError):          # group of 16
        fd.fd_decode_attention_fp8(q, kc, kc, 1.0, 1.0, lens)
    with pytest.raises(fd.FdError):          # zero scale
        fd.fd_decode_attention_fp8(q[:, :8], kc, kc, 0.0, 1.0, lens)


def test_fp8_workload_3():
    # the default decode workload quantized to E4M3, in the bench's launch configuration: every
    # output element against the oracle
    inp = workload(3)
    f8 = make_fp8(inp.k_cache, inp.v_cache)
    del inp.k_cache, inp.v_cache
    out, lse = _run(inp.q, f8.k_codes, f8.v_codes, f8.k_scale, f8.v_scale, inp.cache_lens)
    ro, rl = _oracle(inp.q, f8.k_codes, f8.v_codes, f8.k_scale, f8.v_scale, inp.cache_lens)
    check_out(out, ro, "fp8 w3 out")
    check_lse(lse, rl, "fp8 w3 lse")


@pytest.mark.parametrize("B", [256, 300])
def test_fp8_planner_kernel_batch(B):
    # 256 sequences: the largest batch the split kernel plans itself; above 256 the planner
    # kernel plans the call instead
    rng = np.random.default_rng(660)
    lens = [int(x) for x in rng.integers(0, 400, size=B)]
    inp = make_decode_inputs(B, 16, 2, 128, 400, lens, torch.bfloat16, seed=661, pad_fill=NAN)
    f8 = make_fp8(inp.k_cache, inp.v_cache)
    out, lse = _run(inp.q, f8.k_codes, f8.v_codes, f8.k_scale, f8.v_scale, inp.cache_lens)
    ro, rl = _oracle(inp.q, f8.k_codes, f8.v_codes, f8.k_scale, f8.v_scale, inp.cache_lens)
    check_out(out, ro, f"fp8 B {B} out")
    check_lse(lse, rl, f"fp8 B {B} lse")


def test_fp8_cuda_graph_replay_new_lengths():
    fd = _fd()
    dev = _dev()
    base = make_decode_inputs(3, 64, 8, 128, 2048, [2048] * 3, torch.bfloat16, seed=670)
    f8 = make_fp8(base.k_cache, base.v_cache)
    q, k, v = base.q.to(dev), f8.k_codes.to(dev), f8.v_codes.to(dev)
    lens = base.cache_lens.to(dev)
    out = torch.empty_like(q)
    lse = torch.empty(q.shape[:2], dtype=torch.float32, device=dev)
    s = torch.cuda.Stream()
    nct = fd.fd_decode_num_ctas(0, torch.uint8, 8, 128)
    fd.fd_reserve_workspace(fd.fd_decode_workspace_bytes(3, 64, 8, 2048, 128, 0, nct), stream=s)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        fd.fd_decode_attention_fp8(q, k, v, f8.k_scale, f8.v_scale, lens, 0, out=out, lse=lse,
                                   stream=s)
    for new in ([2048, 100, 1500], [7, 2000, 1]):
        # codes past the new lengths must not be read: poison them with the NaN code
        kk = f8.k_codes.clone()
        vv = f8.v_codes.clone()
        for b, n in enumerate(new):
            kk[b, :, n:] = 0x7F
            vv[b, :, n:] = 0x7F
        k.copy_(kk)
        v.copy_(vv)
        lens.copy_(torch.tensor(new, dtype=torch.int32))
        g.replay()
        torch.cuda.synchronize()
        ro, rl = _oracle(base.q, kk, vv, f8.k_scale, f8.v_scale, torch.tensor(new))
        check_out(out, ro, "fp8 graph out")
        check_lse(lse, rl, "fp8 graph lse")
    del g
