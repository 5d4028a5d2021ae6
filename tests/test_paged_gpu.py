"""GPU parity of fd_decode_attention_paged against the float64 oracle, through the C ABI.

The pages of every case sit at shuffled physical positions; unused page slots hold NaN and
unused block-table entries -1, so reading a wrong page or a row past a sequence's end poisons
the result. The oracle is the contiguous definition over the same keys (equal to the paged oracle
by its pins).
"""

import numpy as np
import pytest
import torch

from oracle import attention as oracle
from oracle import planner as oplan
from parity import check_lse, check_out
from workloads import make_decode_inputs, make_paged, to_numpy_exact, workload

pytestmark = pytest.mark.gpu

NAN = float("nan")


def _fd():
    import split_kv_decode_flashdecoding_b200 as fd
    return fd


def _run_paged(inp, pg, num_splits=0):
    fd = _fd()
    dev = torch.device("cuda", 0)
    q = inp.q.to(dev)
    B, Hq, D = q.shape
    big = torch.full((B + 2, Hq, D), 12345.0, dtype=q.dtype, device=dev)
    out = big[1:B + 1]
    lse = torch.empty((B, Hq), dtype=torch.float32, device=dev)
    fd.fd_decode_attention_paged(q, pg.k_pages.to(dev), pg.v_pages.to(dev),
                                 pg.block_table.to(dev), inp.cache_lens.to(dev), num_splits,
                                 out=out, lse=lse)
    torch.cuda.synchronize()
    assert bool((big[0] == 12345.0).all()) and bool((big[B + 1] == 12345.0).all()), "guard band"
    return out, lse


def _oracle(inp, rows=None):
    return oracle.decode_attention(to_numpy_exact(inp.q), to_numpy_exact(inp.k_cache),
                                   to_numpy_exact(inp.v_cache), inp.cache_lens.tolist(), rows=rows)


CASES = [
    # (dtype, B, Hq, Hkv, D, page_size, lens, cap)
    (torch.bfloat16, 4, 64, 8, 128, 16, [300, 1, 0, 129], 320),      # G = 8, tensor cores
    (torch.bfloat16, 3, 64, 8, 128, 128, [1000, 128, 257], 1024),    # page = one key tile
    (torch.bfloat16, 2, 32, 4, 128, 256, [2000, 255], 2048),         # page = two key tiles
    (torch.bfloat16, 3, 16, 4, 128, 64, [513, 64, 65], 640),         # G = 4
    (torch.bfloat16, 2, 32, 2, 128, 8, [77, 200], 200),              # G = 16, tiny pages
    (torch.bfloat16, 3, 8, 8, 128, 16, [700, 5, 33], 704),           # MHA, CUDA cores (tile 64)
    (torch.bfloat16, 2, 8, 8, 128, 128, [1500, 129], 1536),          # MHA, page >= tile
    (torch.bfloat16, 2, 6, 3, 64, 32, [257, 128], 288),              # D = 64 (tile 128)
    (torch.float32, 2, 8, 8, 64, 8, [300, 17], 304),                 # fp32 (tile 64)
    (torch.float32, 2, 8, 2, 128, 64, [400, 64], 448),               # fp32, G = 4 (tile 32)
]


@pytest.mark.parametrize("case", range(len(CASES)))
@pytest.mark.parametrize("num_splits", [0, 3])
def test_paged_small(case, num_splits):
    dt, B, hq, hkv, d, psz, lens, cap = CASES[case]
    inp = make_decode_inputs(B, hq, hkv, d, cap, lens, dt, seed=400 + case, pad_fill=NAN)
    pg = make_paged(inp.k_cache, inp.v_cache, lens, psz, seed=500 + case)
    out, lse = _run_paged(inp, pg, num_splits)
    ro, rl = _oracle(inp)
    check_out(out, ro, "paged out")
    check_lse(lse, rl, "paged lse")
    assert _fd().fd_poll_status() == 0


@pytest.mark.parametrize("B", [256, 300])
def test_paged_planner_kernel_batch(B):
    # 256 sequences: the largest batch the split kernel plans itself; above, the planner kernel
    # plans the call; aligned splits in both
    rng = np.random.default_rng(77)
    lens = [int(x) for x in rng.integers(0, 400, size=B)]
    inp = make_decode_inputs(B, 16, 2, 128, 400, lens, torch.bfloat16, seed=78, pad_fill=NAN)
    pg = make_paged(inp.k_cache, inp.v_cache, lens, 16, seed=79)
    out, lse = _run_paged(inp, pg)
    ro, rl = _oracle(inp)
    check_out(out, ro, f"paged B {B} out")
    check_lse(lse, rl, f"paged B {B} lse")


def test_paged_device_plan_is_aligned_oracle_plan():
    fd = _fd()
    dev = torch.device("cuda", 0)
    lens = [5000, 1, 0, 130, 2047, 4096]
    for fixed in (0, 3):
        info, splits, items = fd.fd_split_plan(lens, 8, 8192, fixed, 148, key_align=128)
        ref = oplan.decode_plan(lens, 8, 8192, 148, fixed, align=128)
        assert [tuple(x) for x in items] == ref.items
        total, dsplits, ditems = fd.fd_split_plan_device(
            torch.tensor(lens, dtype=torch.int32, device=dev), 8, 8192, fixed, 148,
            items_capacity=len(ref.items), key_align=128)
        torch.cuda.synchronize()
        assert int(total.item()) == len(ref.items)
        assert [tuple(x) for x in ditems.cpu().tolist()] == ref.items


def test_paged_equals_contiguous_call():
    # the same keys through both entry points agree to rounding (their splits differ)
    fd = _fd()
    dev = torch.device("cuda", 0)
    inp = make_decode_inputs(4, 64, 8, 128, 3000, [3000, 1, 2048, 999], torch.bfloat16, seed=90)
    pg = make_paged(inp.k_cache, inp.v_cache, inp.cache_lens.tolist(), 32, seed=91)
    o1, l1 = _run_paged(inp, pg)
    o2, l2 = fd.fd_decode_attention(inp.q.to(dev), inp.k_cache.to(dev), inp.v_cache.to(dev),
                                    inp.cache_lens.to(dev))
    torch.cuda.synchronize()
    ref = o2.float().cpu().numpy().astype(np.float64)
    check_out(o1, ref, "paged vs contiguous")
    check_lse(l1, l2.cpu().numpy().astype(np.float64), "paged vs contiguous lse")


@pytest.mark.parametrize("dtype,hq,hkv", [(torch.bfloat16, 64, 8), (torch.bfloat16, 8, 8)])
def test_paged_bad_page_flag(dtype, hq, hkv):
    # a used page outside the pool is never dereferenced: the call completes and raises the flag
    fd = _fd()
    inp = make_decode_inputs(2, hq, hkv, 128, 512, [512, 100], dtype, seed=95)
    pg = make_paged(inp.k_cache, inp.v_cache, [512, 100], 64, seed=96)
    npages = pg.k_pages.shape[0]
    pg.block_table[0, 2] = npages + 5
    pg.block_table[1, 0] = -7
    fd.fd_poll_status()
    out, lse = _run_paged(inp, pg)
    flags = fd.fd_poll_status()
    assert flags & fd.FD_FLAG_BAD_PAGE
    assert flags & fd.FD_FLAG_WAIT_TIMEOUT == 0


def test_paged_length_clamp():
    fd = _fd()
    inp = make_decode_inputs(2, 16, 2, 128, 256, [256, 40], torch.bfloat16, seed=97)
    pg = make_paged(inp.k_cache, inp.v_cache, [256, 40], 128, seed=98)
    good_o, good_l = _run_paged(inp, pg)
    fd.fd_poll_status()
    inp.cache_lens = torch.tensor([256 + 500, 40], dtype=torch.int32)  # beyond the table's pages
    out, lse = _run_paged(inp, pg)
    assert fd.fd_poll_status() & fd.FD_FLAG_LEN_CLAMPED
    assert torch.equal(out, good_o) and torch.equal(lse, good_l)


def test_paged_rejects_bad_layouts():
    fd = _fd()
    dev = torch.device("cuda", 0)
    q = torch.zeros((1, 8, 128), dtype=torch.bfloat16, device=dev)
    lens = torch.tensor([10], dtype=torch.int32, device=dev)
    table = torch.zeros((1, 4), dtype=torch.int32, device=dev)
    kp = torch.zeros((4, 8, 48, 128), dtype=torch.bfloat16, device=dev)  # page size 48
    with pytest.raises(fd.FdError):
        fd.fd_decode_attention_paged(q, kp, kp, table, lens)
    kp = torch.zeros((4, 8, 16, 64), dtype=torch.bfloat16, device=dev)   # head_dim mismatch
    with pytest.raises(fd.FdError):
        fd.fd_decode_attention_paged(q, kp, kp, table, lens)


@pytest.mark.parametrize("layout", ["head_major", "kv_pool"])
@pytest.mark.parametrize("psz", [8, 16, 32, 64])
def test_paged_pool_layouts(layout, psz):
    # pools that are not [pages, Hkv, page_size, D] contiguous:
    # - head_major: stored [Hkv, pages, page_size, D] (a page's KV heads are not consecutive, so
    #   the tensor-core kernel copies each half of a page separately);
    # - kv_pool: K and V of a page side by side in one [pages, 2, Hkv, page_size, D] pool (a page
    #   stride twice the page's bytes; the heads are consecutive, so a page is one copy).
    fd = _fd()
    dev = torch.device("cuda", 0)
    lens = [700, 1, 129, 0, 383]
    inp = make_decode_inputs(5, 64, 8, 128, 768, lens, torch.bfloat16, seed=610 + psz, pad_fill=NAN)
    pg = make_paged(inp.k_cache, inp.v_cache, lens, psz, seed=620 + psz)
    if layout == "head_major":
        kp = pg.k_pages.permute(1, 0, 2, 3).contiguous().to(dev).permute(1, 0, 2, 3)
        vp = pg.v_pages.permute(1, 0, 2, 3).contiguous().to(dev).permute(1, 0, 2, 3)
        assert kp.stride(1) != psz * 128
    else:
        pool = torch.stack([pg.k_pages, pg.v_pages], dim=1).to(dev)
        kp, vp = pool[:, 0], pool[:, 1]
        assert kp.stride(0) == 2 * kp.shape[1] * psz * 128 and kp.stride(1) == psz * 128
    q = inp.q.to(dev)
    out = torch.empty_like(q)
    lse = torch.empty((5, 64), dtype=torch.float32, device=dev)
    fd.fd_decode_attention_paged(q, kp, vp, pg.block_table.to(dev), inp.cache_lens.to(dev),
                                 out=out, lse=lse)
    torch.cuda.synchronize()
    ro, rl = _oracle(inp)
    check_out(out, ro, f"paged {layout} {psz} out")
    check_lse(lse, rl, f"paged {layout} {psz} lse")
    assert fd.fd_poll_status() == 0


@pytest.mark.parametrize("psz", [128, 16])
def test_paged_workload_3(psz):
    # the default workload's keys in 128- or 16-key pages at shuffled positions: every output
    # element
    inp = workload(3)
    pg = make_paged(inp.k_cache, inp.v_cache, inp.cache_lens.tolist(), psz, seed=1303)
    out, lse = _run_paged(inp, pg)
    ro, rl = _oracle(inp)
    check_out(out, ro, f"paged w3 (pages of {psz}) out")
    check_lse(lse, rl, f"paged w3 (pages of {psz}) lse")
