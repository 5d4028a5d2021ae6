"""GPU parity of fd_decode_attention against the float64 oracle, through the C ABI.

Caches are padded with NaN past every sequence end so a read beyond cache_lens poisons the
result; outputs sit inside guard bands that must stay untouched.
"""

import math

import numpy as np
import pytest
import torch

from oracle import attention as oracle
from oracle import planner as oplan
from parity import check_lse, check_out
from workloads import make_decode_inputs, to_numpy_exact, workload

pytestmark = pytest.mark.gpu

NAN = float("nan")


def _fd():
    import split_kv_decode_flashdecoding_b200 as fd
    return fd


def _run(inp, num_splits=None, guard=True, stream=None):
    fd = _fd()
    dev = torch.device("cuda", 0)
    q = inp.q.to(dev)
    k = inp.k_cache.to(dev)
    v = inp.v_cache.to(dev)
    lens = inp.cache_lens.to(dev)
    B, Hq, D = q.shape
    if guard:
        big = torch.full((B + 2, Hq, D), 12345.0, dtype=q.dtype, device=dev)
        out = big[1:B + 1]
        lbig = torch.full((B * Hq + 64,), 777.0, dtype=torch.float32, device=dev)
        lse = lbig[32:32 + B * Hq].view(B, Hq)
    else:
        out = torch.empty_like(q)
        lse = torch.empty((B, Hq), dtype=torch.float32, device=dev)
    ns = inp.num_splits if num_splits is None else num_splits
    fd.fd_decode_attention(q, k, v, lens, ns, out=out, lse=lse, stream=stream)
    torch.cuda.synchronize()
    if guard:
        assert bool((big[0] == 12345.0).all()) and bool((big[B + 1] == 12345.0).all()), "out guard band"
        assert bool((lbig[:32] == 777.0).all()) and bool((lbig[32 + B * Hq:] == 777.0).all()), "lse guard band"
    assert fd.fd_poll_status() & fd.FD_FLAG_WAIT_TIMEOUT == 0
    return out, lse


def _oracle(inp, rows=None):
    return oracle.decode_attention(to_numpy_exact(inp.q), to_numpy_exact(inp.k_cache),
                                   to_numpy_exact(inp.v_cache), inp.cache_lens.tolist(), rows=rows)


SMALL = [
    # (dtype, B, Hq, Hkv, D, lens, cap)
    (torch.float32, 2, 4, 4, 64, [65, 1], 96),
    (torch.float32, 3, 8, 4, 128, [257, 0, 64], 300),
    (torch.float32, 1, 8, 1, 64, [1000], 1000),
    (torch.bfloat16, 2, 4, 4, 128, [129, 63], 200),
    (torch.bfloat16, 3, 6, 3, 64, [2, 257, 128], 257),
    (torch.bfloat16, 2, 16, 8, 128, [1, 300], 320),      # G = 2, tensor cores
    (torch.bfloat16, 3, 16, 4, 128, [127, 128, 129], 256),  # G = 4
    (torch.bfloat16, 2, 64, 8, 128, [1000, 65], 1024),   # G = 8
    (torch.bfloat16, 2, 32, 2, 128, [777, 16], 800),     # G = 16
    (torch.bfloat16, 1, 8, 1, 128, [64], 64),            # G = 8, capacity below one tile
]


@pytest.mark.parametrize("case", range(len(SMALL)))
@pytest.mark.parametrize("num_splits", [0, 1, 3, 8])
def test_small_shapes(case, num_splits):
    dt, B, Hq, Hkv, D, lens, cap = SMALL[case]
    inp = make_decode_inputs(B, Hq, Hkv, D, cap, lens, dt, seed=17 + case, pad_fill=NAN)
    out, lse = _run(inp, num_splits)
    ro, rl = _oracle(inp)
    check_out(out, ro)
    check_lse(lse, rl)


def test_splits_beyond_length():
    # more fixed splits than keys: trailing splits are empty and must weigh nothing
    for dt, Hq, Hkv in [(torch.float32, 2, 2), (torch.bfloat16, 16, 2)]:
        inp = make_decode_inputs(2, Hq, Hkv, 128, 40, [5, 3], dt, seed=3, pad_fill=NAN)
        out, lse = _run(inp, 16)
        ro, rl = _oracle(inp)
        check_out(out, ro)
        check_lse(lse, rl)


def test_zero_query_gives_mean():
    inp = make_decode_inputs(2, 16, 2, 128, 600, [500, 77], torch.bfloat16, seed=5, pad_fill=NAN)
    inp.q.zero_()
    out, lse = _run(inp)
    ro, rl = _oracle(inp)
    check_out(out, ro)
    check_lse(lse, rl)
    assert np.allclose(lse.cpu().numpy(), np.log([[500.0] * 16, [77.0] * 16]), atol=1e-3)


def test_peaked_keys():
    inp = make_decode_inputs(2, 64, 8, 128, 4096, [4096, 3000], torch.bfloat16, seed=9,
                             peaked_rows=8, peak_scale=8.0, pad_fill=NAN)
    out, lse = _run(inp)
    ro, rl = _oracle(inp)
    check_out(out, ro)
    check_lse(lse, rl)


def test_full_workload_1_fp32():
    inp = workload(1, pad_fill=NAN)
    out, lse = _run(inp)
    ro, rl = _oracle(inp)
    check_out(out, ro, "workload 1 out")
    check_lse(lse, rl, "workload 1 lse")


@pytest.mark.parametrize("index,batch", [(2, None), (3, None), (4, 1), (4, 2)])
def test_full_workloads(index, batch):
    # the benchmark shapes at full size, in the launch configuration bench.py times: every
    # output element against the oracle
    inp = workload(index, batch=batch)
    out, lse = _run(inp, guard=False)
    ro, rl = _oracle(inp)
    check_out(out, ro, f"workload {index} (batch {batch or inp.q.shape[0]}) out")
    check_lse(lse, rl, f"workload {index} (batch {batch or inp.q.shape[0]}) lse")


def test_deterministic_and_stream():
    inp = make_decode_inputs(4, 64, 8, 128, 3000, [3000, 1, 2048, 999], torch.bfloat16, seed=11)
    o1, l1 = _run(inp)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        o2, l2 = _run(inp, stream=s)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_device_plan_equals_host_plan():
    fd = _fd()
    from workloads import uniform_lens
    rng = np.random.default_rng(0)
    for trial in range(13):
        if trial == 0:   # the 70B-like decode workload's plan first
            B, cap, hkv, fixed, nctas = 32, 32768, 8, 0, 148
            lens = uniform_lens(1103, 32, 1024, 32768)
        else:
            B = int(rng.choice([1, 3, 32, 100, 1000]))
            cap = int(rng.choice([64, 1024, 32768]))
            hkv = int(rng.choice([1, 8, 40]))
            fixed = int(rng.choice([0, 0, 4]))
            nctas = int(rng.choice([148, 296]))
            lens = [int(x) for x in rng.integers(-3, cap + 3, size=B)]
        info, splits, items = fd.fd_split_plan(lens, hkv, cap, fixed, nctas)
        ref = oplan.decode_plan(lens, hkv, cap, nctas, fixed)
        dl = torch.tensor(lens, dtype=torch.int32, device="cuda")
        total, dsplits, ditems = fd.fd_split_plan_device(dl, hkv, cap, fixed, nctas,
                                                         items_capacity=info["total_items"])
        torch.cuda.synchronize()
        assert int(total.item()) == info["total_items"] == ref.total_items
        assert dsplits.cpu().tolist() == splits == ref.splits_per_seq
        assert [tuple(x) for x in ditems.cpu().tolist()] == [tuple(x) for x in items] == ref.items
    fd.fd_poll_status()


def test_length_clamp_flag():
    fd = _fd()
    inp = make_decode_inputs(2, 16, 2, 128, 256, [256, 10], torch.bfloat16, seed=21)
    fd.fd_poll_status()
    good_o, good_l = _run(inp)
    inp.cache_lens = torch.tensor([300, -4], dtype=torch.int32)
    dev = torch.device("cuda", 0)
    out, lse = fd.fd_decode_attention(inp.q.to(dev), inp.k_cache.to(dev), inp.v_cache.to(dev),
                                      inp.cache_lens.to(dev))
    flags = fd.fd_poll_status()
    assert flags & fd.FD_FLAG_LEN_CLAMPED
    assert fd.fd_poll_status() == 0, "poll clears the flags"
    assert torch.equal(out[0], good_o[0]) and torch.equal(lse[0], good_l[0])
    assert bool((out[1].float() == 0).all()) and bool(torch.isneginf(lse[1]).all())


def test_cuda_graph_replay_new_lengths():
    fd = _fd()
    from workloads import DecodeInputs
    dev = torch.device("cuda", 0)
    base = make_decode_inputs(3, 64, 8, 128, 2048, [2048] * 3, torch.bfloat16, seed=31)
    q, k, v = base.q.to(dev), base.k_cache.to(dev), base.v_cache.to(dev)
    lens = base.cache_lens.to(dev)
    out = torch.empty_like(q)
    lse = torch.empty(q.shape[:2], dtype=torch.float32, device=dev)
    s = torch.cuda.Stream()
    nct = fd.fd_decode_num_ctas(0, torch.bfloat16, 8, 128)
    fd.fd_reserve_workspace(fd.fd_decode_workspace_bytes(3, 64, 8, 2048, 128, 0, nct), stream=s)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        fd.fd_decode_attention(q, k, v, lens, 0, out=out, lse=lse, stream=s)
    for new in ([2048, 100, 1500], [7, 2000, 1]):
        # cache rows past the new lengths must not be read: poison them with NaN
        kk = base.k_cache.clone()
        vv = base.v_cache.clone()
        for b, n in enumerate(new):
            kk[b, :, n:] = NAN
            vv[b, :, n:] = NAN
        k.copy_(kk)
        v.copy_(vv)
        lens.copy_(torch.tensor(new, dtype=torch.int32))
        g.replay()
        torch.cuda.synchronize()
        ref_in = DecodeInputs(q=base.q, k_cache=kk, v_cache=vv,
                              cache_lens=torch.tensor(new, dtype=torch.int32))
        ro, rl = _oracle(ref_in)
        check_out(out, ro)
        check_lse(lse, rl)
    del g


def test_many_pairs_combine():
    # 300 sequences x 32 query heads = 9,600 (row, head) pairs with 3 splits each: the combine's
    # many-pair warp kernel (4 splits in flight per warp)
    rng = np.random.default_rng(950)
    lens = [int(x) for x in rng.integers(0, 601, size=300)]
    inp = make_decode_inputs(300, 32, 4, 128, 600, lens, torch.bfloat16, seed=951, pad_fill=NAN)
    out, lse = _run(inp, 3)
    ro, rl = _oracle(inp)
    check_out(out, ro, "many pairs out")
    check_lse(lse, rl, "many pairs lse")


@pytest.mark.parametrize("B", [255, 256, 257])
def test_batch_around_in_kernel_plan_limit(B):
    # up to 256 sequences the tensor-core kernel plans the call itself; above, the planner kernel
    # does: both must give the oracle's result
    rng = np.random.default_rng(900 + B)
    lens = [int(x) for x in rng.integers(0, 321, size=B)]
    inp = make_decode_inputs(B, 16, 2, 128, 320, lens, torch.bfloat16, seed=900 + B,
                             pad_fill=NAN)
    out, lse = _run(inp)
    ro, rl = _oracle(inp)
    check_out(out, ro, f"B {B} out")
    check_lse(lse, rl, f"B {B} lse")


def test_paths_share_workspace_cursor():
    # CUDA-core, tensor-core and chunked-prefill calls on one stream share one workspace and its
    # work cursor; every kernel that claims from the cursor leaves it at zero for the next call
    fd = _fd()
    from workloads import make_chunk_inputs
    dev = torch.device("cuda", 0)
    mha = make_decode_inputs(3, 8, 8, 128, 700, [700, 3, 333], torch.bfloat16, seed=71,
                             pad_fill=NAN)
    gqa = make_decode_inputs(4, 64, 8, 128, 1500, [1500, 17, 900, 256], torch.bfloat16, seed=72,
                             pad_fill=NAN)
    chk = make_chunk_inputs([400, 90], [140, 1], 8, 2, 128, 600, torch.bfloat16, seed=73,
                            pad_fill=NAN)
    s = torch.cuda.Stream()

    def chunk_call():
        q = chk.q_chunk.to(dev)
        out, lse = fd.fd_chunk_prefill_attention(q, chk.k_cache.to(dev), chk.v_cache.to(dev),
                                                 chk.prefix_lens.to(dev), chk.chunk_lens.to(dev),
                                                 stream=s)
        torch.cuda.synchronize()
        ro, rl = oracle.chunk_prefill_attention(
            to_numpy_exact(chk.q_chunk), to_numpy_exact(chk.k_cache), to_numpy_exact(chk.v_cache),
            chk.prefix_lens.tolist(), chk.chunk_lens.tolist())
        check_out(out, ro, "chunk out")
        check_lse(lse, rl, "chunk lse")

    def decode_call(inp):
        with torch.cuda.stream(s):
            out, lse = _run(inp, stream=s)
        ro, rl = _oracle(inp)
        check_out(out, ro, "out")
        check_lse(lse, rl, "lse")

    for step in (lambda: decode_call(mha), lambda: decode_call(gqa), chunk_call,
                 lambda: decode_call(gqa), lambda: decode_call(mha), lambda: decode_call(gqa)):
        step()
    assert fd.fd_poll_status(stream=s) & (fd.FD_FLAG_WAIT_TIMEOUT | fd.FD_FLAG_PLAN_OVERFLOW) == 0


def test_many_kv_heads_then_small_calls():
    # 256 sequences x 257 KV heads (G = 2, 65792 groups, the in-kernel plan's largest batch)
    # between two small calls on the same stream: all three match the oracle
    rng = np.random.default_rng(4242)
    B, hkv = 256, 257
    lens = [int(x) for x in rng.integers(0, 33, size=B)]
    big = make_decode_inputs(B, 2 * hkv, hkv, 128, 32, lens, torch.bfloat16, seed=4243,
                             pad_fill=NAN)
    small = make_decode_inputs(3, 64, 8, 128, 700, [700, 5, 300], torch.bfloat16, seed=4244,
                               pad_fill=NAN)
    for inp, ns in ((small, 4), (big, 2), (small, 0)):
        out, lse = _run(inp, ns)
        ro, rl = _oracle(inp)
        check_out(out, ro, f"B {inp.q.shape[0]} x {inp.k_cache.shape[1]} KV heads out")
        check_lse(lse, rl, f"B {inp.q.shape[0]} x {inp.k_cache.shape[1]} KV heads lse")
