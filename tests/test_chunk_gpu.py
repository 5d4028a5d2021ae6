"""GPU parity of fd_chunk_prefill_attention against the float64 oracle, through the C ABI.

Caches hold NaN past every request's prefix + chunk, so a read beyond the causal limit poisons
the result; outputs sit inside guard bands that must stay untouched.
"""

import numpy as np
import pytest
import torch

from oracle import attention as oracle
from parity import check_lse, check_out
from workloads import make_chunk_inputs, to_numpy_exact, workload

pytestmark = pytest.mark.gpu

NAN = float("nan")


def _run(inp, guard=True):
    import split_kv_decode_flashdecoding_b200 as fd
    dev = torch.device("cuda", 0)
    q = inp.q_chunk.to(dev)
    T, Hq, D = q.shape
    if guard:
        big = torch.full((T + 2, Hq, D), 4321.0, dtype=q.dtype, device=dev)
        out = big[1:T + 1]
        lbig = torch.full((T * Hq + 64,), 555.0, dtype=torch.float32, device=dev)
        lse = lbig[32:32 + T * Hq].view(T, Hq)
    else:
        out = torch.empty_like(q)
        lse = torch.empty((T, Hq), dtype=torch.float32, device=dev)
    fd.fd_chunk_prefill_attention(q, inp.k_cache.to(dev), inp.v_cache.to(dev),
                                  inp.prefix_lens.to(dev), inp.chunk_lens.to(dev), out=out, lse=lse)
    torch.cuda.synchronize()
    if guard:
        assert bool((big[0] == 4321.0).all()) and bool((big[T + 1] == 4321.0).all()), "out guard band"
        assert bool((lbig[:32] == 555.0).all()) and bool((lbig[32 + T * Hq:] == 555.0).all()), "lse guard"
    flags = fd.fd_poll_status()
    assert flags & fd.FD_FLAG_WAIT_TIMEOUT == 0 and flags & fd.FD_FLAG_PLAN_OVERFLOW == 0, hex(flags)
    return out, lse


def _oracle(inp, rows=None):
    return oracle.chunk_prefill_attention(
        to_numpy_exact(inp.q_chunk), to_numpy_exact(inp.k_cache), to_numpy_exact(inp.v_cache),
        inp.prefix_lens.tolist(), inp.chunk_lens.tolist(), rows=rows)


CASES = [
    # (prefix_lens, chunk_lens, Hq, Hkv, cap)
    ([0], [5], 2, 2, 64),                          # tiny chunk, no prefix
    ([300], [130], 2, 2, 512),                     # two tiles, ragged second tile
    ([3900], [300], 2, 2, 8192),                   # tile 0 one split, tiles 1-2 two splits
    ([2500, 10, 0, 700, 33], [200, 1, 1, 1, 0], 4, 4, 4096),  # chunk + decode rows + empty
    ([1000, 77, 4000], [129, 1, 1], 16, 2, 4200),  # GQA (G = 8): decode rows on tensor cores
    ([64], [64], 4, 1, 128),                       # GQA G = 4, capacity = prefix + chunk
]


@pytest.mark.parametrize("case", range(len(CASES)))
def test_small_chunks(case):
    prefix, chunk, hq, hkv, cap = CASES[case]
    inp = make_chunk_inputs(prefix, chunk, hq, hkv, 128, cap, torch.bfloat16, seed=300 + case,
                            pad_fill=NAN)
    out, lse = _run(inp)
    ro, rl = _oracle(inp)
    check_out(out, ro, "chunk out")
    check_lse(lse, rl, "chunk lse")


# head_dim 64: the tile kernel's D = 64 instantiation; decode rows of any group run on CUDA cores
CASES_D64 = [
    # (prefix_lens, chunk_lens, Hq, Hkv, cap)
    ([300], [130], 2, 2, 512),                     # two tiles, ragged second tile
    ([3900, 10, 0], [300, 1, 1], 4, 4, 4304),      # one, then two key splits per tile + decode rows
    ([1000, 77, 4000], [129, 1, 1], 16, 2, 4200),  # GQA (G = 8)
    ([3000, 5], [4, 4], 32, 8, 3072),              # verification, head-packed tiles (G = 4)
    ([5000, 50, 2000], [300, 1, 40], 32, 4, 5400),  # 10,912 (row, head) pairs: many-pair combine
]


@pytest.mark.parametrize("case", range(len(CASES_D64)))
def test_small_chunks_head_dim_64(case):
    prefix, chunk, hq, hkv, cap = CASES_D64[case]
    inp = make_chunk_inputs(prefix, chunk, hq, hkv, 64, cap, torch.bfloat16, seed=400 + case,
                            pad_fill=NAN)
    out, lse = _run(inp)
    ro, rl = _oracle(inp)
    check_out(out, ro, "chunk D 64 out")
    check_lse(lse, rl, "chunk D 64 lse")


def test_chunk_equals_decode_rows():
    # a chunk of 3 rows at prefix p gives, row by row, the decode results over p + i + 1 keys
    import split_kv_decode_flashdecoding_b200 as fd
    inp = make_chunk_inputs([777], [3], 8, 8, 128, 1024, torch.bfloat16, seed=41)
    out, lse = _run(inp)
    dev = torch.device("cuda", 0)
    for i in range(3):
        q = inp.q_chunk[i:i + 1].to(dev)
        lens = torch.tensor([778 + i], dtype=torch.int32, device=dev)
        o2, l2 = fd.fd_decode_attention(q, inp.k_cache.to(dev), inp.v_cache.to(dev), lens)
        torch.cuda.synchronize()
        check_out(out[i:i + 1], o2.float().cpu().numpy().astype(np.float64), "chunk row vs decode")
        check_lse(lse[i:i + 1], l2.cpu().numpy().astype(np.float64), "chunk row vs decode lse")


def test_full_mixed_workload():
    # the mixed chunked-prefill step at full size: every output element against the oracle
    inp = workload(5)
    out, lse = _run(inp, guard=False)
    ro, rl = _oracle(inp)
    check_out(out, ro, "workload 5 out")
    check_lse(lse, rl, "workload 5 lse")


def test_many_requests_of_every_kind():
    # 70 requests in one call: empty ones, decode rows, head-packed verification steps (G = 4),
    # single-tile and multi-tile chunks, in an irregular order, so the planner's CTAs each write
    # a share of every item kind and of the row tables
    rng = np.random.default_rng(81)
    kinds = [0, 1, 4, 1, 200, 0, 1, 17, 3, 130, 1, 1, 32, 33, 2, 0, 1, 260, 1, 5]
    chunk = [kinds[i % len(kinds)] if i % 7 else int(rng.integers(0, 40)) for i in range(70)]
    cap = 1536
    prefix = [int(rng.integers(0, cap - c + 1)) for c in chunk]
    inp = make_chunk_inputs(prefix, chunk, 16, 4, 128, cap, torch.bfloat16, seed=82, pad_fill=NAN)
    out, lse = _run(inp)
    ro, rl = _oracle(inp)
    check_out(out, ro, "70 requests out")
    check_lse(lse, rl, "70 requests lse")


def test_chunk_lengths_not_matching_rows():
    # chunk lengths that do not add up to q_chunk's rows: nothing is written, the flag is raised
    import split_kv_decode_flashdecoding_b200 as fd
    dev = torch.device("cuda", 0)
    inp = make_chunk_inputs([300, 40], [20, 1], 8, 2, 128, 512, torch.bfloat16, seed=83)
    q = inp.q_chunk.to(dev)
    out = torch.full_like(q, 7.0)
    lse = torch.full(q.shape[:2], 9.0, dtype=torch.float32, device=dev)
    fd.fd_poll_status()
    fd.fd_chunk_prefill_attention(q, inp.k_cache.to(dev), inp.v_cache.to(dev),
                                  inp.prefix_lens.to(dev),
                                  torch.tensor([20, 2], dtype=torch.int32, device=dev),
                                  out=out, lse=lse)
    torch.cuda.synchronize()
    assert fd.fd_poll_status() & fd.FD_FLAG_LEN_CLAMPED
    assert bool((out == 7.0).all()) and bool((lse == 9.0).all())


def test_chunk_deterministic():
    inp = make_chunk_inputs([1500, 3], [260, 1], 4, 4, 128, 2048, torch.bfloat16, seed=51)
    o1, l1 = _run(inp)
    o2, l2 = _run(inp)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


# Multi-token verification steps: requests of 2 <= c <= 128 / G rows with G >= 2 heads per KV head
# run as head-packed tiles (one tile holds the rows of all G heads of a KV head).
VERIFY = [
    # (prefix_lens, chunk_lens, Hq, Hkv, cap)
    ([3000, 5, 0, 2047], [4, 4, 4, 4], 64, 8, 3072),        # G = 8, k = 4: 32 rows per tile
    ([500, 9000], [16, 2], 64, 8, 9216),                     # k = 16 fills the tile; k = 2
    ([700, 60], [32, 17], 16, 4, 1024),                      # G = 4, k = 32 (full) and 17
    ([1000, 33, 2100], [8, 1, 3], 16, 2, 2304),              # G = 8 with a decode row
    ([4100, 300, 90], [4, 17, 130], 32, 4, 4352),            # packed, per-head (17 > 16) and two tiles
    ([257, 0], [3, 5], 6, 2, 320),                           # G = 3: rows r // 3 and r % 3
    ([900, 40], [8, 8], 16, 1, 1024),                        # G = 16, k = 8 fills the tile
    ([2200, 10], [64, 33], 4, 2, 2304),                      # G = 2, k = 64 (full) and 33
    ([6000, 17], [2, 2], 32, 2, 6144),                       # G = 16, k = 2 (32 rows), many splits
    ([1500, 3000], [16, 9], 4, 2, 3072),                     # G = 2, k = 16 and 9
    ([100, 2500, 40], [8, 5, 1], 32, 8, 2560),               # G = 4 with a decode row
    ([800, 50], [5, 4], 12, 2, 1024),                        # G = 6: quarter items of 30 and 24 rows
    ([1300, 2], [4, 3], 7, 1, 1536),                         # G = 7: 28 and 21 rows
]


@pytest.mark.parametrize("case", range(len(VERIFY)))
def test_verification_head_packed(case):
    prefix, chunk, hq, hkv, cap = VERIFY[case]
    inp = make_chunk_inputs(prefix, chunk, hq, hkv, 128, cap, torch.bfloat16, seed=700 + case,
                            pad_fill=NAN)
    out, lse = _run(inp)
    ro, rl = _oracle(inp)
    check_out(out, ro, "verification out")
    check_lse(lse, rl, "verification lse")


def test_verification_equals_decode_rows():
    # k = 4 tokens of one request, G = 8: token i gives the decode result over prefix + i + 1 keys
    import split_kv_decode_flashdecoding_b200 as fd
    inp = make_chunk_inputs([1500], [4], 64, 8, 128, 2048, torch.bfloat16, seed=720)
    out, lse = _run(inp)
    dev = torch.device("cuda", 0)
    for i in range(4):
        q = inp.q_chunk[i:i + 1].to(dev)
        lens = torch.tensor([1501 + i], dtype=torch.int32, device=dev)
        o, l = fd.fd_decode_attention(q, inp.k_cache.to(dev), inp.v_cache.to(dev), lens)
        torch.cuda.synchronize()
        check_out(out[i:i + 1], o.float().cpu().numpy().astype(np.float64), f"token {i} vs decode")
        check_lse(lse[i:i + 1], l.cpu().numpy().astype(np.float64), f"token {i} lse vs decode")


def test_verification_workload():
    # the 70B-like decode batch verifying 4 speculative tokens per sequence, at full size: every
    # output element against the oracle
    inp = workload(6)
    out, lse = _run(inp, guard=False)
    ro, rl = _oracle(inp)
    check_out(out, ro, "workload 6 out")
    check_lse(lse, rl, "workload 6 lse")


def test_verification_cuda_graph_replay():
    # a captured verification step replayed with new prefix lengths (same chunk lengths)
    import split_kv_decode_flashdecoding_b200 as fd
    from workloads import ChunkInputs
    dev = torch.device("cuda", 0)
    prefix, chunk = [3000, 500, 1000], [4, 4, 4]
    base = make_chunk_inputs(prefix, chunk, 64, 8, 128, 4096, torch.bfloat16, seed=730)
    q, k, v = base.q_chunk.to(dev), base.k_cache.to(dev), base.v_cache.to(dev)
    pl, cl = base.prefix_lens.to(dev), base.chunk_lens.to(dev)
    out = torch.empty_like(q)
    lse = torch.empty(q.shape[:2], dtype=torch.float32, device=dev)
    s = torch.cuda.Stream()
    nct = fd.fd_decode_num_ctas(0, torch.bfloat16, 8, 128)
    fd.fd_reserve_workspace(fd.fd_chunk_workspace_bytes(3, 12, 64, 8, 4096, 128, nct), stream=s)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        fd.fd_chunk_prefill_attention(q, k, v, pl, cl, out=out, lse=lse, stream=s)
    for new in ([3000, 500, 1000], [10, 2500, 0]):
        kk = base.k_cache.clone()
        vv = base.v_cache.clone()
        for b, p0 in enumerate(new):
            kk[b, :, p0 + chunk[b]:] = NAN
            vv[b, :, p0 + chunk[b]:] = NAN
        k.copy_(kk)
        v.copy_(vv)
        pl.copy_(torch.tensor(new, dtype=torch.int32))
        g.replay()
        torch.cuda.synchronize()
        ref_in = ChunkInputs(q_chunk=base.q_chunk, k_cache=kk, v_cache=vv,
                             prefix_lens=torch.tensor(new, dtype=torch.int32),
                             chunk_lens=base.chunk_lens)
        ro, rl = _oracle(ref_in)
        check_out(out, ro, "verification graph out")
        check_lse(lse, rl, "verification graph lse")
    del g
