"""The planner oracle against hand-worked plans and its coverage / bound properties.

Parity of the planner is pinned by properties rather than by the pages' allocator, which
targets whole GPUs and drops tokens: every sequence's splits tile [0, len) in order with no gap
or overlap, no split exceeds the chunk, a split of a multi-split sequence never falls under
the allocator's min_chunk of 128, items come longest first, and the item count stays under the
bound the CUDA library uses to size its workspace.
"""

import random

import pytest

from oracle import planner as P


def _bound(B, Hkv, cap, ctas, num_splits):
    if num_splits > 0:
        return Hkv * B * num_splits
    return Hkv * B + max(P.WAVES * ctas, -(-Hkv * B * cap // P.MAX_CHUNK))


def test_fixed_even():
    # one sequence of 1024 keys, 4 fixed splits -> 256 keys each, for every KV head
    p = P.decode_plan([1024], 8, 1024, 148, num_splits=4)
    assert p.splits_per_seq == [4]
    assert p.total_items == 32
    assert sorted({(t0, t1) for (_, _, _, t0, t1) in p.items}) == [
        (0, 256), (256, 512), (512, 768), (768, 1024)]


def test_fixed_ragged_and_empty():
    # chunk_size = ceil(10 / 4) = 3 -> [0,3) [3,6) [6,9) [9,10); len 2 -> [0,1) [1,2) then empties
    p = P.decode_plan([10, 2], 1, 16, 148, num_splits=4)
    got = {b: [] for b in range(2)}
    for b, h, s, t0, t1 in p.items:
        got[b].append((s, t0, t1))
    assert got[0] == [(0, 0, 3), (1, 3, 6), (2, 6, 9), (3, 9, 10)]
    assert got[1] == [(0, 0, 1), (1, 1, 2), (2, 2, 2), (3, 2, 2)]


def test_auto_hand_worked_13b_shape():
    # 4 x 16384 keys, 40 KV heads, 148 CTAs: ceil(65536*40 / (8*148)) = 2215 -> clamp 1024
    p = P.decode_plan([16384] * 4, 40, 16384, 148)
    assert p.chunk_tokens == 1024
    assert p.splits_per_seq == [16, 16, 16, 16]
    assert p.total_items == 4 * 40 * 16


def test_auto_hand_worked_small():
    # total 1300 tokens, 1 KV head: ceil(1300 / 1184) = 2 -> clamp up to 256
    p = P.decode_plan([1000, 300, 0], 1, 4096, 148)
    assert p.chunk_tokens == 256
    assert p.splits_per_seq == [4, 2, 1]
    assert p.items == [(0, 0, 0, 0, 250), (0, 0, 1, 250, 500), (0, 0, 2, 500, 750),
                       (0, 0, 3, 750, 1000), (1, 0, 0, 0, 150), (1, 0, 1, 150, 300),
                       (2, 0, 0, 0, 0)]


def test_auto_hand_worked_long_context():
    # one 32768-key sequence, 8 KV heads, 148 CTAs (U = 262144 token-heads):
    #   W = 8: chunk max(256, ceil(U / 1184) = 222) = 256, 128 splits, 1024 items, 7 waves x (2 + 2) = 28
    #   W = 4: chunk 443, 74 splits, 592 items, 4 waves x (4 + 2) = 24
    #   W = 2: chunk 886, 37 splits, 296 items, 2 waves x (7 + 2) = 18   <- least
    #   W = 1: chunk min(1772, 1024) = 1024, 32 splits, 256 items, 2 waves x (8 + 2) = 20
    p = P.decode_plan([32768], 8, 32768, 148)
    assert p.chunk_tokens == 886 and p.splits_per_seq == [37] and p.total_items == 296
    # two such sequences: W = 4 (chunk 886, 592 items, 4 waves x 9 = 36) beats W = 2 / 1 (chunk
    # 1024, 512 items, 4 waves x 10 = 40) and W = 8 (chunk 443, 1184 items, 8 waves x 6 = 48)
    p = P.decode_plan([32768, 32768], 8, 32768, 148)
    assert p.chunk_tokens == 886 and p.splits_per_seq == [37, 37]
    # the 70B-like decode batch: chunk 1024 for every W, so the W = 8 plan
    from workloads import uniform_lens
    lens = uniform_lens(1103, 32, 1024, 32768)
    p = P.decode_plan(lens, 8, 32768, 148)
    assert p.chunk_tokens == 1024
    assert p.splits_per_seq == [-(-n // 1024) for n in lens]


def test_auto_clamps_lengths():
    p = P.decode_plan([-5, 10**9], 2, 3000, 148)
    assert p.splits_per_seq[0] == 1
    spans = [(t0, t1) for (b, h, s, t0, t1) in p.items if b == 1 and h == 0]
    assert spans[0][0] == 0 and spans[-1][1] == 3000


@pytest.mark.parametrize("seed", range(40))
def test_properties_random(seed):
    rng = random.Random(seed)
    B = rng.choice([1, 2, 3, 7, 32, 100])
    Hkv = rng.choice([1, 2, 8, 40])
    cap = rng.choice([1, 63, 64, 65, 257, 1024, 4096, 32768])
    ctas = rng.choice([1, 8, 148])
    num_splits = rng.choice([0, 0, 0, 1, 3, 8, 40])
    lens = [rng.choice([0, 1, cap - 1, cap, rng.randint(0, cap)]) for _ in range(B)]
    p = P.decode_plan(lens, Hkv, cap, ctas, num_splits)
    again = P.decode_plan(lens, Hkv, cap, ctas, num_splits)
    assert p == again, "deterministic"
    assert p.total_items == Hkv * sum(p.splits_per_seq)
    assert p.total_items <= _bound(B, Hkv, cap, ctas, num_splits)
    if num_splits == 0:
        assert P.MIN_CHUNK <= p.chunk_tokens <= P.MAX_CHUNK
    per = {}
    for b, h, s, t0, t1 in p.items:
        per.setdefault((b, h), []).append((s, t0, t1))
    keys = []
    for b in range(B):
        n = max(0, min(lens[b], cap))
        for h in range(Hkv):
            sp = per[(b, h)]
            assert [s for s, _, _ in sp] == list(range(len(sp)))
            assert sp[0][1] == 0 and sp[-1][2] == n, "splits cover [0, len)"
            for (_, a0, a1), (_, c0, c1) in zip(sp, sp[1:]):
                assert a1 == c0, "no gap, no overlap"
            for _, t0, t1 in sp:
                assert 0 <= t0 <= t1 <= n
                if num_splits == 0:
                    assert t1 - t0 <= p.chunk_tokens
                    if len(sp) > 1:
                        assert t1 - t0 >= 128, "no piece under min_chunk"
        keys.append(max(t1 - t0 for _, t0, t1 in per[(b, 0)]))
    # longest-first order over sequences
    order = []
    for b, h, s, t0, t1 in p.items:
        if not order or order[-1] != b:
            order.append(b)
    assert len(order) == B, "a sequence's items are contiguous"
    ks = [keys[b] for b in order]
    assert ks == sorted(ks, reverse=True)


def test_chunk_plan_hand_worked():
    # request 0: chunk 300 at prefix 5000, 2 heads; request 1: decode row over 70 keys
    cp = P.chunk_plan([5000, 69], [300, 1], 2, 2, 8192, 148)
    assert cp.decode_requests == [1]
    assert cp.decode.splits_per_seq == [1]
    # tiles see <= 5128, 5256, 5300 keys -> 2 splits each on the 4096-key grid
    assert cp.row_splits == [2] * 300 + [1]
    spans = sorted({(t, s, k0, k1) for (b, t, h, s, k0, k1) in cp.tile_items if t == 0})
    assert spans == [(0, 0, 0, 4096), (0, 1, 4096, 5128)]
    assert len(cp.tile_items) == 3 * 2 * 2
    # order: head, split, tile
    assert [(h, s, t) for (b, t, h, s, k0, k1) in cp.tile_items[:4]] == [
        (0, 0, 0), (0, 0, 1), (0, 0, 2), (0, 1, 0)]


def test_chunk_plan_tiles_with_fewer_splits():
    # a 300-row chunk at prefix 3900: tile 0 sees <= 4028 keys (1 split), tiles 1-2 see more (2)
    cp = P.chunk_plan([3900], [300], 1, 1, 8192, 148)
    assert cp.row_splits == [1] * 128 + [2] * 172
    assert [(t, s, k0, k1) for (b, t, h, s, k0, k1) in cp.tile_items] == [
        (0, 0, 0, 4028), (1, 0, 0, 4096), (2, 0, 0, 4096), (1, 1, 4096, 4156), (2, 1, 4096, 4200)]


# ---- aligned plans (paged cache): split boundaries on multiples of the key tile ----------------

def test_aligned_plan_hand_cases():
    # planner mode: 300 keys, 2 splits of whole 128-key units: units = 3 -> [0, 128), [128, 300)
    assert P._split_bounds_equal(300, 2, 128) == [(0, 128), (128, 300)]
    # 1000 keys, 3 splits: units = 8 -> boundaries at units 0, 2, 5, 8
    assert P._split_bounds_equal(1000, 3, 128) == [(0, 256), (256, 640), (640, 1000)]
    # fixed mode: chunk ceil(300 / 2) = 150 rounded up to 256
    assert P._split_bounds_fixed(300, 2, 128) == [(0, 256), (256, 300)]
    assert P._split_bounds_fixed(100, 4, 16) == [(0, 32), (32, 64), (64, 96), (96, 100)]
    # align 1 is the unaligned rule
    assert P._split_bounds_equal(1000, 3, 1) == P._split_bounds_equal(1000, 3)


@pytest.mark.parametrize("seed", range(6))
def test_aligned_plan_properties(seed):
    rng = random.Random(seed)
    B = rng.randint(1, 39)
    lens = [rng.randint(0, 19999) for _ in range(B)]
    for fixed in (0, 3):
        plan = P.decode_plan(lens, 4, 20000, 148, fixed, align=128)
        ref = P.decode_plan(lens, 4, 20000, 148, fixed)
        # same split counts and order, only the boundaries move
        assert plan.splits_per_seq == ref.splits_per_seq
        assert [it[:3] for it in plan.items] == [it[:3] for it in ref.items]
        for b in range(B):
            bounds = [(t0, t1) for (bb, h, s, t0, t1) in plan.items if bb == b and h == 0]
            assert bounds[0][0] == 0 and bounds[-1][1] == lens[b]
            for (a0, a1), (c0, c1) in zip(bounds, bounds[1:]):
                assert a1 == c0
            for t0, t1 in bounds:
                # boundaries on the 128-key grid, except at the sequence end (trailing empty
                # splits of a fixed count sit at [len, len))
                assert t0 <= t1 and (t0 % 128 == 0 or t0 == lens[b])
                assert t1 % 128 == 0 or t1 == lens[b]


def test_chunk_plan_head_packed_requests():
    # G = 8: chunks of 2..16 rows are head-packed (one tile per KV head and split), longer ones
    # and decode rows are not; G = 1 never packs
    cp = P.chunk_plan([5000, 40, 100, 7], [4, 16, 17, 1], 64, 8, 8192, 148)
    assert cp.head_packed == [0, 1]
    heads0 = sorted({h for (b, t, h, s, k0, k1) in cp.tile_items if b == 0})
    assert heads0 == list(range(8))
    # request 0 sees 5004 keys: two splits per KV head, one query tile
    assert sorted({(t, s, k0, k1) for (b, t, h, s, k0, k1) in cp.tile_items if b == 0}) == \
        [(0, 0, 0, 4096), (0, 1, 4096, 5004)]
    assert len([1 for it in cp.tile_items if it[0] == 2]) == 64      # per query head
    assert cp.row_splits[:4] == [2, 2, 2, 2] and cp.row_splits[4:20] == [1] * 16
    assert P.chunk_plan([10], [4], 8, 8, 1024, 148).head_packed == []


@pytest.mark.parametrize("seed", range(6))
def test_chunk_plan_head_packed_coverage(seed):
    # every chunk request is covered exactly once per (head, split, tile): KV heads for
    # head-packed requests (2 <= c <= 128 / G, G >= 2), query heads otherwise
    rng = random.Random(seed)
    hkv = rng.choice([1, 2, 4, 8])
    G = rng.choice([1, 2, 3, 4, 8, 16])
    hq = hkv * G
    cap = 8192
    B = rng.randint(1, 10)
    chunk = [rng.choice([0, 1, 2, 4, 8, 16, 17, 33, 64, 130, 300]) for _ in range(B)]
    prefix = [rng.randint(0, cap - c) for c in chunk]
    cp = P.chunk_plan(prefix, chunk, hq, hkv, cap, 148)
    want_packed = [b for b in range(B) if G >= 2 and 2 <= chunk[b] and chunk[b] * G <= 128]
    assert cp.head_packed == want_packed
    for b in range(B):
        c = chunk[b]
        if c < 2:
            assert not [it for it in cp.tile_items if it[0] == b]
            continue
        heads = hkv if b in want_packed else hq
        n_tiles = -(-c // 128)
        seen = {}
        for (bb, t, h, s, k0, k1) in cp.tile_items:
            if bb == b:
                seen[(t, h, s)] = seen.get((t, h, s), 0) + 1
                assert 0 <= h < heads and 0 <= t < n_tiles and k0 <= k1
        assert set(seen.values()) == {1}
        # each (tile, head) covers the tile's keys [0, K_t) exactly, split by split
        for t in range(n_tiles):
            kt = min(prefix[b] + min(c, 128 * (t + 1)), cap)
            for h in range(heads):
                spans = sorted((k0, k1) for (bb, tt, hh, s, k0, k1) in cp.tile_items
                               if bb == b and tt == t and hh == h)
                assert spans[0][0] == 0 and spans[-1][1] == kt
                assert all(a[1] == b_[0] for a, b_ in zip(spans, spans[1:]))
