"""Checks that pin the float64 oracle to things other than itself.

Each ``pin_*`` takes the oracle's attention module (``oracle.attention`` or a deliberately
mutated copy of it) and raises AssertionError when the module disagrees with:

* hand-derived closed-form fixtures under tests/golden/ (decode and causal chunk);
* closed forms: q = 0 gives the mean of the visible V rows and LSE = ln n; n = 1 gives v_0 and
  LSE = s_0; two keys give sigmoid weights; a dominant score selects one V row; equal scores
  give the mean;
* library routines computed independently on the CPU: torch.softmax / torch.logsumexp in
  float64 followed by a matmul, and torch's scaled_dot_product_attention with a causal mask;
* invariants: any split of the keys merged by log-sum-exp equals no split; jointly permuting K
  and V rows changes nothing; the pages' sequential online softmax and split-then-merge
  algorithms (oracle/formulations.py) give the same result.

tests/test_oracle_pins.py runs them on the real oracle; tests/test_oracle_mutations.py plants
mistakes in a copy of the oracle and checks that some pin catches each one.
"""

from __future__ import annotations

import json
import math
import os

import numpy as np
import torch

from oracle import formulations

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")
TOL = 1e-12


def _close(a, b, tol=TOL, what=""):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    assert a.shape == b.shape, f"{what}: shape {a.shape} vs {b.shape}"
    both_inf = np.isinf(a) & np.isinf(b) & (np.sign(a) == np.sign(b))
    with np.errstate(invalid="ignore"):  # inf - inf where both sides are the same infinity
        err = np.where(both_inf, 0.0, np.abs(a - b))
    assert np.all(np.isfinite(err)), f"{what}: non-finite mismatch"
    m = float(err.max()) if err.size else 0.0
    assert m <= tol * max(1.0, float(np.abs(np.where(both_inf, 0, b)).max() if b.size else 1.0)), \
        f"{what}: max abs err {m:.3e}"


def _rand(shape, seed, scale=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * scale


def _torch_reference(q, k, v, lens, scale):
    """softmax(q·Kᵀ·scale)·V and logsumexp with torch float64 library routines, head h -> kv h//G."""
    B, Hq, D = q.shape
    Hkv = k.shape[1]
    G = Hq // Hkv
    out = np.zeros((B, Hq, D))
    lse = np.zeros((B, Hq))
    for b in range(B):
        n = int(lens[b])
        for h in range(Hq):
            if n == 0:
                out[b, h] = 0.0
                lse[b, h] = -math.inf
                continue
            K = torch.from_numpy(np.ascontiguousarray(k[b, h // G, :n], dtype=np.float64))
            V = torch.from_numpy(np.ascontiguousarray(v[b, h // G, :n], dtype=np.float64))
            qq = torch.from_numpy(np.ascontiguousarray(q[b, h], dtype=np.float64))
            s = torch.mv(K, qq) * scale
            out[b, h] = (torch.softmax(s, dim=0) @ V).numpy()
            lse[b, h] = float(torch.logsumexp(s, dim=0))
    return out, lse


# ---- fixtures -------------------------------------------------------------------------------

def pin_golden_decode(att):
    with open(os.path.join(GOLDEN, "decode_two_keys_exact.json")) as f:
        g = json.load(f)
    q = np.array(g["q"])
    k = np.array(g["k_cache"])
    v = np.array(g["v_cache"])
    out, lse = att.decode_attention(q, k, v, g["cache_lens"])
    _close(out, g["expected_out"], g["tolerance"], "golden decode O")
    _close(lse, g["expected_lse"], g["tolerance"], "golden decode LSE")


def pin_golden_chunk(att):
    with open(os.path.join(GOLDEN, "chunk_causal_exact.json")) as f:
        g = json.load(f)
    out, lse = att.chunk_prefill_attention(np.array(g["q_chunk"]), np.array(g["k_cache"]),
                                           np.array(g["v_cache"]), g["prefix_lens"],
                                           g["chunk_lens"])
    _close(out, g["expected_out"], g["tolerance"], "golden chunk O")
    _close(lse, g["expected_lse"], g["tolerance"], "golden chunk LSE")


# ---- closed forms ---------------------------------------------------------------------------

def pin_zero_query_is_mean(att):
    # GQA G = 2, distinct V per KV head, ragged lengths: O = mean of the visible V rows.
    B, Hq, Hkv, S, D = 2, 4, 2, 9, 8
    q = np.zeros((B, Hq, D))
    k = _rand((B, Hkv, S, D), 1)
    v = _rand((B, Hkv, S, D), 2)
    lens = [5, 9]
    out, lse = att.decode_attention(q, k, v, lens)
    for b in range(B):
        for h in range(Hq):
            _close(out[b, h], v[b, h // 2, :lens[b]].mean(axis=0), what="q=0 mean")
            _close(lse[b, h], math.log(lens[b]), what="q=0 LSE")


def pin_single_key(att):
    B, Hq, Hkv, S, D = 1, 2, 1, 4, 16
    q = _rand((B, Hq, D), 3)
    k = _rand((B, Hkv, S, D), 4)
    v = _rand((B, Hkv, S, D), 5)
    out, lse = att.decode_attention(q, k, v, [1])
    for h in range(Hq):
        s0 = math.fsum(float(a) * float(c) for a, c in zip(q[0, h], k[0, 0, 0])) / math.sqrt(D)
        _close(out[0, h], v[0, 0, 0], what="n=1 O")
        _close(lse[0, h], s0, what="n=1 LSE")


def pin_two_keys_sigmoid(att):
    D = 8
    q = _rand((1, 1, D), 6)
    k = _rand((1, 1, 2, D), 7)
    v = _rand((1, 1, 2, D), 8)
    out, lse = att.decode_attention(q, k, v, [2])
    s = [math.fsum(float(a) * float(c) for a, c in zip(q[0, 0], k[0, 0, j])) / math.sqrt(D)
         for j in range(2)]
    sig = lambda x: 1.0 / (1.0 + math.exp(-x))
    expect = sig(s[0] - s[1]) * v[0, 0, 0] + sig(s[1] - s[0]) * v[0, 0, 1]
    _close(out[0, 0], expect, what="two-key O")
    hi, lo = max(s), min(s)
    _close(lse[0, 0], hi + math.log1p(math.exp(lo - hi)), what="two-key LSE")


def pin_one_hot(att):
    # Orthogonal query heads; each head has its own key that beats every other score by
    # hundreds of nats, so O is that key's V row to float64 precision.
    B, Hq, Hkv, S, D = 1, 4, 2, 12, 16
    q = np.zeros((B, Hq, D))
    for h in range(Hq):
        q[0, h, h] = 3.0
    k = _rand((B, Hkv, S, D), 10, scale=1e-3)
    v = _rand((B, Hkv, S, D), 11)
    hot = {0: 3, 1: 7, 2: 1, 3: 10}
    for h, j in hot.items():
        k[0, h // 2, j, h] = 400.0
    out, lse = att.decode_attention(q, k, v, [S])
    for h, j in hot.items():
        _close(out[0, h], v[0, h // 2, j], what=f"one-hot head {h}")
        _close(lse[0, h], float(q[0, h] @ k[0, h // 2, j]) / 4.0, 1e-9, f"one-hot LSE {h}")


def pin_equal_scores(att):
    B, Hq, Hkv, S, D = 1, 2, 1, 7, 8
    q = _rand((B, Hq, D), 12)
    row = _rand((D,), 13)
    k = np.broadcast_to(row, (B, Hkv, S, D)).copy()
    v = _rand((B, Hkv, S, D), 14)
    out, lse = att.decode_attention(q, k, v, [6])
    for h in range(Hq):
        s = math.fsum(float(a) * float(c) for a, c in zip(q[0, h], row)) / math.sqrt(D)
        _close(out[0, h], v[0, 0, :6].mean(axis=0), what="equal scores O")
        _close(lse[0, h], s + math.log(6), what="equal scores LSE")


def pin_empty_and_clamp(att):
    B, Hq, Hkv, S, D = 3, 2, 1, 5, 4
    q = _rand((B, Hq, D), 15)
    k = _rand((B, Hkv, S, D), 16)
    v = _rand((B, Hkv, S, D), 17)
    out, lse = att.decode_attention(q, k, v, [0, 99, -3])
    assert np.all(out[0] == 0.0) and np.all(lse[0] == -math.inf), "len 0: O = 0, LSE = -inf"
    assert np.all(out[2] == 0.0) and np.all(lse[2] == -math.inf), "negative len clamps to 0"
    ref, rl = att.decode_attention(q, k, v, [0, S, 0])
    _close(out[1], ref[1], what="len > capacity clamps")
    _close(lse[1], rl[1], what="len > capacity clamps (LSE)")


# ---- library routines -----------------------------------------------------------------------

def pin_torch_softmax(att):
    B, Hq, Hkv, S, D = 3, 8, 2, 37, 16
    q = _rand((B, Hq, D), 20, 2.0)
    k = _rand((B, Hkv, S, D), 21)
    v = _rand((B, Hkv, S, D), 22)
    lens = [37, 1, 20]
    out, lse = att.decode_attention(q, k, v, lens)
    ro, rl = _torch_reference(q, k, v, lens, 1.0 / math.sqrt(D))
    _close(out, ro, 1e-11, "torch softmax O")
    _close(lse, rl, 1e-11, "torch logsumexp")


def _sdpa_causal(q, k, v, scale):
    """q/k/v [H, L, D] float64 -> (O [H, L, D], LSE [H, L]) with a square causal mask."""
    Q, K, V = (torch.from_numpy(np.ascontiguousarray(x)) for x in (q, k, v))
    O = torch.nn.functional.scaled_dot_product_attention(Q, K, V, is_causal=True, scale=scale)
    s = (Q @ K.transpose(-1, -2)) * scale
    L = s.shape[-1]
    s = s.masked_fill(torch.ones(L, L, dtype=torch.bool).triu(1), -math.inf)
    return O.numpy(), torch.logsumexp(s, dim=-1).numpy()


def pin_chunk_equals_full_causal(att):
    # A sequence of 23 tokens: chunked prefill of rows [prefix, prefix + chunk) over a cache
    # that already holds all 23 K/V rows must equal rows of full causal attention.
    H, L, D = 2, 23, 8
    q = _rand((H, L, D), 30)
    k = _rand((H, L, D), 31)
    v = _rand((H, L, D), 32)
    scale = 1.0 / math.sqrt(D)
    full_o, full_l = _sdpa_causal(q, k, v, scale)
    cache_k = k[None]
    cache_v = v[None]
    for prefix, chunk in [(0, 23), (5, 7), (10, 13), (22, 1)]:
        qc = np.transpose(q[:, prefix:prefix + chunk], (1, 0, 2))
        o, l = att.chunk_prefill_attention(qc, cache_k, cache_v, [prefix], [chunk])
        _close(o, np.transpose(full_o[:, prefix:prefix + chunk], (1, 0, 2)), 1e-11,
               f"chunk ({prefix},{chunk}) O")
        _close(l, full_l[:, prefix:prefix + chunk].T, 1e-11, f"chunk ({prefix},{chunk}) LSE")
    # decode over len keys equals the last row of full causal attention over len tokens
    for n in (1, 9, 23):
        o, l = att.decode_attention(q[None, :, n - 1], cache_k, cache_v, [n])
        _close(o[0], full_o[:, n - 1], 1e-11, "decode = last causal row")
        _close(l[0], full_l[:, n - 1], 1e-11, "decode LSE = last causal row")


def pin_chunk_batch_gqa(att):
    # Several packed requests with GQA against torch softmax per row.
    Hq, Hkv, S, D = 4, 2, 40, 8
    prefix = [0, 17, 30]
    chunk = [5, 1, 10]
    B = 3
    total = sum(chunk)
    q = _rand((total, Hq, D), 40)
    k = _rand((B, Hkv, S, D), 41)
    v = _rand((B, Hkv, S, D), 42)
    out, lse = att.chunk_prefill_attention(q, k, v, prefix, chunk)
    p = 0
    for b in range(B):
        for i in range(chunk[b]):
            n = prefix[b] + i + 1
            ro, rl = _torch_reference(q[p][None], k[b:b + 1], v[b:b + 1], [n], 1 / math.sqrt(D))
            _close(out[p], ro[0], 1e-11, "packed chunk O")
            _close(lse[p], rl[0], 1e-11, "packed chunk LSE")
            p += 1


# ---- invariants -----------------------------------------------------------------------------

def pin_split_invariance(att):
    B, Hq, Hkv, S, D = 1, 2, 1, 50, 16
    q = _rand((B, Hq, D), 50, 3.0)
    k = _rand((B, Hkv, S, D), 51)
    v = _rand((B, Hkv, S, D), 52)
    n = 47
    full_o, full_l = att.decode_attention(q, k, v, [n])
    for cuts in ([20], [1, 2, 46], [10, 20, 30, 40], [0, 47]):
        bounds = [0] + cuts + [n]
        outs, lses = [], []
        for a, c in zip(bounds[:-1], bounds[1:]):
            o, l = att.decode_attention(q, k[:, :, a:], v[:, :, a:], [c - a])
            outs.append(o)
            lses.append(l)
        for h in range(Hq):
            mo, ml = formulations.merge_partials([o[0, h] for o in outs],
                                                 [float(l[0, h]) for l in lses])
            _close(mo, full_o[0, h], 1e-12, f"split {cuts} O")
            _close(ml, full_l[0, h], 1e-12, f"split {cuts} LSE")


def pin_permutation_invariance(att):
    B, Hq, Hkv, S, D = 1, 2, 1, 30, 8
    q = _rand((B, Hq, D), 60)
    k = _rand((B, Hkv, S, D), 61)
    v = _rand((B, Hkv, S, D), 62)
    perm = np.random.default_rng(63).permutation(S)
    o1, l1 = att.decode_attention(q, k, v, [S])
    o2, l2 = att.decode_attention(q, k[:, :, perm], v[:, :, perm], [S])
    _close(o1, o2, 1e-12, "permuted O")
    _close(l1, l2, 1e-12, "permuted LSE")


def pin_page_formulations(att):
    B, Hq, Hkv, S, D = 1, 3, 1, 301, 16
    q = _rand((B, Hq, D), 70, 2.0)
    k = _rand((B, Hkv, S, D), 71)
    v = _rand((B, Hkv, S, D), 72)
    n = 289
    out, lse = att.decode_attention(q, k, v, [n])
    scale = 1.0 / math.sqrt(D)
    for h in range(Hq):
        for block in (1, 7, 64, 256, 1000):
            o, l = formulations.online_softmax_row(q[0, h], k[0, 0], v[0, 0], n, scale, block)
            _close(o, out[0, h], 1e-12, f"online block {block} O")
            _close(l, lse[0, h], 1e-12, f"online block {block} LSE")
        for chunks in (1, 2, 3, 8, 289, 400):
            o, l = formulations.split_merge_row(q[0, h], k[0, 0], v[0, 0], n, scale, chunks)
            _close(o, out[0, h], 1e-12, f"split-merge {chunks} O")
            _close(l, lse[0, h], 1e-12, f"split-merge {chunks} LSE")


def pin_bf16_widening(att):
    # bf16 bit patterns must widen to exactly the values torch gives them.
    x = torch.randn(1000, dtype=torch.float32).to(torch.bfloat16)
    bits = x.view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(att.widen(bits), x.to(torch.float64).numpy()), "bf16 widening"
    special = torch.tensor([0.0, -0.0, 1e38, -1e-38, float("inf")], dtype=torch.bfloat16)
    sb = special.view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(att.widen(sb), special.to(torch.float64).numpy()), "bf16 specials"


def _paged_case(seed, B, Hkv, psz, lens, pages_per_seq, D=8, Hq=None):
    """A contiguous cache and the same keys scattered over shuffled physical pages; unused page
    slots hold NaN, and block-table entries past a sequence's pages hold -1."""
    Hq = Hq or 2 * Hkv
    rng = np.random.default_rng(seed)
    cap = pages_per_seq * psz
    q = _rand((B, Hq, D), seed + 1, 2.0)
    k = _rand((B, Hkv, cap, D), seed + 2)
    v = _rand((B, Hkv, cap, D), seed + 3)
    npages = B * pages_per_seq + 3
    phys = rng.permutation(npages)
    kp = np.full((npages, Hkv, psz, D), np.nan)
    vp = np.full((npages, Hkv, psz, D), np.nan)
    table = [[-1] * pages_per_seq for _ in range(B)]
    i = 0
    for b in range(B):
        used = -(-max(0, min(lens[b], cap)) // psz)
        for j in range(used):
            pg = int(phys[i])
            i += 1
            table[b][j] = pg
            kp[pg] = k[b, :, j * psz:(j + 1) * psz]
            vp[pg] = v[b, :, j * psz:(j + 1) * psz]
    return q, k, v, kp, vp, table


def pin_paged_equals_contiguous(att):
    # the paged form is the contiguous definition over the gathered keys: any wrong page or row
    # index reads another page (or a NaN slot) and changes the result
    for seed, psz, lens in ((80, 1, [5, 0, 3]), (81, 3, [7, 9, 1]), (82, 16, [33, 16, 0, 47])):
        B = len(lens)
        pps = max(1, -(-max(lens) // psz))
        q, k, v, kp, vp, table = _paged_case(seed, B, 2, psz, lens, pps)
        o1, l1 = att.decode_attention(q, k, v, lens)
        o2, l2 = att.decode_attention_paged(q, kp, vp, table, lens)
        _close(o2, o1, 1e-12, f"paged psz {psz} O")
        _close(l2, l1, 1e-12, f"paged psz {psz} LSE")


def pin_paged_swapped_pages(att):
    # page size 2, a 4-key sequence stored as [keys 2-3 | keys 0-1]; the first key dominates, so
    # the output is v_0 exactly when (and only when) page 0 of the sequence is read as keys 0-1
    D = 4
    keys = np.zeros((4, D))
    keys[0] = 40.0
    vals = np.arange(4 * D, dtype=np.float64).reshape(4, D)
    q = np.ones((1, 1, D))
    kp = np.stack([keys[2:4], keys[0:2]])[:, None]   # [2 pages, 1 head, 2 rows, D]
    vp = np.stack([vals[2:4], vals[0:2]])[:, None]
    o, l = att.decode_attention_paged(q, kp, vp, [[1, 0]], [4])
    _close(o[0, 0], vals[0], 1e-12, "dominant first key from the second physical page")
    s0 = 40.0 * D / math.sqrt(D)
    _close(l[0, 0], s0 + math.log1p(3 * math.exp(-s0)), 1e-12, "LSE of one dominant key")



# ---- FP8 (E4M3) cache -----------------------------------------------------------------------

def pin_e4m3_closed_forms(att):
    # values fixed by the E4M3 definition: zeros, the subnormal step 2^-9, the smallest normal
    # 2^-6, one, the largest finite 448, the NaN codes
    cases = {0x00: 0.0, 0x80: -0.0, 0x01: 2.0 ** -9, 0x07: 7 * 2.0 ** -9, 0x08: 2.0 ** -6,
             0x30: 0.5, 0x38: 1.0, 0x3F: 1.875, 0x40: 2.0, 0x7E: 448.0, 0xFE: -448.0,
             0xB8: -1.0, 0x5A: 20.0}
    for code, want in cases.items():
        got = att.e4m3_value(code)
        assert got == want and math.copysign(1, got) == math.copysign(1, want), (hex(code), got)
    assert math.isnan(att.e4m3_value(0x7F)) and math.isnan(att.e4m3_value(0xFF))
    vals = [att.e4m3_value(c) for c in range(0x7F)]
    assert all(a < b for a, b in zip(vals, vals[1:])), "positive codes are ordered"


def pin_e4m3_torch(att):
    # every code against torch's float8_e4m3fn decoding (a library routine)
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = att.dequant_e4m3(codes, 1.0)
    same = (got == ref) | (np.isnan(got) & np.isnan(ref))
    assert same.all(), f"codes {np.nonzero(~same)[0][:8]}"
    assert np.array_equal(att.dequant_e4m3(codes[:0x7F], 0.375), ref[:0x7F] * 0.375)


def _fp8_codes(shape, seed, lo=0x00, hi=0x7E):
    rng = np.random.default_rng(seed)
    c = rng.integers(lo, hi + 1, size=shape).astype(np.uint8)
    return c | (rng.integers(0, 2, size=shape).astype(np.uint8) << 7)   # random signs


def pin_fp8_torch_softmax(att):
    # the whole FP8 path against torch: codes decoded by torch, scores / softmax / logsumexp by
    # torch in float64
    B, Hq, Hkv, S, D = 2, 8, 2, 29, 16
    q = _rand((B, Hq, D), 60)
    kc = _fp8_codes((B, Hkv, S, D), 61, hi=0x50)
    vc = _fp8_codes((B, Hkv, S, D), 62)
    ks, vs = 0.0625, 0.75
    lens = [29, 11]
    out, lse = att.decode_attention_fp8(q, kc, vc, ks, vs, lens)
    tk = torch.from_numpy(kc).view(torch.float8_e4m3fn).to(torch.float64).numpy() * ks
    tv = torch.from_numpy(vc).view(torch.float8_e4m3fn).to(torch.float64).numpy() * vs
    ro, rl = _torch_reference(q, tk, tv, lens, 1.0 / math.sqrt(D))
    _close(out, ro, 1e-11, "fp8 torch O")
    _close(lse, rl, 1e-11, "fp8 torch LSE")


def pin_fp8_scale_laws(att):
    # v_scale multiplies O and leaves LSE alone; k_scale acts exactly like scaling q
    B, Hq, Hkv, S, D = 2, 4, 1, 17, 8
    q = _rand((B, Hq, D), 63)
    kc = _fp8_codes((B, Hkv, S, D), 64, hi=0x48)
    vc = _fp8_codes((B, Hkv, S, D), 65)
    lens = [17, 6]
    o1, l1 = att.decode_attention_fp8(q, kc, vc, 0.5, 1.0, lens)
    o2, l2 = att.decode_attention_fp8(q, kc, vc, 0.5, 4.0, lens)
    _close(o2, 4.0 * o1, 1e-12, "v_scale scales O")
    _close(l2, l1, 1e-12, "v_scale leaves LSE")
    o3, l3 = att.decode_attention_fp8(q * 0.5, kc, vc, 1.0, 1.0, lens)
    _close(o3, o1, 1e-12, "k_scale is a scale of the scores")
    _close(l3, l1, 1e-12, "k_scale is a scale of the scores (LSE)")


def pin_fp8_one_hot(att):
    # key 3 holds code 0x7E (448) in every element, the others 0x00: with q = 1 it dominates
    # and O is its V row, v_scale times the E4M3 values of that row's codes
    S, D = 6, 4
    kc = np.zeros((1, 1, S, D), dtype=np.uint8)
    kc[0, 0, 3] = 0x7E
    vc = np.zeros((1, 1, S, D), dtype=np.uint8)
    vc[0, 0, 3] = [0x38, 0x40, 0xB8, 0x01]          # 1, 2, -1, 2^-9
    vc[0, 0, 0] = 0x7E
    q = np.ones((1, 1, D))
    out, lse = att.decode_attention_fp8(q, kc, vc, 1.0, 3.0, [S])
    _close(out[0, 0], 3.0 * np.array([1.0, 2.0, -1.0, 2.0 ** -9]), 1e-12, "fp8 one-hot O")
    s3 = 448.0 * D / math.sqrt(D)
    _close(lse[0, 0], s3 + math.log1p((S - 1) * math.exp(-s3)), 1e-12, "fp8 one-hot LSE")


def pin_fp8_paged(att):
    # the paged FP8 form is the contiguous FP8 form over the same codes
    B, Hkv, psz, D = 2, 2, 4, 8
    lens = [9, 4]
    pps = 3
    kc = _fp8_codes((B, Hkv, pps * psz, D), 66, hi=0x48)
    vc = _fp8_codes((B, Hkv, pps * psz, D), 67)
    q = _rand((B, 2 * Hkv, D), 68)
    order = np.random.default_rng(69).permutation(B * pps)
    kp = np.zeros((B * pps + 1, Hkv, psz, D), dtype=np.uint8)
    vp = np.zeros_like(kp)
    table = [[0] * pps for _ in range(B)]
    for b in range(B):
        for j in range(pps):
            pg = int(order[b * pps + j])
            table[b][j] = pg
            kp[pg] = kc[b, :, j * psz:(j + 1) * psz]
            vp[pg] = vc[b, :, j * psz:(j + 1) * psz]
    o1, l1 = att.decode_attention_fp8(q, kc, vc, 0.25, 2.0, lens)
    o2, l2 = att.decode_attention_paged_fp8(q, kp, vp, 0.25, 2.0, table, lens)
    _close(o2, o1, 1e-12, "paged fp8 O")
    _close(l2, l1, 1e-12, "paged fp8 LSE")



def pin_fp8_rows_match_full(att):
    # the row-sampled form (used at full size, one (sequence, KV head) slab dequantized at a
    # time) equals the full computation at those rows
    B, Hq, Hkv, S, D = 3, 8, 2, 21, 16
    q = _rand((B, Hq, D), 70)
    kc = _fp8_codes((B, Hkv, S, D), 71, hi=0x48)
    vc = _fp8_codes((B, Hkv, S, D), 72)
    lens = [21, 0, 9]
    o, l = att.decode_attention_fp8(q, kc, vc, 0.125, 3.0, lens)
    rows = [(0, 5), (2, 0), (2, 7), (1, 3)]
    o2, l2 = att.decode_attention_fp8(q, kc, vc, 0.125, 3.0, lens, rows=rows)
    for b, h in rows:
        _close(o2[b, h], o[b, h], 1e-12, f"fp8 row ({b}, {h}) O")
        _close(l2[b, h], l[b, h], 1e-12, f"fp8 row ({b}, {h}) LSE")
    assert np.isnan(o2[0, 0]).all(), "rows not asked for stay NaN"

ALL_PINS = [
    pin_golden_decode, pin_golden_chunk, pin_zero_query_is_mean, pin_single_key,
    pin_two_keys_sigmoid, pin_one_hot, pin_equal_scores, pin_empty_and_clamp,
    pin_torch_softmax, pin_chunk_equals_full_causal, pin_chunk_batch_gqa,
    pin_split_invariance, pin_permutation_invariance, pin_page_formulations,
    pin_bf16_widening, pin_paged_equals_contiguous, pin_paged_swapped_pages,
    pin_e4m3_closed_forms, pin_e4m3_torch, pin_fp8_torch_softmax, pin_fp8_scale_laws,
    pin_fp8_one_hot, pin_fp8_paged, pin_fp8_rows_match_full,
]
