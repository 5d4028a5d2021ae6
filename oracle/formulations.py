"""Second and third float64 formulations of decode attention, used only to pin the oracle.

TEST INFRASTRUCTURE ONLY (see ``oracle/attention.py``). These restate the pages' own
algorithms, in float64 and in code of this project's own, so that the plain definition in
``attention.py`` can be checked against independently written arithmetic:

* ``online_softmax_row``: the block-wise online softmax of the ChunkedPrefill page
  ("大语言模型长序列推理优化：ChunkedPrefill与FlashDecoding技术解析", §3.1 "分块并行计算原理"):
  the keys are visited one block at a time and only a running summary is kept (largest
  score, sum of exponentials, weighted sum of V rows), corrected by exp(old max - new max)
  when a block raises the maximum, and divided out at the end. Written here as a fold of
  per-block summaries.
* ``split_merge_row``: the split-then-merge form of the FlashDecoding page
  ("大模型推理加速FlashDecoding算法原理与多GPU并行解码实战", section
  "FlashDecoding算法原理与标准注意力机制对比" for the per-chunk pass with
  chunk_size = ceil(seq_len / num_chunks), and section "多GPU张量并行扩展下的FlashDecoding实现"
  for the merge). The merge printed there weights each chunk output by exp(m_i - M) times a
  quantity it calls lse_i; that only yields the right answer when the quantity is the chunk's
  plain sum of exponentials l_i (not its logarithm), which is the reading used here.
* ``merge_partials``: the log-sum-exp merge of already-normalised partial results.
"""

from __future__ import annotations

import math
from typing import List, Sequence, Tuple

import numpy as np

__all__ = ["online_softmax_row", "split_merge_row", "merge_partials"]


def _fold(a: Tuple[float, float, np.ndarray],
          b: Tuple[float, float, np.ndarray]) -> Tuple[float, float, np.ndarray]:
    """Combine two softmax states over disjoint key sets.

    A state (m, l, acc) summarises a set of keys by its largest score m, l = sum exp(s - m) and
    acc = sum exp(s - m) v. Both states are brought to the common reference max(m_a, m_b) and
    added; an empty state (l = 0) contributes nothing, whatever its m.
    """
    m_a, l_a, acc_a = a
    m_b, l_b, acc_b = b
    ref = max(m_a, m_b)
    c_a = math.exp(m_a - ref) if l_a > 0.0 else 0.0
    c_b = math.exp(m_b - ref) if l_b > 0.0 else 0.0
    return ref, c_a * l_a + c_b * l_b, c_a * acc_a + c_b * acc_b


def online_softmax_row(q: np.ndarray, keys: np.ndarray, values: np.ndarray, n: int,
                       scale: float, block_size: int) -> Tuple[np.ndarray, float]:
    """One query row over its first n keys, walked in blocks of ``block_size`` keys.

    Each block is reduced on its own to a state (block max, its sum of exponentials, its
    exponential-weighted sum of V rows); the running state absorbs it with ``_fold``, which
    rescales whichever side has the smaller max. After the last block O = acc / l and
    LSE = m + ln l. Float64 inputs.
    """
    D = q.shape[0]
    state = (-math.inf, 0.0, np.zeros(D, dtype=np.float64))
    for lo in range(0, max(n, 0), block_size):
        hi = min(lo + block_size, n)
        s = scale * (keys[lo:hi] @ q)
        m_blk = float(s.max())
        w = np.exp(s - m_blk)
        state = _fold(state, (m_blk, float(w.sum()), w @ values[lo:hi]))
    m, l, acc = state
    if l == 0.0:
        return np.zeros(D, dtype=np.float64), -math.inf
    return acc / l, m + math.log(l)


def split_merge_row(q: np.ndarray, keys: np.ndarray, values: np.ndarray, n: int,
                    scale: float, num_chunks: int) -> Tuple[np.ndarray, float]:
    """Per-chunk softmax, then the exp(m_i - M) * l_i weighted merge (float64 inputs)."""
    D = q.shape[0]
    chunk_size = max(1, -(-n // num_chunks))   # ceil(seq_len / num_chunks)
    outs: List[np.ndarray] = []
    maxes: List[float] = []
    sums: List[float] = []
    for start in range(0, n, chunk_size):
        stop = min(start + chunk_size, n)
        s = (keys[start:stop] @ q) * scale
        m = s.max()
        p = np.exp(s - m)
        l = p.sum()
        outs.append((p / l) @ values[start:stop])   # softmax within the chunk, then ·V
        maxes.append(m)
        sums.append(l)
    if not outs:
        return np.zeros(D, dtype=np.float64), -math.inf
    M = max(maxes)
    num = np.zeros(D, dtype=np.float64)
    den = 0.0
    for o, m, l in zip(outs, maxes, sums):
        w = math.exp(m - M) * l
        num += o * w
        den += w
    return num / den, M + math.log(den)


def merge_partials(outs: Sequence[np.ndarray], lses: Sequence[float]) -> Tuple[np.ndarray, float]:
    """Merge normalised partials (O_s, LSE_s): weights exp(LSE_s - max LSE); -inf parts drop."""
    finite = [i for i, l in enumerate(lses) if l != -math.inf]
    if not finite:
        return np.zeros_like(np.asarray(outs[0], dtype=np.float64)), -math.inf
    M = max(lses[i] for i in finite)
    num = np.zeros_like(np.asarray(outs[0], dtype=np.float64))
    den = 0.0
    for i in finite:
        w = math.exp(lses[i] - M)
        num += np.asarray(outs[i], dtype=np.float64) * w
        den += w
    return num / den, M + math.log(den)
