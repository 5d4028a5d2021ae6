"""Second and third float64 formulations of decode attention, used only to pin the oracle.

TEST INFRASTRUCTURE ONLY (see ``oracle/attention.py``). These follow the pages' own
algorithms step by step, in float64, so that the plain definition in ``attention.py`` can be
checked against independently written arithmetic:

* ``online_softmax_row``: the sequential block loop of the ChunkedPrefill page
  ("大语言模型长序列推理优化：ChunkedPrefill与FlashDecoding技术解析", §3.1 "分块并行计算原理"):
  a running maximum, the accumulated output and the running sum are both rescaled by
  exp(old max - new max) whenever a block raises the maximum; the block's exp(s - new max)
  weights are then added; the output is divided by the sum at the end.
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


def online_softmax_row(q: np.ndarray, keys: np.ndarray, values: np.ndarray, n: int,
                       scale: float, block_size: int) -> Tuple[np.ndarray, float]:
    """Sequential online softmax over blocks of ``block_size`` keys (float64 inputs)."""
    D = q.shape[0]
    global_out = np.zeros(D, dtype=np.float64)
    global_max = -math.inf
    global_sum = 0.0
    for start in range(0, n, block_size):
        stop = min(start + block_size, n)
        scores = (keys[start:stop] @ q) * scale
        block_max = scores.max()
        new_max = max(global_max, block_max)
        # exp(-inf - finite) = 0 rescales the still-empty accumulators; the page's
        # exp(global_max - new_max) would be exp(-inf - (-inf)) = NaN only if a block were
        # empty, which the loop bounds exclude.
        exp_diff = math.exp(global_max - new_max) if global_max != -math.inf else 0.0
        global_out *= exp_diff
        global_sum *= exp_diff
        exp_scores = np.exp(scores - new_max)
        global_out += exp_scores @ values[start:stop]
        global_sum += exp_scores.sum()
        global_max = new_max
    if n <= 0:
        return np.zeros(D, dtype=np.float64), -math.inf
    return global_out / global_sum, global_max + math.log(global_sum)


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
