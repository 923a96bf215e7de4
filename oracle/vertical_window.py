"""Oracle of the vertical-line / local-window selector.  TEST INFRASTRUCTURE,
under the same import rule as the rest of ``oracle``.

HyQuant (abstract in the body of the page titled "LampAttention: Look-Ahead
Mixed-Precision FlashAttention for Dedicated Accelerators") keeps full
precision for the keys that many queries attend to -- vertical lines of the
attention map -- and for a sliding window beside the diagonal, and picks them
by a cheap signal of the attention pattern.  The abstract gives no formula;
this is the plainest block-level reading, on the same FP16 budget as the
ThriftAttention selector so the two can be compared at equal rho:

  s(i, j)   the pooled block scores of ``oracle.pooled_scores`` (FP32 values);
  v_j       sum over valid rows i of softmax over the row's valid j' of s(i, j'),
            taken at j: the pooled attention mass key block j receives (FP64);
  rank      columns by v descending, ties to the lower j;
  order     window pairs (i - W < j <= i with the causal mask, |i - j| < W
            without) first, then by the column's rank, then by s(i, j)
            descending, then by the lower i; the first k = ceil(rho * #valid - 1e-9)
            pairs are kept.

Plain numpy: a loop over rows for the softmax and one lexicographic sort of
all valid pairs per (batch, query head).
"""
from __future__ import annotations

import numpy as np


def column_signal(scores: np.ndarray, causal: bool) -> np.ndarray:
    """v_j for one head: scores [nb, nb] (FP32, NaN or anything above the
    diagonal ignored when causal) -> float64 [nb]."""
    s = np.asarray(scores, np.float64)
    nb = s.shape[0]
    v = np.zeros(nb, np.float64)
    for i in range(nb):
        row = s[i, :i + 1] if causal else s[i, :]
        e = np.exp(row - row.max())
        v[:row.size] += e / e.sum()
    return v


def column_ranks(v: np.ndarray) -> np.ndarray:
    """Rank of every column: 0 for the largest v, ties to the lower index."""
    order = sorted(range(v.size), key=lambda j: (-v[j], j))
    rank = np.empty(v.size, np.int64)
    rank[order] = np.arange(v.size)
    return rank


def in_window(i, j, window: int, causal: bool):
    if causal:
        return (j <= i) & (j > i - window)
    return np.abs(i - j) < window


def select_head(scores: np.ndarray, causal: bool, rho: float, window: int, budget) -> np.ndarray:
    """Mask [nb, nb] (u8) of one head from its pooled scores."""
    nb = scores.shape[0]
    ii, jj = np.meshgrid(np.arange(nb), np.arange(nb), indexing="ij")
    valid = (jj <= ii) if causal else np.ones((nb, nb), bool)
    i, j = ii[valid], jj[valid]
    sc = np.asarray(scores, np.float64)[valid]
    rank = column_ranks(column_signal(scores, causal))
    # np.lexsort sorts by the last key first: window, then rank, score, row.
    order = np.lexsort((i, -sc, rank[j], ~in_window(i, j, window, causal)))
    k = budget(rho, int(valid.sum()))
    mask = np.zeros((nb, nb), np.uint8)
    mask[i[order[:k]], j[order[:k]]] = 1
    return mask
