"""Oracle of the tiered block selection (FP16 / NVFP4 / skip).  TEST
INFRASTRUCTURE, under the same import rule as the rest of ``oracle``.

TriAttention (abstract on the paper page of arXiv 2611.07256) gives each
query-key tile one of several precisions, skipping the interactions that
matter least and lowering the precision of the rest; its per-head boundaries
come from offline calibration, which needs models and data.  The reading
here keeps ThriftAttention's own ranking of block pairs (forced pairs first,
then the pooled score descending, then the lower linear index) and cuts it
in three:

  the first k16 = ceil(rho * #valid - 1e-9) pairs      FP16   (mask 1)
  the next  k8  = min(ceil(rho8 * #valid - 1e-9),
                      #valid - k16) pairs               MXFP8  (mask 3)
  the last  ks  = min(ceil(sigma * #valid - 1e-9),
                      #valid - max(k16 + k8, #forced))  skip   (mask 2)
  the rest                                              NVFP4  (mask 0)

so precision falls with rank, forced, FP16 and 8-bit pairs are never
skipped, and rho8 = sigma = 0 gives the method's two-class mask.  A skipped
pair is absent from the softmax (the row oracle's mask value 2).
"""
from __future__ import annotations

import numpy as np


def select_head(scores: np.ndarray, causal: bool, rho: float, sigma: float, budget, rho8: float = 0.0) -> np.ndarray:
    """Mask [nb, nb] (u8: 1 FP16, 3 MXFP8, 0 NVFP4, 2 skip) of one head from its pooled scores."""
    nb = scores.shape[0]
    ii, jj = np.meshgrid(np.arange(nb), np.arange(nb), indexing="ij")
    valid = (jj <= ii) if causal else np.ones((nb, nb), bool)
    i, j = ii[valid], jj[valid]
    sc = np.asarray(scores, np.float64)[valid]
    forced = (i == j) | (j == 0)
    # np.lexsort sorts by the last key first: forced, then score, then index
    order = np.lexsort((i * nb + j, -sc, ~forced))
    n = int(valid.sum())
    k16 = budget(rho, n)
    k8 = min(budget(rho8, n), n - k16)
    ks = min(budget(sigma, n), n - max(k16 + k8, int(forced.sum())))
    mask = np.zeros((nb, nb), np.uint8)
    mask[i[order[:k16]], j[order[:k16]]] = 1
    mask[i[order[k16:k16 + k8]], j[order[k16:k16 + k8]]] = 3
    if ks > 0:
        mask[i[order[n - ks:]], j[order[n - ks:]]] = 2
    return mask
