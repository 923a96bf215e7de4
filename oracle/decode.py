"""Oracle of one decode step over the prefill's caches.  TEST INFRASTRUCTURE,
under the same import rule as the rest of ``oracle``.

The ThriftAttention page ("ThriftAttention: Selective Mixed Precision for
Long-Context FP4 Attention", abstract and summary) describes prefill only.
Re-using the block-scaled FP4 K/V of prefill as a compressed cache for
decoding is the step TriAttention takes (abstract on the paper page of
arXiv 2611.07256).  The reading of one decode step taken here applies the
ThriftAttention method to a single new query row q per (batch, query head):

  selection  the query row is its own query block: score_j =
             fl32(sm_scale * fl32(q . kmean_j)) over the nb = N / blk key
             blocks, kmean_j the FP32 block mean of K (exact FP64 sum of the
             block's fp16 rows, divided by blk, rounded once: the same means
             as the prefill heuristic), the dot product in FP64 rounded once;
             k = ceil(rho * nb - 1e-9) blocks, the first block (j = 0) and the
             last one (the query's own, j = nb - 1) first, then by score
             descending, ties to the lower j;
  attention  q sits at position N - 1 and attends to all N cached keys; the
             selected key blocks run in FP16 (fp16 q, K, V), all others in
             block-scaled FP4 (q quantised along D like a row of Q, the
             prefill's NVFP4 K and V), with the prefill's online softmax
             (integer running maximum, P pre-scaled by 2^11, l over the
             unquantised P).

The attention is therefore exactly the prefill oracle's output for row N - 1
of a Q whose row N - 1 is q, with the decode selection as the last row of the
block mask; ``attention`` builds that problem and calls ``attention_rows``.
"""
from __future__ import annotations

from types import SimpleNamespace

import numpy as np


def block_means(Kh: np.ndarray, blk: int) -> np.ndarray:
    """FP32 block means of one head's K [N, D] (fp16) -> [nb, D]."""
    N, D = Kh.shape
    sums = Kh.astype(np.float64).reshape(N // blk, blk, D).sum(axis=1)  # exact: fp16 sums fit 53 bits
    return (sums / blk).astype(np.float32)


def scores(qh: np.ndarray, Kh: np.ndarray, blk: int, sm_scale: float) -> np.ndarray:
    """score_j of one head: q [D] fp16, K [N, D] fp16 -> float32 [nb]."""
    km = block_means(Kh, blk).astype(np.float64)
    dot = (km @ qh.astype(np.float64)).astype(np.float32)
    return (np.float64(np.float32(sm_scale)) * dot.astype(np.float64)).astype(np.float32)


def select(q, K, blk, sm_scale, rho, budget):
    """Decode selection: q [B, Hq, D], K [B, Hkv, N, D] (fp16) -> mask
    [B, Hq, nb] (u8, 1 = FP16 block)."""
    B, Hq, _ = q.shape
    group = Hq // K.shape[1]
    nb = K.shape[2] // blk
    mask = np.zeros((B, Hq, nb), np.uint8)
    k = budget(rho, nb)
    for b in range(B):
        for h in range(Hq):
            sc = scores(q[b, h], K[b, h // group], blk, sm_scale)
            forced = (np.arange(nb) == 0) | (np.arange(nb) == nb - 1)
            order = sorted(range(nb), key=lambda j: (not forced[j], -float(sc[j]), j))
            mask[b, h, order[:k]] = 1
    return mask


def attention(q, K, V, mask, blk, sm_scale, heads, p_log2=None):
    """Decode output (float64, before fp16 rounding) for the (b, h) pairs in
    `heads` -> [len(heads), D]; mask [B, Hq, nb] as from ``select``."""
    import oracle
    if p_log2 is None:
        p_log2 = oracle.P_LOG2_DEFAULT
    Hq, D = q.shape[1], q.shape[2]
    group = Hq // K.shape[1]
    N = K.shape[2]
    nb = N // blk
    kv = {}
    out = np.empty((len(heads), D), np.float64)
    for t, (b, h) in enumerate(heads):
        key = (b, h // group)
        if key not in kv:
            Kh = np.ascontiguousarray(K[b, h // group][None, None])
            Vh = np.ascontiguousarray(V[b, h // group][None, None])
            k4, ks = oracle.quantize_rows(Kh)
            v4, vs = oracle.quantize_v(Vh)
            kv[key] = (Kh, Vh, k4, ks, v4, vs)
        Kh, Vh, k4, ks, v4, vs = kv[key]
        Qh = np.zeros((1, 1, N, D), np.float16)
        Qh[0, 0, N - 1] = q[b, h]
        q4, qs = oracle.quantize_rows(Qh)
        qz = SimpleNamespace(q4=q4, qs=qs, k4=k4, ks=ks, v4=v4, vs=vs)
        m = np.zeros((1, 1, nb, nb), np.uint8)
        m[0, 0, nb - 1] = mask[b, h]
        out[t] = oracle.attention_rows(Qh, Kh, Vh, m, [(0, 0, N - 1)], blk, True, sm_scale, qz, p_log2=p_log2)[0]
    return out
