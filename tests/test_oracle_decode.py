"""Pins of the decode-step oracle (no GPU).

The decode step (one new query row per head over the prefill's caches, the
ThriftAttention method applied to that row) is pinned to: exact sums and a
library mean for the block means, the orientation of the score, exhaustive
search for the selection on tiny inputs, the budget's special cases and the
GQA head mapping, exact softmax attention at rho = 1, an independent pure-FP4
loop at rho = 0, constant values, and the prefill oracle's own last row.
"""
import itertools

import numpy as np
import pytest
import torch

import oracle
import synth
from oracle import decode


def _f16(x):
    return np.asarray(x, np.float64).astype(np.float16)


def _case(w):
    Q, K, V = synth.generate(w)
    q = np.ascontiguousarray(Q[:, :, -1])                      # the query of the last position
    return Q, K, V, q


# ---------------------------------------------------------------- selection --
def test_block_means_are_exact_and_match_torch_mean():
    rng = np.random.default_rng(0)
    blk, D = 16, 32
    K = _f16(rng.standard_normal((4 * blk, D)) * 3)
    ref = torch.from_numpy(K.astype(np.float64)).reshape(4, blk, D).mean(1).numpy().astype(np.float32)
    assert np.array_equal(decode.block_means(K, blk), ref)
    Kc = np.repeat(_f16(rng.standard_normal((4, D))), blk, axis=0)   # constant blocks: the mean is the row
    assert np.array_equal(decode.block_means(Kc, blk), Kc[::blk].astype(np.float32))


def test_score_is_q_dot_the_block_mean_times_sm_scale():
    rng = np.random.default_rng(1)
    blk, D, nb = 16, 32, 5
    K = _f16(rng.standard_normal((nb * blk, D)))
    km = decode.block_means(K, blk)
    for d in (0, 7, 31):
        q = np.zeros(D, np.float16)
        q[d] = 2.0
        expect = (np.float64(np.float32(0.125)) * (2.0 * km[:, d].astype(np.float64))).astype(np.float32)
        assert np.array_equal(decode.scores(q, K, blk, 0.125), expect)


def _brute(sc, rho):
    nb = sc.size
    k = oracle.budget(rho, nb)
    best, best_key = None, None
    for sub in itertools.combinations(range(nb), k):
        forced = sum(1 for j in sub if j in (0, nb - 1))
        key = (forced, sorted((float(sc[j]) for j in sub), reverse=True), [-j for j in sub])
        if best_key is None or key > best_key:
            best, best_key = sub, key
    m = np.zeros(nb, np.uint8)
    m[list(best)] = 1
    return m


@pytest.mark.parametrize("rho,seed", [(0.2, 0), (0.5, 1), (0.7, 2), (0.4, 3)])
def test_selection_matches_exhaustive_search(rho, seed):
    rng = np.random.default_rng(seed)
    nb, blk, D = 7, 16, 16
    K = _f16(rng.standard_normal((1, 1, nb * blk, D)) + rng.standard_normal((1, 1, nb * blk, 1)))
    q = _f16(rng.standard_normal((1, 1, D)))
    sc = decode.scores(q[0, 0], K[0, 0], blk, 0.25)
    assert np.array_equal(decode.select(q, K, blk, 0.25, rho, oracle.budget)[0, 0], _brute(sc, rho))


def test_selection_special_cases_prefix_and_kv_heads():
    w = synth.GQA_N32K.with_(N=2048, Hq=4, Hkv=2)
    Q, K, V, q = _case(w)
    nb = w.N // w.blk
    sel = lambda rho: decode.select(q, K, w.blk, w.sm_scale, rho, oracle.budget)
    assert sel(0.0).sum() == 0
    assert np.all(sel(1.0) == 1)
    prev = sel(0.0)
    for rho in (0.1, 0.2, 0.5, 0.9):
        m = sel(rho)
        assert np.all(m.sum(-1) == oracle.budget(rho, nb))
        assert np.all(m[..., 0] == 1) and np.all(m[..., nb - 1] == 1)
        assert np.all(m >= prev)
        prev = m
    m = sel(0.3)
    for h in range(4):
        single = decode.select(q[:, h:h + 1], K[:, h // 2:h // 2 + 1], w.blk, w.sm_scale, 0.3, oracle.budget)
        assert np.array_equal(m[:, h], single[:, 0])


# ---------------------------------------------------------------- attention --
def _exact(q, K, V, sm_scale, heads):
    G = q.shape[1] // K.shape[1]
    out = []
    for b, h in heads:
        s = K[b, h // G].astype(np.float64) @ q[b, h].astype(np.float64) * np.float64(np.float32(sm_scale))
        p = np.exp(s - s.max())
        out.append(p @ V[b, h // G].astype(np.float64) / p.sum())
    return np.array(out)


W_SMALL = synth.GQA_N32K.with_(N=1024, Hq=4, Hkv=2)
HEADS = [(0, 0), (0, 1), (0, 3)]


def test_all_fp16_equals_exact_attention():
    Q, K, V, q = _case(W_SMALL)
    nb = W_SMALL.N // W_SMALL.blk
    o = decode.attention(q, K, V, np.ones((1, 4, nb), np.uint8), W_SMALL.blk, W_SMALL.sm_scale, HEADS)
    ex = _exact(q, K, V, W_SMALL.sm_scale, HEADS)
    assert np.linalg.norm(o - ex) / np.linalg.norm(ex) < 1e-3


def test_all_fp4_equals_the_pure_fp4_loop():
    Q, K, V, q = _case(W_SMALL)
    w = W_SMALL
    nb = w.N // w.blk
    o = decode.attention(q, K, V, np.zeros((1, 4, nb), np.uint8), w.blk, w.sm_scale, HEADS)
    for t, (b, h) in enumerate(HEADS):
        Qh = np.zeros((1, 1, w.N, w.D), np.float16)
        Qh[0, 0, -1] = q[b, h]
        Kh, Vh = K[b:b + 1, h // 2:h // 2 + 1], V[b:b + 1, h // 2:h // 2 + 1]
        o4 = oracle.attention_fp4_rows(Qh, Kh, Vh, [(0, 0, w.N - 1)], w.blk, True, w.sm_scale)[0]
        assert np.abs(o[t] - o4).max() < 1e-3


def test_constant_values_come_back_scaled_by_one_factor():
    """V constant along keys, with values 6 s (s an E4M3 value) that NVFP4
    encodes exactly: every channel is the same weighted sum of P-tilde over
    l, so O_d / v_d is one factor per head (sum P-tilde / sum P; 1 would need
    l over the quantised P, which this reading does not take)."""
    Q, K, V, q = _case(W_SMALL)
    w = W_SMALL
    row = _f16(np.resize([0.75, -1.5, 2.25, -3.0, 3.0, 1.5], w.D))
    Vc = np.broadcast_to(row, V.shape).copy()
    m = decode.select(q, K, w.blk, w.sm_scale, 0.25, oracle.budget)
    o = decode.attention(q, K, Vc, m, w.blk, w.sm_scale, HEADS)
    ratio = o / row.astype(np.float64)
    assert np.abs(ratio - ratio[:, :1]).max() < 1e-12
    assert np.all(np.abs(ratio[:, 0] - 1) < 0.1)


def test_decode_is_the_prefill_row_after_the_cache():
    """q = Q[N - 1] with the prefill mask's last row: the decode output is the
    prefill oracle's output for row N - 1, bit for bit."""
    w = W_SMALL
    Q, K, V, q = _case(w)
    pm = oracle.select(Q, K, w.blk, w.causal, w.sm_scale, 0.2)
    o = decode.attention(q, K, V, pm[:, :, -1], w.blk, w.sm_scale, HEADS)
    rows = [(b, h, w.N - 1) for b, h in HEADS]
    ref = oracle.attention_rows(Q, K, V, pm, rows, w.blk, True, w.sm_scale)
    assert np.array_equal(o, ref)
