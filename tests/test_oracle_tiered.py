"""Pins of the tiered selection (FP16 / NVFP4 / skip) and of skipped pairs in
the row oracle (no GPU).

The tiered selection keeps the method's ranking and cuts it in three (first
k16 FP16, last ks skipped, never a forced or FP16 pair).  Its pins: sigma = 0
reproduces the C oracle's two-class selection exactly; the class counts; the
skipped pairs are the lowest-ranked non-forced pairs (scores, then the
higher index first); the prefix property in both budgets.  Skipped pairs in
the row oracle: with every kept pair in FP16, the output equals an exact
FP64 softmax over the kept keys only (skipping is removal from the softmax,
not a zero weight inside it).
"""
import numpy as np
import pytest

import oracle
import synth
from oracle import tiered


def _case(**kw):
    w = synth.CAUSAL_MH_N8K.with_(**kw)
    Q, K, V = synth.generate(w)
    return w, Q, K, V


def _valid(nb, causal):
    return np.tril(np.ones((nb, nb), bool)) if causal else np.ones((nb, nb), bool)


@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("rho", [0.0, 0.05, 0.3])
def test_sigma_zero_is_the_method_selection(causal, rho):
    w, Q, K, V = _case(N=1024, Hq=2, Hkv=1, causal=causal)
    m2 = oracle.select_tiered(Q, K, w.blk, causal, w.sm_scale, rho, 0.0)
    assert np.array_equal(m2, oracle.select(Q, K, w.blk, causal, w.sm_scale, rho))


@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("rho,sigma", [(0.05, 0.25), (0.1, 0.5), (0.3, 0.9), (0.0, 1.0), (0.05, 1.0)])
def test_counts_and_the_skipped_pairs_are_the_lowest_ranked(causal, rho, sigma):
    w, Q, K, V = _case(N=1024, Hq=2, Hkv=2, causal=causal)
    nb = w.N // w.blk
    valid = _valid(nb, causal)
    n = int(valid.sum())
    forced = np.zeros((nb, nb), bool)
    forced[np.arange(nb), np.arange(nb)] = True
    forced[:, 0] = True
    forced &= valid
    m = oracle.select_tiered(Q, K, w.blk, causal, w.sm_scale, rho, sigma)
    k16 = oracle.budget(rho, n)
    ks = min(oracle.budget(sigma, n), n - max(k16, int(forced.sum())))
    for h in range(w.Hq):
        mh = m[0, h]
        assert (mh == 1).sum() == k16 and (mh == 2).sum() == ks
        assert not np.any((mh != 0) & ~valid)
        assert not np.any((mh == 2) & forced)
        sc = oracle.pooled_scores(Q[0, h], K[0, h], w.blk, causal, w.sm_scale)
        skipped = mh == 2
        kept = valid & (mh == 0) & ~forced
        if skipped.any() and kept.any():
            lo_kept, hi_skip = sc[kept].min(), sc[skipped].max()
            assert hi_skip <= lo_kept
            if hi_skip == lo_kept:  # equal scores: the higher linear index is skipped first
                idx = np.arange(nb * nb).reshape(nb, nb)
                assert idx[skipped & (sc == hi_skip)].min() > idx[kept & (sc == lo_kept)].max()


def test_forced_pairs_survive_a_full_skip_budget_and_budgets_nest():
    w, Q, K, V = _case(N=1024, Hq=1, Hkv=1)
    nb = w.N // w.blk
    valid = _valid(nb, True)
    m = oracle.select_tiered(Q, K, w.blk, True, w.sm_scale, 0.02, 1.0)[0, 0]
    forced = np.zeros((nb, nb), bool)
    forced[np.arange(nb), np.arange(nb)] = True
    forced[:, 0] = True
    assert np.all(m[forced & valid] != 2)
    assert np.all((m == 2) == (valid & ~forced & (m != 1)))
    prev = None
    for sigma in [0.0, 0.1, 0.3, 0.6, 0.9]:
        cur = oracle.select_tiered(Q, K, w.blk, True, w.sm_scale, 0.05, sigma)[0, 0] == 2
        if prev is not None:
            assert np.all(cur >= prev)
        prev = cur


def test_a_skipped_pair_is_absent_from_the_softmax():
    """Kept pairs all FP16, some pairs skipped: the row oracle equals the exact
    FP64 softmax over the kept keys only (within the FP16 path's 1e-3)."""
    w, Q, K, V = _case(N=512, Hq=2, Hkv=1)
    nb = w.N // w.blk
    rng = np.random.default_rng(3)
    mask = np.ones((1, w.Hq, nb, nb), np.uint8)
    skip = rng.random((w.Hq, nb, nb)) < 0.4
    skip[:, np.arange(nb), np.arange(nb)] = False          # every row keeps its diagonal block
    mask[0][skip] = 2
    rows = oracle.all_rows(1, w.Hq, w.N)
    o = oracle.attention_rows(Q, K, V, mask, rows, w.blk, True, w.sm_scale)
    ex = np.empty_like(o)
    for t, (b, h, r) in enumerate(rows):
        keys = np.arange(r + 1)
        keys = keys[mask[0, h, r // w.blk, keys // w.blk] != 2]
        s = K[0, 0, keys].astype(np.float64) @ Q[0, h, r].astype(np.float64) * np.float64(np.float32(w.sm_scale))
        p = np.exp(s - s.max())
        ex[t] = p @ V[0, 0, keys].astype(np.float64) / p.sum()
    assert np.linalg.norm(o - ex) / np.linalg.norm(ex) < 1e-3


@pytest.mark.parametrize("causal", [True, False])
def test_eight_bit_pairs_come_next_in_rank(causal):
    """With an 8-bit budget: the FP16 pairs are unchanged, the 8-bit pairs are
    the next ones of the ranking (every 8-bit pair's score between the FP16
    cut and the NVFP4 pairs' scores), and skipping spares them."""
    w, Q, K, V = _case(N=1024, Hq=2, Hkv=1, causal=causal)
    nb = w.N // w.blk
    n = int(_valid(nb, causal).sum())
    for rho, rho8, sigma in [(0.05, 0.1, 0.0), (0.05, 0.2, 0.5), (0.0, 0.3, 0.9)]:
        m = oracle.select_tiered(Q, K, w.blk, causal, w.sm_scale, rho, sigma, rho8)
        base = oracle.select_tiered(Q, K, w.blk, causal, w.sm_scale, rho, 0.0)
        assert np.array_equal(m == 1, base == 1)
        for h in range(w.Hq):
            mh = m[0, h]
            assert (mh == 3).sum() == oracle.budget(rho8, n)
            sc = oracle.pooled_scores(Q[0, h], K[0, h // 2], w.blk, causal, w.sm_scale)
            forced = np.zeros((nb, nb), bool)
            forced[np.arange(nb), np.arange(nb)] = True
            forced[:, 0] = True
            free4 = (mh == 0) & ~forced & _valid(nb, causal)
            free8 = (mh == 3) & ~forced
            if free8.any() and free4.any():
                assert sc[free8].min() >= sc[free4].max()


@pytest.mark.parametrize("causal", [True, False])
def test_full_eight_bit_budget_leaves_no_nvfp4_or_skipped_pair(causal):
    """rho8 = 1: k8 = #valid - k16, so every valid pair is FP16 or 8-bit and
    the skip budget is capped at zero whatever sigma asks; rho = 1 leaves no
    room for 8-bit pairs."""
    w, Q, K, V = _case(N=512, Hq=2, Hkv=1, causal=causal)
    nb = w.N // w.blk
    valid = _valid(nb, causal)
    for sigma in (0.0, 0.7):
        m = oracle.select_tiered(Q, K, w.blk, causal, w.sm_scale, 0.05, sigma, 1.0)
        assert np.all(np.isin(m[:, :, valid], (1, 3))) and not np.any(m[:, :, ~valid])
        assert np.array_equal(m == 1, oracle.select_tiered(Q, K, w.blk, causal, w.sm_scale, 0.05, 0.0) == 1)
    m = oracle.select_tiered(Q, K, w.blk, causal, w.sm_scale, 1.0, 0.5, 0.5)
    assert np.all(m[:, :, valid] == 1)
