"""Pins of the vertical-line / local-window selector's oracle (no GPU).

The selector (after HyQuant, whose abstract stands on the page titled
"LampAttention: Look-Ahead Mixed-Precision FlashAttention for Dedicated
Accelerators") keeps the local window first, then whole key-block columns by
the pooled attention mass they receive.  Each test below ties one part of the
oracle to a closed form, a library routine or a structural fact: the softmax
axis (a transposed softmax fails the row-independent closed form), the
causal range of the column sums (the harmonic tail), the rank direction (a
sink column comes first), the score direction and tie order inside a column,
the window band, the budget, the prefix property and the GQA head mapping.
"""
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from oracle import vertical_window as vw


def _f16(x):
    return np.asarray(x, np.float64).astype(np.float16)


def _band(nb, window, causal):
    m = np.zeros((nb, nb), np.uint8)
    for i in range(nb):
        for j in range(nb):
            if causal and i - window < j <= i:
                m[i, j] = 1
            if not causal and abs(i - j) < window:
                m[i, j] = 1
    return m


# ---------------------------------------------------------------- signal -----
def test_column_signal_of_row_independent_scores_is_scaled_softmax():
    """s(i, j) = a_j for every row: each row's softmax is softmax(a), so
    v = nb * softmax(a).  A softmax over the wrong axis gives v = 1."""
    rng = np.random.default_rng(0)
    nb = 9
    a = rng.standard_normal(nb) * 3
    s = np.tile(a, (nb, 1)).astype(np.float32)
    e = np.exp(a.astype(np.float32).astype(np.float64) - a.max())
    assert np.allclose(vw.column_signal(s, False), nb * e / e.sum(), rtol=1e-13, atol=0)


def test_causal_column_signal_of_equal_scores_is_the_harmonic_tail():
    """Equal scores, causal: row i spreads 1/(i+1) over columns 0..i, so
    v_j = sum_{i=j}^{nb-1} 1/(i+1)."""
    nb = 12
    v = vw.column_signal(np.zeros((nb, nb), np.float32), True)
    expect = [float(sum(Fraction(1, i + 1) for i in range(j, nb))) for j in range(nb)]
    assert np.allclose(v, expect, rtol=1e-14, atol=0)


@pytest.mark.parametrize("causal", [True, False])
def test_column_signal_matches_torch_softmax_and_conserves_mass(causal):
    rng = np.random.default_rng(1)
    nb = 17
    s = (rng.standard_normal((nb, nb)) * 4).astype(np.float32)
    v = vw.column_signal(s, causal)
    t = torch.from_numpy(s.astype(np.float64))
    if causal:
        t = t.masked_fill(torch.triu(torch.ones(nb, nb, dtype=torch.bool), 1), float("-inf"))
    assert np.allclose(v, torch.softmax(t, dim=-1).sum(0).numpy(), rtol=1e-12, atol=1e-15)
    assert abs(v.sum() - nb) < 1e-12                 # every valid row carries mass 1
    # a constant added to a row changes none of that row's softmax
    shift = (rng.standard_normal((nb, 1)) * 10).astype(np.float32)
    s2 = (s.astype(np.float64) + shift).astype(np.float32)
    assert np.allclose(vw.column_signal(s2, causal), v, rtol=1e-5, atol=1e-6)


def test_column_ranks_descending_with_ties_to_lower_index():
    v = np.array([0.5, 2.0, 0.5, 3.0, 2.0])
    assert list(vw.column_ranks(v)) == [3, 1, 4, 0, 2]


# ---------------------------------------------------------------- selection --
@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("window", [1, 2, 3])
def test_budget_of_the_window_size_selects_exactly_the_band(causal, window):
    rng = np.random.default_rng(window)
    nb = 10
    s = (rng.standard_normal((nb, nb)) * 3).astype(np.float32)
    band = _band(nb, window, causal)
    valid = nb * (nb + 1) // 2 if causal else nb * nb
    m = vw.select_head(s, causal, band.sum() / valid, window, oracle.budget)
    assert np.array_equal(m, band)


def _sink_inputs(nb, blk, D, sink_cols, rising=False):
    """Q rows all equal to (r+1)/4 * ones in query block r when `rising`, else
    ones; K rows of block c equal to 4 * ones for the head's sink column c,
    zero elsewhere.  One K head per sink column."""
    N = nb * blk
    q = np.ones((N, D))
    if rising:
        q *= (np.arange(N) // blk + 1)[:, None] / 4
    Q = _f16(np.broadcast_to(q, (1, len(sink_cols), N, D)))
    K = np.zeros((1, len(sink_cols), N, D))
    for h, c in enumerate(sink_cols):
        K[0, h, c * blk:(c + 1) * blk] = 4.0
    return Q, _f16(K)


def test_the_sink_column_is_ranked_first():
    nb, blk, D = 8, 16, 16
    Q, K = _sink_inputs(nb, blk, D, [5])
    m = oracle.select_vertical_window(Q, K, blk, False, 0.25, nb / (nb * nb), 0)[0, 0]
    expect = np.zeros((nb, nb), np.uint8)
    expect[:, 5] = 1
    assert np.array_equal(m, expect)


def test_inside_a_column_higher_scores_come_first():
    nb, blk, D = 8, 16, 16
    Q, K = _sink_inputs(nb, blk, D, [2], rising=True)     # s(i, 2) grows with i
    m = oracle.select_vertical_window(Q, K, blk, False, 0.25, 3 / (nb * nb), 0)[0, 0]
    assert sorted(zip(*np.nonzero(m))) == [(5, 2), (6, 2), (7, 2)]


def test_equal_scores_fill_columns_left_to_right_and_rows_top_down():
    """Q = 0: every pooled score is 0.  Causal: the harmonic tail ranks the
    columns 0, 1, 2, ...; inside a column the lower row wins the tie."""
    nb, blk, D = 8, 16, 16
    Q = np.zeros((1, 1, nb * blk, D), np.float16)
    K = _f16(np.random.default_rng(3).standard_normal((1, 1, nb * blk, D)))
    valid = nb * (nb + 1) // 2
    k = nb + 3
    m = oracle.select_vertical_window(Q, K, blk, True, 0.25, k / valid, 0)[0, 0]
    expect = np.zeros((nb, nb), np.uint8)
    expect[:, 0] = 1
    expect[1:4, 1] = 1
    assert np.array_equal(m, expect)


def test_budget_special_cases_and_prefix_property():
    rng = np.random.default_rng(4)
    nb, blk, D = 12, 16, 32
    Q = _f16(rng.standard_normal((1, 2, nb * blk, D)) + rng.standard_normal((1, 2, nb * blk, 1)))
    K = _f16(rng.standard_normal((1, 2, nb * blk, D)))
    valid = nb * (nb + 1) // 2
    assert oracle.select_vertical_window(Q, K, blk, True, 0.25, 0.0, 2).sum() == 0
    full = oracle.select_vertical_window(Q, K, blk, True, 0.25, 1.0, 2)
    assert np.array_equal(full[0, 1], np.tril(np.ones((nb, nb), np.uint8)))
    prev = np.zeros_like(full)
    for rho in [0.02, 0.1, 0.2, 0.35, 0.5, 0.8]:
        m = oracle.select_vertical_window(Q, K, blk, True, 0.25, rho, 2)
        assert np.all(m.reshape(2, -1).sum(1) == oracle.budget(rho, valid))
        assert np.all(m[0][:, np.triu(np.ones((nb, nb), bool), 1)] == 0)
        assert np.all(m >= prev)
        prev = m


def test_each_query_head_reads_its_kv_head():
    nb, blk, D = 8, 16, 16
    Q, K = _sink_inputs(nb, blk, D, [3, 6])                 # kv head 0: column 3, kv head 1: column 6
    Q = np.concatenate([Q, Q], axis=1)                       # 4 query heads, groups of 2
    m = oracle.select_vertical_window(Q, K, blk, False, 0.25, nb / (nb * nb), 0)[0]
    for h, c in enumerate([3, 3, 6, 6]):
        assert np.array_equal(np.nonzero(m[h].any(0))[0], [c]) and m[h][:, c].all()
