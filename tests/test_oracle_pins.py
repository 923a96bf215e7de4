"""Pins of the CPU oracle to facts outside itself (no GPU).

Each test ties one oracle function to a format definition, a library routine,
a closed form, an invariant of the method, or brute force on a tiny input, so
that a plausible slip in the oracle (a dropped term, a wrong sign, a swapped
index, a transposed operand) fails at least one of them.
"""
import itertools
import math

import numpy as np
import pytest
import torch

import oracle
import synth


# ---------------------------------------------------------------- fp16 -------
def test_f16_decode_matches_numpy_for_every_pattern():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = bits.view(np.float16).astype(np.float64)
    got = np.array([oracle.f16_value(int(b)) for b in bits])
    fin = np.isfinite(ref)
    assert np.array_equal(got[fin], ref[fin])
    assert np.array_equal(np.isnan(got), np.isnan(ref))


def test_f16_encode_matches_numpy_rounding():
    rng = np.random.default_rng(1)
    vals = np.concatenate([
        rng.standard_normal(4000) * 10.0 ** rng.integers(-9, 5, 4000),
        # exact midpoints between neighbouring fp16 values (ties to even)
        (np.arange(2000, dtype=np.uint16).view(np.float16).astype(np.float64)
         + np.arange(1, 2001, dtype=np.uint16).view(np.float16).astype(np.float64)) / 2,
        [65504.0, 65519.99, 65520.0, 1e6, 2.0 ** -24, 2.0 ** -25, 3 * 2.0 ** -26, -0.0],
    ])
    for v in vals:
        with np.errstate(over="ignore"):
            ref = int(np.array(v).astype(np.float16).view(np.uint16))
        assert oracle.f16_encode(v) == ref, v


# ---------------------------------------------------------------- E2M1 -------
def _e2m1_from_bits(code):
    """E2M1 value from its fields: sign bit 3, exponent bits 2:1 (bias 1), mantissa bit 0."""
    s, e, m = (code >> 3) & 1, (code >> 1) & 3, code & 1
    mag = (m * 0.5) if e == 0 else (1 + m / 2) * 2.0 ** (e - 1)
    return -mag if s else mag


def test_e2m1_decode_matches_format_fields():
    for c in range(16):
        assert oracle.e2m1_value(c) == _e2m1_from_bits(c)


@pytest.mark.parametrize("v,expect", [
    (0.25, 0.0), (0.75, 1.0), (1.25, 1.0), (1.75, 2.0), (2.5, 2.0), (3.5, 4.0), (5.0, 4.0),
    (0.2500001, 0.5), (4.99, 4.0), (5.01, 6.0), (7.0, 6.0), (1e9, 6.0), (-5.0, -4.0), (-0.75, -1.0),
])
def test_e2m1_round_to_nearest_even_and_saturate(v, expect):
    assert oracle.e2m1_value(oracle.e2m1_encode(v)) == expect


def test_e2m1_keeps_sign_of_values_rounding_to_zero():
    assert oracle.e2m1_encode(-0.1) == 8
    assert oracle.e2m1_encode(0.1) == 0


def test_e2m1_encode_is_nearest_by_brute_force():
    grid = sorted({abs(_e2m1_from_bits(c)) for c in range(8)})
    rng = np.random.default_rng(2)
    for v in rng.uniform(-7, 7, 3000):
        got = abs(oracle.e2m1_value(oracle.e2m1_encode(v)))
        assert abs(abs(v) - got) <= min(abs(abs(v) - g) for g in grid) + 1e-15


# ---------------------------------------------------------------- E4M3 -------
def test_e4m3_decode_matches_torch_float8():
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).double().numpy()
    got = np.array([oracle.e4m3_value(c) for c in range(256)])
    fin = np.isfinite(ref)
    assert np.array_equal(got[fin], ref[fin])
    assert np.array_equal(np.isnan(got), np.isnan(ref))


def test_e4m3_encode_matches_torch_rounding_in_range():
    rng = np.random.default_rng(3)
    finite = np.array([oracle.e4m3_value(c) for c in range(127)])
    mids = (finite[:-1] + finite[1:]) / 2
    vals = np.concatenate([rng.uniform(0, 448, 3000), 2.0 ** rng.uniform(-12, 8.8, 3000), mids, [0.0, 448.0]])
    ref = torch.tensor(vals, dtype=torch.float64).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([oracle.e4m3_encode(v) for v in vals])
    assert np.array_equal(got, ref)


def test_e4m3_saturates_to_448():
    for v in [449.0, 463.9, 500.0, 1e6]:
        assert oracle.e4m3_value(oracle.e4m3_encode(v)) == 448.0


# ---------------------------------------------------------------- NVFP4 -------
def _f16(a):
    return np.asarray(a, np.float64).astype(np.float16)


def test_nvfp4_quant_dequant_is_idempotent():
    rng = np.random.default_rng(4)
    x = _f16(rng.standard_normal((64, 128)) * np.exp(rng.uniform(-6, 6, (64, 1))))
    c1, s1 = oracle.quantize_rows(x)
    y = oracle.dequantize(c1, s1)
    assert np.array_equal(y.astype(np.float16).astype(np.float64), y)  # NVFP4 values are exact in fp16
    c2, s2 = oracle.quantize_rows(_f16(y))
    y2 = oracle.dequantize(c2, s2)
    # Idempotent on the grid wherever the scale is an E4M3 normal (>= 2^-6): the
    # scale's relative rounding error (<= 1/16) keeps amax/scale in the code-7 cell,
    # so the decoded maximum is exactly 6*scale and re-encodes to the same scale.
    normal = np.repeat(s1 >= 8, 16, axis=1)
    assert normal.mean() > 0.5
    assert np.array_equal(y2[normal], y[normal])
    assert np.array_equal(s1[s1 >= 8], s2[s1 >= 8])
    # With a subnormal scale the relative step is coarser and the round trip may move.


def test_nvfp4_group_closed_forms():
    # A group whose amax is 6*s for a representable scale s encodes to scale s and code 7.
    for s in [0.5, 1.125, 3.0, 40.0]:
        x = _f16(np.full((1, 16), 6 * s))
        c, sc = oracle.quantize_rows(x)
        assert oracle.e4m3_value(int(sc[0, 0])) == s
        assert np.all(c == 0x77)
    # Exact tie x/s = 0.75 rounds up to 1.0 (even code), x/s = 1.25 rounds down to 1.0.
    x = _f16([[6.0, 0.75, 1.25, -0.75] + [0.0] * 12])
    c, sc = oracle.quantize_rows(x)
    v = oracle.dequantize(c, sc)[0]
    assert oracle.e4m3_value(int(sc[0, 0])) == 1.0
    assert list(v[:4]) == [6.0, 1.0, 1.0, -1.0]
    # An all-zero group and a group below the smallest scale encode as zeros.
    x = _f16([[0.0] * 16, [1e-4] * 16])
    c, sc = oracle.quantize_rows(x)
    assert np.all(c == 0) and np.all(sc == 0)


def test_nvfp4_groups_are_16_consecutive_elements_with_low_nibble_first():
    x = np.zeros((1, 32), np.float64)
    x[0, 0] = 6.0      # group 0, element 0 -> low nibble of byte 0
    x[0, 17] = -3.0    # group 1, element 1 -> high nibble of byte 8
    c, sc = oracle.quantize_rows(_f16(x))
    assert c[0, 0] == 0x07 and c[0, 8] == 0xF0
    assert oracle.e4m3_value(int(sc[0, 0])) == 1.0 and oracle.e4m3_value(int(sc[0, 1])) == 0.5


def test_v_is_quantised_along_keys():
    rng = np.random.default_rng(5)
    V = _f16(rng.standard_normal((1, 2, 64, 32)))
    c, s = oracle.quantize_v(V)
    ct, st = oracle.quantize_rows(np.ascontiguousarray(np.swapaxes(V, 2, 3)))
    assert np.array_equal(c, ct) and np.array_equal(s, st)


# ---------------------------------------------------------------- selection ---
def _structured_qk(nb, blk, D, a, b):
    """Q block i = a[i] * e0 on every row, K block j = b[j] * e0: mean-q . mean-k = a_i b_j."""
    Q = np.zeros((1, 1, nb * blk, D))
    K = np.zeros((1, 1, nb * blk, D))
    for i in range(nb):
        Q[0, 0, i * blk:(i + 1) * blk, 0] = a[i]
        K[0, 0, i * blk:(i + 1) * blk, 0] = b[i]
    return _f16(Q), _f16(K)


def test_pooled_scores_closed_form_and_orientation():
    nb, blk, D = 4, 16, 32
    a, b = [1, 2, 3, 4], [0.5, -1, 0.25, 2]
    Q, K = _structured_qk(nb, blk, D, a, b)
    sc = oracle.pooled_scores(Q[0, 0], K[0, 0], blk, False, 0.5)
    expect = 0.5 * np.outer(a, b)  # row = query block, column = key block
    assert np.array_equal(sc, expect.astype(np.float32))
    sc_c = oracle.pooled_scores(Q[0, 0], K[0, 0], blk, True, 0.5)
    assert np.all(np.isnan(sc_c[np.triu_indices(nb, 1)]))


def test_pooled_scores_use_block_means():
    # Zero-mean noise inside a block leaves the mean, hence the score, unchanged.
    nb, blk, D = 3, 16, 16
    Q, K = _structured_qk(nb, blk, D, [1, 2, 3], [1, 1, 1])
    noise = np.zeros((1, 1, nb * blk, D))
    noise[0, 0, 0:blk:2, 1] = 0.5
    noise[0, 0, 1:blk:2, 1] = -0.5
    s0 = oracle.pooled_scores(Q[0, 0], K[0, 0], blk, False, 1.0)
    s1 = oracle.pooled_scores(_f16(Q + noise)[0, 0], K[0, 0], blk, False, 1.0)
    assert np.array_equal(s0, s1)


def test_budget_rounding():
    assert oracle.budget(0.05, 256) == 13
    assert oracle.budget(0.05, 8256) == 413
    assert oracle.budget(0.1, 2080) == 208      # 0.1*2080 is 208.00000000000003 in FP64
    assert oracle.budget(0.0, 100) == 0 and oracle.budget(1.0, 100) == 100
    assert oracle.budget(0.01, 32896) == 329


def _brute_select(scores, causal, rho):
    """Exhaustive search: among all subsets of size k, the one that maximises
    (#forced, then the sorted score vector, then prefers lower indices)."""
    nb = scores.shape[0]
    pairs = [(i, j) for i in range(nb) for j in range(nb) if not (causal and j > i)]
    k = oracle.budget(rho, len(pairs))
    best, best_key = None, None
    for sub in itertools.combinations(range(len(pairs)), k):
        chosen = [pairs[t] for t in sub]
        forced = sum(1 for (i, j) in chosen if i == j or j == 0)
        key = (forced, sorted((scores[i, j] for (i, j) in chosen), reverse=True),
               [-(i * nb + j) for (i, j) in sorted(chosen, key=lambda p: p[0] * nb + p[1])])
        if best_key is None or key > best_key:
            best, best_key = chosen, key
    m = np.zeros((nb, nb), np.uint8)
    for (i, j) in best:
        m[i, j] = 1
    return m


@pytest.mark.parametrize("causal,rho,seed", [(True, 0.5, 0), (False, 0.3, 1), (True, 0.2, 2), (False, 0.75, 3)])
def test_selection_matches_exhaustive_search(causal, rho, seed):
    rng = np.random.default_rng(seed)
    nb, blk, D = 4, 16, 16
    Q = _f16(rng.standard_normal((1, 1, nb * blk, D)) + rng.standard_normal((1, 1, nb * blk, 1)))
    K = _f16(rng.standard_normal((1, 1, nb * blk, D)))
    scores = oracle.pooled_scores(Q[0, 0], K[0, 0], blk, causal, 0.25)
    mask = oracle.select(Q, K, blk, causal, 0.25, rho)[0, 0]
    assert np.array_equal(mask, _brute_select(scores, causal, rho))


def test_selection_special_cases_and_invariants():
    w = synth.CAUSAL_MH_N8K.with_(N=1024, Hq=2, Hkv=2)
    Q, K, V = synth.generate(w)
    nb = w.N // w.blk
    m0 = oracle.select(Q, K, w.blk, True, w.sm_scale, 0.0)
    m1 = oracle.select(Q, K, w.blk, True, w.sm_scale, 1.0)
    assert m0.sum() == 0
    assert np.array_equal(m1[0, 0], np.tril(np.ones((nb, nb), np.uint8)))
    prev = m0
    for rho in [0.05, 0.1, 0.3, 0.6]:
        m = oracle.select(Q, K, w.blk, True, w.sm_scale, rho)
        k = oracle.budget(rho, nb * (nb + 1) // 2)
        assert np.all(m.reshape(2, -1).sum(1) == k)
        assert np.all(m[..., np.triu_indices(nb, 1)[0], np.triu_indices(nb, 1)[1]] == 0)
        if k >= 2 * nb - 1:  # every forced pair fits in the budget
            assert np.all(m[..., np.arange(nb), np.arange(nb)] == 1) and np.all(m[..., :, 0] == 1)
        assert np.all(m >= prev)  # a larger budget keeps every earlier pick
        prev = m
    # top-k property of the non-forced picks
    m = oracle.select(Q, K, w.blk, True, w.sm_scale, 0.4)[0, 0]   # budget 55 > 31 forced pairs
    sc = oracle.pooled_scores(Q[0, 0], K[0, 0], w.blk, True, w.sm_scale)
    free = np.tril(np.ones((nb, nb), bool))
    free[np.arange(nb), np.arange(nb)] = False
    free[:, 0] = False
    picked, left = sc[free & (m == 1)], sc[free & (m == 0)]
    assert picked.size and left.size and picked.min() >= left.max()


def test_selection_uses_the_kv_head_of_each_query_head():
    rng = np.random.default_rng(6)
    nb, blk, D = 4, 16, 16
    Q = _f16(rng.standard_normal((1, 4, nb * blk, D)))
    K = _f16(rng.standard_normal((1, 2, nb * blk, D)) + rng.standard_normal((1, 2, nb * blk, 1)) * 2)
    m = oracle.select(Q, K, blk, False, 0.25, 0.4)
    for h in range(4):
        single = oracle.select(Q[:, h:h + 1], K[:, h // 2:h // 2 + 1], blk, False, 0.25, 0.4)
        assert np.array_equal(m[:, h], single[:, 0])


# ---------------------------------------------------------------- attention ---
def _small(w, **kw):
    w = w.with_(**kw)
    Q, K, V = synth.generate(w)
    return w, Q, K, V


def test_exact_attention_matches_torch_sdpa():
    for w in [synth.TINY_NONCAUSAL_D64.with_(N=256), synth.GQA_N32K.with_(N=256, Hq=4, Hkv=2)]:
        Q, K, V = synth.generate(w)
        rows = oracle.all_rows(w.B, w.Hq, w.N)
        got = oracle.exact_rows(Q, K, V, rows, w.causal, w.sm_scale).reshape(w.B, w.Hq, w.N, w.D)
        G = w.Hq // w.Hkv
        t = lambda a: torch.from_numpy(a.astype(np.float64))
        ref = torch.nn.functional.scaled_dot_product_attention(
            t(Q), t(K).repeat_interleave(G, 1), t(V).repeat_interleave(G, 1), is_causal=w.causal,
            scale=w.sm_scale).numpy()
        assert np.abs(got - ref).max() < 1e-12


@pytest.mark.parametrize("w", [synth.TINY_NONCAUSAL_D64.with_(N=512), synth.CAUSAL_MH_N8K.with_(N=512, Hq=2, Hkv=2),
                               synth.GQA_N32K.with_(N=512, Hq=4, Hkv=2, blk=128)])
def test_rho_one_equals_exact_attention(w):
    Q, K, V = synth.generate(w)
    rows = oracle.all_rows(w.B, w.Hq, w.N)
    nb = w.N // w.blk
    mask = np.ones((w.B, w.Hq, nb, nb), np.uint8)
    o = oracle.attention_rows(Q, K, V, mask, rows, w.blk, w.causal, w.sm_scale)
    ex = oracle.exact_rows(Q, K, V, rows, w.causal, w.sm_scale)
    assert np.linalg.norm(o - ex) / np.linalg.norm(ex) < 1e-3


@pytest.mark.parametrize("w", [synth.TINY_NONCAUSAL_D64.with_(N=512), synth.CAUSAL_MH_N8K.with_(N=512, Hq=2, Hkv=2)])
def test_rho_zero_equals_pure_fp4(w):
    Q, K, V = synth.generate(w)
    rows = oracle.all_rows(w.B, w.Hq, w.N)
    nb = w.N // w.blk
    qz = oracle.Quantised(Q, K, V)
    o = oracle.attention_rows(Q, K, V, np.zeros((w.B, w.Hq, nb, nb), np.uint8), rows, w.blk, w.causal,
                              w.sm_scale, qz)
    o4 = oracle.attention_fp4_rows(Q, K, V, rows, w.blk, w.causal, w.sm_scale, qz)
    # Equal except where an NVFP4 scale of P falls into the E4M3 subnormal range
    # (groups far below the running maximum): bounded well under 1e-3 here.
    assert np.abs(o - o4).max() < 1e-3
    assert np.abs(o - o4).mean() < 1e-5


def test_output_does_not_depend_on_merge_order():
    w, Q, K, V = _small(synth.TINY_NONCAUSAL_D64, N=512)
    rows = oracle.all_rows(w.B, w.Hq, w.N)
    mask = oracle.select(Q, K, w.blk, w.causal, w.sm_scale, 0.2)
    qz = oracle.Quantised(Q, K, V)
    base = oracle.attention_rows(Q, K, V, mask, rows, w.blk, w.causal, w.sm_scale, qz)
    rng = np.random.default_rng(8)
    for _ in range(3):
        order = rng.permutation(w.N // w.blk)
        o = oracle.attention_rows(Q, K, V, mask, rows, w.blk, w.causal, w.sm_scale, qz, order=order)
        assert np.abs(o - base).max() < 1e-3
        assert np.abs(o - base).mean() < 1e-5
    # With only FP16 pairs the order enters only through fp16 subnormals of P*2^11
    # (P < 2^-25 of the running maximum) and FP64 rounding.
    ones = np.ones_like(mask)
    a = oracle.attention_rows(Q, K, V, ones, rows, w.blk, w.causal, w.sm_scale, qz)
    b = oracle.attention_rows(Q, K, V, ones, rows, w.blk, w.causal, w.sm_scale, qz, order=order)
    assert np.abs(a - b).max() < 1e-8


@pytest.mark.parametrize("causal", [False, True])
def test_zero_queries_average_the_encoded_values(causal):
    # Q = 0 gives t = 0 for every key, so M = 0 and P = 1 exactly.  FP16 blocks
    # carry P = 1; FP4 blocks carry E2M1(2048/352)*352/2048 = 2112/2048 (scale
    # E4M3(2048/6) = 352, code 6), while l counts every key once.  Keys cut off
    # by the causal edge carry P = 0 and leave the group maximum at 1.
    N, D, blk = 256, 64, 64
    rng = np.random.default_rng(9)
    Q = np.zeros((1, 1, N, D), np.float16)
    K = _f16(rng.standard_normal((1, 1, N, D)))
    V = _f16(rng.standard_normal((1, 1, N, D)))
    nb = N // blk
    mask = (rng.random((1, 1, nb, nb)) < 0.5).astype(np.uint8)
    rows = oracle.all_rows(1, 1, N)
    o = oracle.attention_rows(Q, K, V, mask, rows, blk, causal, 0.125)
    v4 = oracle.dequantize(*oracle.quantize_v(V))[0, 0].T      # [N, D] decoded along keys
    v16 = V[0, 0].astype(np.float64)
    for r in range(N):
        nk = r + 1 if causal else N
        w = np.array([1.0 if mask[0, 0, r // blk, k // blk] else 2112 / 2048 for k in range(nk)])
        vals = np.where(mask[0, 0, r // blk, np.arange(nk) // blk][:, None] == 1, v16[:nk], v4[:nk])
        np.testing.assert_allclose(o[r], (w[:, None] * vals).sum(0) / nk, rtol=0, atol=1e-12)


def test_causal_first_row_returns_first_value():
    w, Q, K, V = _small(synth.CAUSAL_MH_N8K, N=256, Hq=1, Hkv=1)
    nb = w.N // w.blk
    mask = oracle.select(Q, K, w.blk, True, w.sm_scale, 0.05)
    assert mask[0, 0, 0, 0] == 1
    o = oracle.attention_rows(Q, K, V, mask, [(0, 0, 0)], w.blk, True, w.sm_scale)
    # P_0 = 2^(t - ceil t) in (1/2, 1]; its fp16 encoding is within 2^-11 relative.
    np.testing.assert_allclose(o[0], V[0, 0, 0].astype(np.float64), rtol=2 ** -10, atol=0)


def test_dominant_key_is_returned():
    N, D, blk = 128, 64, 64
    rng = np.random.default_rng(10)
    K = _f16(rng.standard_normal((1, 1, N, D)) * 0.1)
    V = _f16(rng.standard_normal((1, 1, N, D)))
    K = K.copy()
    K[0, 0, 77] = _f16(np.ones(D) * 3)                      # every query points at key 77
    Q = _f16(np.broadcast_to(np.ones(D) * 3, (1, 1, N, D)))
    nb = N // blk
    ones = np.ones((1, 1, nb, nb), np.uint8)
    o = oracle.attention_rows(Q, K, V, ones, [(0, 0, 5)], blk, False, 1.0)
    np.testing.assert_allclose(o[0], V[0, 0, 77].astype(np.float64), rtol=1e-3, atol=1e-6)


def test_query_heads_share_their_kv_head():
    w, Q, K, V = _small(synth.GQA_N32K, N=256, Hq=4, Hkv=2, blk=64)
    Q = Q.copy()
    Q[:, 1] = Q[:, 0]           # heads 0,1 share kv head 0; head 2 uses kv head 1
    Q[:, 2] = Q[:, 0]
    nb = w.N // w.blk
    mask = np.zeros((1, 4, nb, nb), np.uint8)
    rows = [(0, 0, 200), (0, 1, 200), (0, 2, 200)]
    o = oracle.attention_rows(Q, K, V, mask, rows, w.blk, True, w.sm_scale)
    assert np.array_equal(o[0], o[1])
    assert not np.allclose(o[0], o[2])
    K2, V2 = K[:, ::-1].copy(), V[:, ::-1].copy()   # swapping the kv heads swaps the outputs
    o2 = oracle.attention_rows(Q, K2, V2, mask, rows, w.blk, True, w.sm_scale)
    assert np.array_equal(o2[2], o[0])


def test_gap_recovered_closed_forms():
    rng = np.random.default_rng(11)
    ex = rng.standard_normal((10, 8))
    o4, o16 = ex + 0.1 * rng.standard_normal(ex.shape), ex + 0.001 * rng.standard_normal(ex.shape)
    assert oracle.gap_recovered(o4, o4, o16, ex) == 0.0
    assert abs(oracle.gap_recovered(o4, o16, o16, ex) - 100.0) < 1e-12


def test_to_f16_matches_numpy():
    x = np.random.default_rng(12).standard_normal(1000) * 3
    assert np.array_equal(oracle.to_f16(x), x.astype(np.float16))


def test_p_jitter_only_moves_rows_at_rounding_ties():
    """The test-only nudge of the encoded P: zero leaves every output as it
    was; 2^-19 (relative) only flips codes of P within that distance of an
    E2M1 / fp16 rounding boundary, so outputs move by tiny amounts (fp16
    boundaries are dense) and almost no row moves by more than 1e-3."""
    w, Q, K, V = _small(synth.CAUSAL_MH_N8K, N=512, Hq=2, Hkv=2)
    rows = oracle.all_rows(w.B, w.Hq, w.N)
    mask = oracle.select(Q, K, w.blk, w.causal, w.sm_scale, 0.1)
    qz = oracle.Quantised(Q, K, V)
    base = oracle.attention_rows(Q, K, V, mask, rows, w.blk, w.causal, w.sm_scale, qz)
    same = oracle.attention_rows(Q, K, V, mask, rows, w.blk, w.causal, w.sm_scale, qz, p_jitter=0.0)
    assert np.array_equal(base, same)
    for j in (2.0 ** -19, -(2.0 ** -19)):
        nudged = oracle.attention_rows(Q, K, V, mask, rows, w.blk, w.causal, w.sm_scale, qz, p_jitter=j)
        moved = np.abs(nudged - base).max(axis=1) > 1e-3
        assert moved.mean() < 0.01
        assert np.abs(nudged - base).mean() < 1e-5
