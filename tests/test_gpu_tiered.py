"""Parity of the tiered selection (FP16 / MXFP8 / NVFP4 / skip) and of attention with
skipped pairs on the GPU (through the C ABI) with the oracle.

Selection: exactly k16 FP16, k8 8-bit and ks skipped pairs per head; the
masks agree except for pairs whose pooled score lies within 1e-5 (relative)
of a score beside one of the three cuts of the ranking, where FP32 summation
order may swap neighbours.  Attention:
the oracle's mask given to the GPU, outputs within max-abs 2e-2 and mean-abs
1e-3 of the oracle's (the prefill bars), where a row that misses the bar is
re-checked against the oracle with its encoded P nudged by 2^-19 both ways
(rounding ties of P, which skipping makes visible by concentrating a row's
weight on few NVFP4 keys; at most one row in a thousand); blk 128 leaves
skipped tiles out of every role's work, blk 64 masks skipped blocks inside a
128-key tile.
"""
import numpy as np
import pytest

import fp16_block_attention_b200 as thrift
import oracle
import synth
from gpu_helpers import ATOL_MAX, ATOL_MEAN, compare_o_with_ties, shape_of, to_dev

pytestmark = pytest.mark.gpu

CASES = [
    synth.TINY_NONCAUSAL_D64,                                         # blk 64, non-causal
    synth.CAUSAL_MH_N8K.with_(N=1536, Hq=2, Hkv=2),                   # blk 64, causal
    synth.GQA_N32K.with_(N=2048, Hq=4, Hkv=2),                        # blk 128, GQA
    synth.BATCHED_GQA_N16K.with_(N=1280, B=2, Hq=4, Hkv=2),           # blk 128, batched, ragged tail
]
IDS = [f"{w.name}-N{w.N}-B{w.B}-H{w.Hq}x{w.Hkv}-blk{w.blk}" for w in CASES]


def _valid(nb, causal):
    return np.tril(np.ones((nb, nb), bool)) if causal else np.ones((nb, nb), bool)


def _cut_scores(sc, nb, causal, cuts):
    """Pooled scores on both sides of each cut position of the ranking (forced
    pairs first, then score descending, then the lower linear index)."""
    ii, jj = np.meshgrid(np.arange(nb), np.arange(nb), indexing="ij")
    valid = _valid(nb, causal)
    i, j, v = ii[valid], jj[valid], sc[valid]
    order = np.lexsort((i * nb + j, -v, ~((i == j) | (j == 0))))
    n = len(order)
    return [v[order[k + d]] for k in cuts if 0 < k < n for d in (-1, 0)]


@pytest.mark.parametrize("rho,rho8,sigma", [(0.05, 0.0, 0.25), (0.0, 0.0, 0.6), (0.3, 0.0, 0.5), (0.05, 0.0, 1.0),
                                            (0.05, 0.1, 0.0), (0.05, 0.2, 0.5), (0.0, 0.3, 0.9), (0.02, 1.0, 0.0)])
@pytest.mark.parametrize("w", CASES, ids=IDS)
def test_tiered_select_matches_oracle(w, rho, rho8, sigma):
    Q, K, _ = synth.generate(w)
    Qd, Kd = to_dev(Q, K)
    m = thrift.select_blocks_tiered(Qd, Kd, shape_of(w), rho, sigma, rho8=rho8).cpu().numpy()
    ref = oracle.select_tiered(Q, K, w.blk, w.causal, w.sm_scale, rho, sigma, rho8)
    nb = w.N // w.blk
    valid = _valid(nb, w.causal)
    n = int(valid.sum())
    forced = np.zeros((nb, nb), bool)
    forced[np.arange(nb), np.arange(nb)] = True
    forced[:, 0] = True
    G = w.Hq // w.Hkv
    for b in range(w.B):
        for h in range(w.Hq):
            mg, mo = m[b, h], ref[b, h]
            for c in (1, 2, 3):
                assert (mg == c).sum() == (mo == c).sum(), (b, h, c)
            assert not np.any((mg == 2) & forced) and not np.any((mg != 0) & ~valid)
            diff = mg != mo
            if not diff.any():
                continue
            sc = oracle.pooled_scores(Q[b, h], K[b, h // G], w.blk, w.causal, w.sm_scale)
            k16, k8, ks = (int((mo == c).sum()) for c in (1, 3, 2))
            near = np.zeros_like(diff)
            for c in _cut_scores(sc, nb, w.causal, (k16, k16 + k8, n - ks)):
                near |= np.abs(sc - c) <= 1e-5 * max(abs(c), 1e-30)
            assert np.all(near[diff]), (b, h)


@pytest.mark.parametrize("rho,sigma", [(0.05, 0.25), (0.0, 0.6), (0.3, 0.9)])
@pytest.mark.parametrize("w", CASES, ids=IDS)
def test_attention_with_skipped_pairs_matches_oracle(w, rho, sigma):
    Q, K, V = synth.generate(w)
    Qd, Kd, Vd = to_dev(Q, K, V)
    sh = shape_of(w)
    m = oracle.select_tiered(Q, K, w.blk, w.causal, w.sm_scale, rho, sigma)
    assert (m == 2).any()
    md, = to_dev(m)
    qz = thrift.quantize_all(Qd, Kd, Vd, sh)
    o = thrift.attention_tiered(Qd, Kd, Vd, md, qz, sh)
    assert thrift.last_device_error() == 0
    o = o.cpu().numpy()
    rows = oracle.all_rows(w.B, w.Hq, w.N)
    if rows.shape[0] > 8192:
        rows = rows[np.random.default_rng(2).choice(rows.shape[0], 8192, replace=False)]
    mx, mean, resolved = compare_o_with_ties(o[rows[:, 0], rows[:, 1], rows[:, 2]], Q, K, V, m, rows, w.blk,
                                             w.causal, w.sm_scale)
    assert mx <= ATOL_MAX and mean <= ATOL_MEAN, (mx, mean)
    assert resolved <= max(1, rows.shape[0] // 1000), resolved  # ties are rare


@pytest.mark.parametrize("sigma", [0.0, 0.25, 0.5, 0.75])
def test_quality_cost_of_skipping(sigma):
    """The relative error of the output against exact attention on sampled
    rows of the causal GQA generator (N = 8192) at rho = 5% as the skipped
    share grows, GPU beside the oracle (within one point of the FP4-to-FP16
    gap).  Run with -s for the series."""
    w = synth.GQA_N32K.with_(N=8192)
    Q, K, V = synth.generate(w)
    Qd, Kd, Vd = to_dev(Q, K, V)
    sh = shape_of(w)
    rows = synth.sample_rows(w, 48, per_block=8)
    ex = oracle.exact_rows(Q, K, V, rows, w.causal, w.sm_scale)
    qd = thrift.quantize_all(Qd, Kd, Vd, sh)
    qz = oracle.Quantised(Q, K, V)

    def gpu(mask_d):
        o = thrift.attention_tiered(Qd, Kd, Vd, mask_d, qd, sh).cpu().numpy()
        assert thrift.last_device_error() == 0
        return o[rows[:, 0], rows[:, 1], rows[:, 2]].astype(np.float64)

    err = lambda o: float(np.linalg.norm(o - ex) / np.linalg.norm(ex))
    e4 = err(gpu(thrift.select_blocks(Qd, Kd, sh, 0.0)))
    e16 = err(gpu(thrift.select_blocks(Qd, Kd, sh, 1.0)))
    m = thrift.select_blocks_tiered(Qd, Kd, sh, w.rho, sigma)
    eg = err(gpu(m))
    er = err(oracle.to_f16(oracle.attention_rows(Q, K, V, m.cpu().numpy(), rows, w.blk, w.causal, w.sm_scale, qz)))
    skipped = float((m.cpu().numpy() == 2).mean() / (0.5 + 0.5 / (w.N // w.blk)))
    gap = lambda e: 100.0 * (e4 - e) / (e4 - e16)
    print(f"\nskip sigma={sigma}: skipped share {skipped:.3f} E(gpu)={eg:.5f} E(oracle)={er:.5f} "
          f"E(rho=0)={e4:.5f} E(rho=1)={e16:.5f} gap_gpu={gap(eg):.2f} gap_oracle={gap(er):.2f}")
    assert abs(gap(eg) - gap(er)) <= 1.0
