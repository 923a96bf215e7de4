"""Parity of the vertical-line / local-window selector on the GPU (through the
C ABI) with its oracle, and its gap recovered against the method's own
selector at equal rho.

The GPU sums the column signal in FP32 and the oracle in FP64, so two columns
whose signals lie within the FP32 error bound of each other may swap ranks.
A swap changes the mask only when it straddles the budget's cut, and then
only inside those columns.  The bar: every mask holds exactly k pairs, and
every pair where the GPU and the oracle differ lies outside the window, in
columns whose oracle signals agree within 2 (nb + 8) 2^-24 relative (each of
the <= nb FP32 terms of a column sum carries a few ulps, and the running sum
one rounding per term).  Pooled scores are bit-exact on both sides, so the
order inside a column never differs.
"""
import numpy as np
import pytest

import fp16_block_attention_b200 as thrift
import oracle
import synth
from oracle import vertical_window as vw
from gpu_helpers import shape_of, to_dev

pytestmark = pytest.mark.gpu

SMALL = [
    synth.TINY_NONCAUSAL_D64,
    synth.CAUSAL_MH_N8K.with_(N=2048, Hq=2, Hkv=2),                  # blk 64, nb 32
    synth.GQA_N32K.with_(N=4096, Hq=4, Hkv=2),                       # GQA, blk 128
    synth.BATCHED_GQA_N16K.with_(N=3072, B=2, Hq=4, Hkv=2, blk=64),  # batched
    synth.TINY_NONCAUSAL_D64.with_(N=64, blk=64),                    # one block
]
FULL = [
    synth.GQA_N32K,                                                  # nb 256, 32 heads
    synth.GQA_N128K.with_(Hq=8, Hkv=2),                              # nb 1024
    synth.CAUSAL_MH_N8K.with_(N=131072, Hq=2, Hkv=1),                # blk 64: nb 2048, the largest
]


def _ids(ws):
    return [f"{w.name}-N{w.N}-B{w.B}-H{w.Hq}x{w.Hkv}-blk{w.blk}-c{int(w.causal)}" for w in ws]


def _heads(w, Q, K):
    group = w.Hq // w.Hkv
    for b in range(w.B):
        for h in range(w.Hq):
            yield b, h, oracle.pooled_scores(Q[b, h], K[b, h // group], w.blk, w.causal, w.sm_scale)


def _check(w, m_gpu, Q, K, rho, window):
    nb = w.N // w.blk
    tol = 2.0 * (nb + 8) * 2.0 ** -24
    for b, h, sc in _heads(w, Q, K):
        mg = m_gpu[b, h]
        mo = vw.select_head(sc, w.causal, rho, window, oracle.budget)
        assert mg.sum() == mo.sum(), (b, h)
        if w.causal:
            assert not np.any(np.triu(mg, 1)), (b, h)
        di, dj = np.nonzero(mg != mo)
        if di.size == 0:
            continue
        assert not np.any(vw.in_window(di, dj, window, w.causal)), (b, h)
        v = vw.column_signal(sc, w.causal)[np.unique(dj)]
        assert v.max() - v.min() <= tol * v.max(), (b, h, np.unique(dj), v)


@pytest.mark.parametrize("w", SMALL, ids=_ids(SMALL))
@pytest.mark.parametrize("rho", [0.0, 0.01, 0.05, 0.3, 1.0])
@pytest.mark.parametrize("window", [0, 1, 2, 4])
def test_vertical_window_select_matches_oracle(w, rho, window):
    Q, K, _ = synth.generate(w)
    Qd, Kd = to_dev(Q, K)
    m = thrift.select_blocks_vertical_window(Qd, Kd, shape_of(w), rho, window).cpu().numpy()
    assert thrift.last_device_error() == 0
    _check(w, m, Q, K, rho, window)


@pytest.mark.parametrize("w", FULL, ids=_ids(FULL))
def test_vertical_window_select_matches_oracle_at_full_size(w):
    Q, K, _ = synth.generate(w)
    Qd, Kd = to_dev(Q, K)
    m = thrift.select_blocks_vertical_window(Qd, Kd, shape_of(w), w.rho, 2).cpu().numpy()
    assert thrift.last_device_error() == 0
    _check(w, m, Q, K, w.rho, 2)


def test_window_larger_than_the_grid_keeps_every_pair():
    w = synth.CAUSAL_MH_N8K.with_(N=1024, Hq=1, Hkv=1)
    Q, K, _ = synth.generate(w)
    Qd, Kd = to_dev(Q, K)
    nb = w.N // w.blk
    m = thrift.select_blocks_vertical_window(Qd, Kd, shape_of(w), 1.0, 10 * nb).cpu().numpy()
    assert np.array_equal(m[0, 0], np.tril(np.ones((nb, nb), np.uint8)))


def _rel_err(o, ex):
    return float(np.linalg.norm(o - ex) / np.linalg.norm(ex))


@pytest.mark.parametrize("window", [1, 2, 4])
def test_gap_recovered_against_the_method_selector(window):
    """Both selectors at the same rho on the causal GQA generator (N = 8192):
    the GPU's gap on sampled rows must agree with the oracle's within one
    point for the vertical-line selector.  Run with -s for both gaps."""
    w = synth.GQA_N32K.with_(N=8192)
    Q, K, V = synth.generate(w)
    Qd, Kd, Vd = to_dev(Q, K, V)
    sh = shape_of(w)
    rows = synth.sample_rows(w, 48, per_block=8)
    qz = oracle.Quantised(Q, K, V)
    qd = thrift.quantize_all(Qd, Kd, Vd, sh)
    ex = oracle.exact_rows(Q, K, V, rows, w.causal, w.sm_scale)

    def gpu_rows(mask_d):
        o = thrift.attention(Qd, Kd, Vd, mask_d, qd, sh).cpu().numpy()
        assert thrift.last_device_error() == 0
        return o[rows[:, 0], rows[:, 1], rows[:, 2]].astype(np.float64)

    def ref_rows(mask):
        return oracle.to_f16(oracle.attention_rows(Q, K, V, mask, rows, w.blk, w.causal, w.sm_scale, qz)
                             ).astype(np.float64)

    g = {r: gpu_rows(thrift.select_blocks(Qd, Kd, sh, r)) for r in (0.0, w.rho, 1.0)}
    m_vw = thrift.select_blocks_vertical_window(Qd, Kd, sh, w.rho, window)
    g_vw = gpu_rows(m_vw)
    r_vw = ref_rows(m_vw.cpu().numpy())
    r = {rho: ref_rows(oracle.select(Q, K, w.blk, w.causal, w.sm_scale, rho)) for rho in (0.0, 1.0)}
    gap_thrift = oracle.gap_recovered(g[0.0], g[w.rho], g[1.0], ex)
    gap_vw = oracle.gap_recovered(g[0.0], g_vw, g[1.0], ex)
    gap_vw_ref = oracle.gap_recovered(r[0.0], r_vw, r[1.0], ex)
    print(f"\nselector gap N={w.N} rho={w.rho} W={window}: E(rho=0)={_rel_err(g[0.0], ex):.5f} "
          f"E(thrift)={_rel_err(g[w.rho], ex):.5f} E(vertical+window)={_rel_err(g_vw, ex):.5f} "
          f"E(rho=1)={_rel_err(g[1.0], ex):.5f} gap_thrift={gap_thrift:.2f} gap_vw={gap_vw:.2f} "
          f"gap_vw_oracle={gap_vw_ref:.2f}")
    assert abs(gap_vw - gap_vw_ref) <= 1.0, (gap_vw, gap_vw_ref)
