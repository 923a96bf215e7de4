"""Parity of the CUDA path (through the C ABI) with the CPU oracle.

Bars: NVFP4 codes and scales bit-exact; selection masks bit-exact except for
pairs whose pooled score lies within 1e-5 (relative) of the k-th score;
attention output within max-abs 2e-2 and mean-abs 1e-3 of the oracle's
fp16 output; the recovered share of the FP4-to-FP16 error gap within one
point of the oracle's.
"""
import numpy as np
import pytest
import torch

import fp16_block_attention_b200 as thrift
import oracle
import synth
from gpu_helpers import (ATOL_MAX, ATOL_MEAN, canon_qk_scales, canon_v_scales, compare_o, near_tie_pairs,
                         qk_scale_padding, shape_of, to_dev)

pytestmark = pytest.mark.gpu

# Small cases: several tiles, ragged tails, both block sizes, both head dims.
SMALL = [
    synth.TINY_NONCAUSAL_D64,                                               # the full tiny workload
    synth.CAUSAL_MH_N8K.with_(N=576, Hq=2, Hkv=2),                          # blk 64, last query tile half full
    synth.GQA_N32K.with_(N=640, Hq=4, Hkv=2),                               # GQA, blk 128
    synth.BATCHED_GQA_N16K.with_(N=384, B=2, Hq=4, Hkv=2, blk=64),          # batched, seed per batch
    synth.TINY_NONCAUSAL_D64.with_(N=192, causal=True, n_heavy=2),          # D 64 causal, ragged
    synth.CAUSAL_MH_N8K.with_(N=64, Hq=1, Hkv=1),                           # a single 64-row tile
    synth.TINY_NONCAUSAL_D64.with_(N=384, blk=128, Hq=2, Hkv=1),            # D 64, blk 128, non-causal
]
IDS = [f"{w.name}-N{w.N}-B{w.B}-H{w.Hq}x{w.Hkv}-blk{w.blk}-c{int(w.causal)}" for w in SMALL]


@pytest.fixture(scope="module")
def data():
    cache = {}

    def get(w):
        if w not in cache:
            cache[w] = synth.generate(w)
        return cache[w]
    return get


@pytest.mark.parametrize("w", SMALL, ids=IDS)
def test_quantize_bit_exact(w, data):
    Q, K, V = data(w)
    Qd, Kd, Vd = to_dev(Q, K, V)
    sh = shape_of(w)
    qz = thrift.quantize_all(Qd, Kd, Vd, sh)
    torch.cuda.synchronize()
    for x, codes, scales, H in ((Q, qz.q4, qz.qs, w.Hq), (K, qz.k4, qz.ks, w.Hkv)):
        c_ref, s_ref = oracle.quantize_rows(x)
        assert np.array_equal(codes.cpu().numpy().reshape(c_ref.shape), c_ref)
        assert np.array_equal(canon_qk_scales(scales, w.B, H, w.N, w.D), s_ref)
        assert not qk_scale_padding(scales, w.B, H, w.N, w.D).any()
    c_ref, s_ref = oracle.quantize_v(V)
    assert np.array_equal(qz.v4.cpu().numpy().reshape(c_ref.shape), c_ref)
    assert np.array_equal(canon_v_scales(qz.vs, w.B, w.Hkv, w.N, w.D), s_ref)


def _tie_groups():
    """Groups whose amax is 6*s for every positive E4M3 scale s, filled with exact
    E2M1 ties (x/s in {0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5}), grid points and
    their negatives."""
    taus = [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, -0.25, -0.75, -1.25, -1.75, -2.5, -3.5, -5.0, 0.5]
    groups = []
    for code in range(1, 127):
        s = oracle.e4m3_value(code)
        groups.append([6 * s] + [t * s for t in taus])
        groups.append([-6 * s] + [t * s for t in reversed(taus)])
    return np.array(groups, np.float64).astype(np.float16)


def test_quantize_exact_ties_and_every_fp16_value():
    ties = _tie_groups().reshape(-1)
    allf = np.arange(0, 65536, dtype=np.uint32).astype(np.uint16).view(np.float16)
    allf = allf[np.isfinite(allf.astype(np.float32))]
    np.random.default_rng(0).shuffle(allf)
    vals = np.concatenate([ties, allf])
    D = 128
    rows = -(-vals.size // D)
    rows = -(-rows // 64) * 64
    x = np.zeros(rows * D, np.float16)
    x[:vals.size] = vals
    x = x.reshape(1, 1, rows, D)
    xd, = to_dev(x)
    sh = thrift.Shape(1, 1, 1, rows, D, 64, True)
    codes, scales = thrift.quantize_nvfp4(xd, thrift.Q, sh)
    c_ref, s_ref = oracle.quantize_rows(x)
    assert np.array_equal(canon_qk_scales(scales, 1, 1, rows, D), s_ref)
    got = codes.cpu().numpy().reshape(c_ref.shape)
    bad = np.argwhere(got != c_ref)
    detail = [(x[0, 0, r, 2 * c:2 * c + 2].tolist(), int(got[0, 0, r, c]), int(c_ref[0, 0, r, c]))
              for (_, _, r, c) in bad[:8]]
    assert bad.size == 0, detail


def _mask_ok(m_gpu, m_ref, tie):
    diff = m_gpu != m_ref
    return (not diff.any()) or bool(np.all(tie[diff]))


@pytest.mark.parametrize("rho", [0.0, 0.05, 0.3, 1.0])
@pytest.mark.parametrize("w", SMALL, ids=IDS)
def test_select_matches_oracle(w, rho, data):
    Q, K, _ = data(w)
    Qd, Kd = to_dev(Q, K)
    m = thrift.select_blocks(Qd, Kd, shape_of(w), rho).cpu().numpy()
    m_ref, tie = near_tie_pairs(Q, K, w, rho)
    assert _mask_ok(m, m_ref, tie)
    nb = w.N // w.blk
    valid = nb * (nb + 1) // 2 if w.causal else nb * nb
    assert np.all(m.reshape(w.B * w.Hq, -1).sum(1) == oracle.budget(rho, valid))


@pytest.mark.parametrize("rho", [0.0, 0.05, 0.3, 1.0])
@pytest.mark.parametrize("w", SMALL, ids=IDS)
def test_attention_matches_oracle(w, rho, data):
    Q, K, V = data(w)
    Qd, Kd, Vd = to_dev(Q, K, V)
    sh = shape_of(w)
    m_ref = oracle.select(Q, K, w.blk, w.causal, w.sm_scale, rho)
    md, = to_dev(m_ref)
    qz = thrift.quantize_all(Qd, Kd, Vd, sh)
    o = thrift.attention(Qd, Kd, Vd, md, qz, sh)
    assert thrift.last_device_error() == 0
    o = o.cpu().numpy()
    rows = oracle.all_rows(w.B, w.Hq, w.N)
    ref = oracle.to_f16(oracle.attention_rows(Q, K, V, m_ref, rows, w.blk, w.causal, w.sm_scale))
    mx, mean = compare_o(o.reshape(-1, w.D), ref)
    assert mx <= ATOL_MAX and mean <= ATOL_MEAN, (mx, mean)


@pytest.mark.parametrize("w", SMALL, ids=IDS)
def test_fused_equals_the_separate_calls(w, data):
    Q, K, V = data(w)
    Qd, Kd, Vd = to_dev(Q, K, V)
    sh = shape_of(w)
    o_f = thrift.attention_fused(Qd, Kd, Vd, sh, w.rho)
    qz = thrift.quantize_all(Qd, Kd, Vd, sh)
    m = thrift.select_blocks(Qd, Kd, sh, w.rho)
    o_s = thrift.attention(Qd, Kd, Vd, m, qz, sh)
    assert torch.equal(o_f, o_s)


# ---- full-size workloads, sampled rows (the benchmark's launch configuration) ----
FULL = [synth.CAUSAL_MH_N8K, synth.GQA_N32K, synth.BATCHED_GQA_N16K, synth.GQA_N128K]


@pytest.mark.parametrize("w", FULL, ids=[w.name for w in FULL])
def test_full_size_sampled_rows(w):
    Q, K, V = synth.generate(w)
    Qd, Kd, Vd = to_dev(Q, K, V)
    sh = shape_of(w)
    o_f = thrift.attention_fused(Qd, Kd, Vd, sh, w.rho)
    m = thrift.select_blocks(Qd, Kd, sh, w.rho)
    assert thrift.last_device_error() == 0
    m_ref, tie = near_tie_pairs(Q, K, w, w.rho)
    assert _mask_ok(m.cpu().numpy(), m_ref, tie)
    rows = synth.sample_rows(w, 96, per_block=16)
    qz = oracle.Quantised(Q, K, V)
    ref = oracle.to_f16(oracle.attention_rows(Q, K, V, m_ref, rows, w.blk, w.causal, w.sm_scale, qz))
    o = o_f.cpu().numpy()
    got = o[rows[:, 0], rows[:, 1], rows[:, 2]]
    mx, mean = compare_o(got, ref)
    assert mx <= ATOL_MAX and mean <= ATOL_MEAN, (mx, mean)


def test_gap_recovered_agrees_with_oracle():
    w = synth.GQA_N32K
    Q, K, V = synth.generate(w)
    Qd, Kd, Vd = to_dev(Q, K, V)
    sh = shape_of(w)
    rows = synth.sample_rows(w, 64, per_block=16)
    qz = oracle.Quantised(Q, K, V)
    ex = oracle.exact_rows(Q, K, V, rows, w.causal, w.sm_scale)
    gpu, ref = {}, {}
    for rho in (0.0, w.rho, 1.0):
        o = thrift.attention_fused(Qd, Kd, Vd, sh, rho).cpu().numpy()
        gpu[rho] = o[rows[:, 0], rows[:, 1], rows[:, 2]].astype(np.float64)
        m = oracle.select(Q, K, w.blk, w.causal, w.sm_scale, rho)
        ref[rho] = oracle.to_f16(oracle.attention_rows(Q, K, V, m, rows, w.blk, w.causal, w.sm_scale, qz)
                                 ).astype(np.float64)
    g = oracle.gap_recovered(gpu[0.0], gpu[w.rho], gpu[1.0], ex)
    r = oracle.gap_recovered(ref[0.0], ref[w.rho], ref[1.0], ex)
    assert abs(g - r) <= 1.0, (g, r)


def test_mma_rate_probe_runs_without_error():
    from fp16_block_attention_b200 import probe
    probe.mma_rate(0, 64)
    probe.mma_rate(1, 64)
    assert probe.last_error() == 0
