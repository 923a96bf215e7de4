"""Parity of attention with 8-bit pairs (mask 3, MXFP8) on the GPU (through
the C ABI) with the oracle.

The oracle's mask (four classes: FP16, MXFP8, NVFP4, skipped) is given to the
GPU, which takes S of an 8-bit pair from the MXFP8 copies of Q and K and
P * 2^11 as MXFP8 per 32 keys times the MXFP8 copy of V.  Outputs within
max-abs 2e-2 and mean-abs 1e-3 of the oracle's (the prefill bars), a row
that misses the bar re-checked with its encoded P nudged by 2^-19 both ways
(a P at a rounding tie of E4M3, E2M1 or of the E8M0 exponent; at most one row
in a thousand).  Also: the error paths (a 3 without the copies, the copies
with blk 64) and the quality series of the 8-bit budget beside the oracle's.
"""
import numpy as np
import pytest
import torch

import fp16_block_attention_b200 as thrift
import oracle
import synth
from gpu_helpers import ATOL_MAX, ATOL_MEAN, compare_o_with_ties, shape_of, to_dev

pytestmark = pytest.mark.gpu

CASES = [
    synth.GQA_N32K.with_(N=2048, Hq=4, Hkv=2),                        # causal GQA
    synth.TINY_NONCAUSAL_D64.with_(blk=128, Hq=2, Hkv=1),             # D 64, non-causal
    synth.BATCHED_GQA_N16K.with_(N=1280, B=2, Hq=4, Hkv=2),           # batched, odd tile count
]
IDS = [f"{w.name}-N{w.N}-B{w.B}-H{w.Hq}x{w.Hkv}-D{w.D}" for w in CASES]


def _run(w, rho, rho8, sigma):
    Q, K, V = synth.generate(w)
    Qd, Kd, Vd = to_dev(Q, K, V)
    sh = shape_of(w)
    m = oracle.select_tiered(Q, K, w.blk, w.causal, w.sm_scale, rho, sigma, rho8)
    md, = to_dev(m)
    q4 = thrift.quantize_all(Qd, Kd, Vd, sh)
    q8 = thrift.quantize_all_mxfp8(Qd, Kd, Vd, sh)
    o = thrift.attention_tiered(Qd, Kd, Vd, md, q4, sh, q8=q8)
    assert thrift.last_device_error() == 0
    return Q, K, V, m, o.cpu().numpy()


@pytest.mark.parametrize("rho,rho8,sigma", [(0.0, 1.0, 0.0), (0.05, 0.2, 0.0), (0.05, 0.3, 0.4), (0.2, 0.5, 0.2)])
@pytest.mark.parametrize("w", CASES, ids=IDS)
def test_attention_with_eight_bit_pairs_matches_oracle(w, rho, rho8, sigma):
    Q, K, V, m, o = _run(w, rho, rho8, sigma)
    assert (m == 3).any()
    rows = oracle.all_rows(w.B, w.Hq, w.N)
    if rows.shape[0] > 6144:
        rows = rows[np.random.default_rng(5).choice(rows.shape[0], 6144, replace=False)]
    qz = oracle.Quantised(Q, K, V, mx8=True)
    mx, mean, resolved = compare_o_with_ties(o[rows[:, 0], rows[:, 1], rows[:, 2]], Q, K, V, m, rows, w.blk,
                                             w.causal, w.sm_scale, qz)
    assert mx <= ATOL_MAX and mean <= ATOL_MEAN, (mx, mean)
    assert resolved <= max(1, rows.shape[0] // 1000), resolved


@pytest.mark.parametrize("rho,rho8,sigma", [(0.05, 0.2, 0.0), (0.05, 0.0, 0.4), (0.1, 0.3, 0.3)])
@pytest.mark.parametrize("w", CASES[:2], ids=IDS[:2])
def test_fused_tiered_equals_the_separate_calls(w, rho, rho8, sigma):
    Q, K, V = synth.generate(w)
    Qd, Kd, Vd = to_dev(Q, K, V)
    sh = shape_of(w)
    o1 = thrift.attention_fused_tiered(Qd, Kd, Vd, sh, rho, rho8, sigma)
    assert thrift.last_device_error() == 0
    m = thrift.select_blocks_tiered(Qd, Kd, sh, rho, sigma, rho8=rho8)
    q8 = thrift.quantize_all_mxfp8(Qd, Kd, Vd, sh) if rho8 > 0 else None
    o2 = thrift.attention_tiered(Qd, Kd, Vd, m, thrift.quantize_all(Qd, Kd, Vd, sh), sh, q8=q8)
    assert thrift.last_device_error() == 0
    assert torch.equal(o1, o2)


EDGE = [
    synth.GQA_N32K.with_(N=128, Hq=2, Hkv=1),                          # one key tile
    synth.TINY_NONCAUSAL_D64.with_(N=256, blk=128, Hq=1, Hkv=1),       # two tiles, non-causal, D 64
    synth.BATCHED_GQA_N16K.with_(N=384, B=1, Hq=2, Hkv=2),             # three tiles, Hq = Hkv
]


@pytest.mark.parametrize("fill", ["all8", "all8_diag16", "alternate"])
@pytest.mark.parametrize("w", EDGE, ids=[f"N{w.N}-D{w.D}-{'c' if w.causal else 'nc'}" for w in EDGE])
def test_eight_bit_edge_masks(w, fill):
    """Hand-made masks on one to three key tiles: every valid pair 8-bit; all
    8-bit but the diagonal in FP16; 8-bit and NVFP4 alternating by key tile
    (so consecutive tiles change ring slot use), against the oracle."""
    Q, K, V = synth.generate(w)
    Qd, Kd, Vd = to_dev(Q, K, V)
    sh = shape_of(w)
    nb = w.N // w.blk
    m = np.full((w.B, w.Hq, nb, nb), 3, np.uint8)
    if fill == "all8_diag16":
        m[:, :, np.arange(nb), np.arange(nb)] = 1
    elif fill == "alternate":
        m[..., 1::2] = 0
    if w.causal:
        m &= np.tril(np.ones((nb, nb), np.uint8))[None, None] * 255
    md, = to_dev(m)
    o = thrift.attention_tiered(Qd, Kd, Vd, md, thrift.quantize_all(Qd, Kd, Vd, sh), sh,
                                q8=thrift.quantize_all_mxfp8(Qd, Kd, Vd, sh))
    assert thrift.last_device_error() == 0
    o = o.cpu().numpy()
    rows = oracle.all_rows(w.B, w.Hq, w.N)
    mx, mean, resolved = compare_o_with_ties(o[rows[:, 0], rows[:, 1], rows[:, 2]], Q, K, V, m, rows, w.blk,
                                             w.causal, w.sm_scale, oracle.Quantised(Q, K, V, mx8=True))
    assert mx <= ATOL_MAX and mean <= ATOL_MEAN, (mx, mean)
    assert resolved <= 1, resolved


def test_eight_bit_mask_without_the_copies_is_reported():
    """A 3 in the mask with no MXFP8 copies: the call returns, the device
    error word says invalid argument (1), the tile is computed in NVFP4."""
    w = CASES[0]
    Q, K, V = synth.generate(w)
    Qd, Kd, Vd = to_dev(Q, K, V)
    sh = shape_of(w)
    m = oracle.select_tiered(Q, K, w.blk, w.causal, w.sm_scale, 0.05, 0.0, 0.2)
    md, = to_dev(m)
    q4 = thrift.quantize_all(Qd, Kd, Vd, sh)
    thrift.attention_tiered(Qd, Kd, Vd, md, q4, sh)
    assert thrift.last_device_error() == 1
    assert thrift.last_device_error() == 0  # read and cleared
    o = thrift.attention_tiered(Qd, Kd, Vd, md, q4, sh, q8=thrift.quantize_all_mxfp8(Qd, Kd, Vd, sh))
    assert thrift.last_device_error() == 0 and np.isfinite(o.float().cpu().numpy()).all()


def test_eight_bit_copies_need_128_blocks():
    w = synth.CAUSAL_MH_N8K.with_(N=512, Hq=2, Hkv=2)      # blk 64
    Q, K, V = synth.generate(w)
    Qd, Kd, Vd = to_dev(Q, K, V)
    sh = shape_of(w)
    md, = to_dev(np.zeros((1, 2, 8, 8), np.uint8))
    with pytest.raises(thrift.ThriftError):
        thrift.attention_tiered(Qd, Kd, Vd, md, thrift.quantize_all(Qd, Kd, Vd, sh), sh,
                                q8=thrift.quantize_all_mxfp8(Qd, Kd, Vd, sh))


@pytest.mark.parametrize("rho8", [0.0, 0.1, 0.25, 0.5, 1.0])
def test_quality_of_the_eight_bit_budget(rho8):
    """Relative error against exact attention on sampled rows of the causal
    GQA generator (N = 8192) at rho = 5% as the 8-bit share grows, GPU beside
    the oracle (within one point of the FP4-to-FP16 gap).  Run with -s for
    the series."""
    w = synth.GQA_N32K.with_(N=8192)
    Q, K, V = synth.generate(w)
    Qd, Kd, Vd = to_dev(Q, K, V)
    sh = shape_of(w)
    rows = synth.sample_rows(w, 48, per_block=8)
    ex = oracle.exact_rows(Q, K, V, rows, w.causal, w.sm_scale)
    q4 = thrift.quantize_all(Qd, Kd, Vd, sh)
    q8 = thrift.quantize_all_mxfp8(Qd, Kd, Vd, sh)
    qz = oracle.Quantised(Q, K, V, mx8=True)

    def gpu(mask_d):
        o = thrift.attention_tiered(Qd, Kd, Vd, mask_d, q4, sh, q8=q8).cpu().numpy()
        assert thrift.last_device_error() == 0
        return o[rows[:, 0], rows[:, 1], rows[:, 2]].astype(np.float64)

    err = lambda o: float(np.linalg.norm(o - ex) / np.linalg.norm(ex))
    e4 = err(gpu(thrift.select_blocks(Qd, Kd, sh, 0.0)))
    e16 = err(gpu(thrift.select_blocks(Qd, Kd, sh, 1.0)))
    m = thrift.select_blocks_tiered(Qd, Kd, sh, w.rho, 0.0, rho8=rho8)
    eg = err(gpu(m))
    er = err(oracle.to_f16(oracle.attention_rows(Q, K, V, m.cpu().numpy(), rows, w.blk, w.causal, w.sm_scale, qz)))
    gap = lambda e: 100.0 * (e4 - e) / (e4 - e16)
    share = float((m.cpu().numpy() == 3).mean() / (0.5 + 0.5 / (w.N // w.blk)))
    print(f"\n8-bit rho8={rho8}: share {share:.3f} E(gpu)={eg:.5f} E(oracle)={er:.5f} "
          f"E(rho=0)={e4:.5f} E(rho=1)={e16:.5f} gap_gpu={gap(eg):.2f} gap_oracle={gap(er):.2f}")
    assert abs(gap(eg) - gap(er)) <= 1.0
