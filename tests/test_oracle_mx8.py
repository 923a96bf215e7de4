"""Pins of the oracle's MXFP8 path (8-bit pairs, mask value 3; no GPU).

MXFP8 is the OCP microscaling format with E4M3 elements: 32 values share one
E8M0 scale X = 2^(floor(log2 amax) - 8); elements are E4M3(v / X), nearest
even, saturating at 448.  Pins: the direct E4M3 rounding against the
exhaustive nearest-value search and against torch's float8_e4m3fn; E8M0
values; closed-form groups (an exact power-of-two range, saturation, zero);
quantise-dequantise-quantise idempotence; V quantised along keys; and in
attention: zero queries return the mean of the MXFP8-decoded values, and an
all-8-bit output sits between the all-FP16 and all-FP4 outputs in error.
"""
import numpy as np
import pytest
import torch

import oracle
import synth


def _f16(x):
    return np.asarray(x, np.float64).astype(np.float16)


def test_direct_e4m3_rounding_matches_the_nearest_value_search():
    vals = np.array([oracle.e4m3_value(c) for c in range(127)])           # 0 .. 448
    mids = (vals[1:] + vals[:-1]) / 2                                       # every tie
    rng = np.random.default_rng(0)
    rand = np.concatenate([rng.uniform(0, 480, 2000), np.exp2(rng.uniform(-14, 9, 2000))])
    xs = np.concatenate([vals, mids, np.nextafter(mids, 0), np.nextafter(mids, 1e9), rand,
                         [448.0, 463.9, 464.0, 500.0, 1e6, 2.0 ** -10, 2.0 ** -12]])
    for x in xs:
        for v in (x, -x):
            assert oracle.e4m3_encode_direct(v) == oracle.e4m3_encode(v), v


def test_e4m3_rounding_matches_torch_float8():
    rng = np.random.default_rng(1)
    x = np.concatenate([rng.uniform(-448, 448, 4000), np.exp2(rng.uniform(-12, 8.8, 2000))])
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([oracle.e4m3_encode_direct(v) for v in x], np.uint8)
    assert np.array_equal(got, ref)


def test_e8m0_values():
    for e in (0, 1, 100, 127, 128, 200, 254):
        assert oracle.e8m0_value(e) == 2.0 ** (e - 127)


def _group(vals):
    row = np.zeros((1, 32))
    row[0, :len(vals)] = vals
    return oracle.quantize_rows_mx8(_f16(row))


def test_group_closed_forms():
    c, s = _group([448.0, 1.0, -2.0])          # floor(log2 448) = 8: X = 1
    assert s[0, 0] == 127 and c[0, 0] == 0x7E and oracle.e4m3_value(int(c[0, 1])) == 1.0
    c, s = _group([1.0, 0.5])                  # X = 2^-8: 1 -> 256, 0.5 -> 128
    assert s[0, 0] == 119
    assert oracle.e4m3_value(int(c[0, 0])) == 256.0 and oracle.e4m3_value(int(c[0, 1])) == 128.0
    c, s = _group([511.0, 3.0])                # X = 1: 511 saturates to 448
    assert s[0, 0] == 127 and c[0, 0] == 0x7E
    c, s = _group([])                          # all zero
    assert s[0, 0] == 0 and not c.any()


def test_quantise_dequantise_quantise_is_idempotent():
    rng = np.random.default_rng(2)
    x = _f16(rng.standard_normal((64, 128)) * np.exp2(rng.integers(-6, 7, (64, 1))))
    c, s = oracle.quantize_rows_mx8(x)
    d = oracle.dequantize_mx8(c, s)
    X = np.repeat(np.array([[oracle.e8m0_value(e) for e in r] for r in s]), 32, axis=1)
    xf = x.astype(np.float64)
    # half an E4M3 step (2^-4 relative; subnormal steps 2^-9 X), or saturation at 448 X (< 1/8 of the value)
    assert np.all(np.abs(d - xf) <= np.maximum(np.abs(xf) * 2.0 ** -4, X * 2.0 ** -10) + (np.abs(xf) > 448 * X) *
                  np.abs(xf) / 8)
    c2, s2 = oracle.quantize_rows_mx8(_f16(d))
    assert np.array_equal(s, s2) and np.array_equal(c, c2)


def test_v_is_quantised_along_keys():
    rng = np.random.default_rng(3)
    V = _f16(rng.standard_normal((1, 2, 96, 64)))
    c, s = oracle.quantize_v_mx8(V)
    for h in range(2):
        for d in (0, 17, 63):
            cr, sr = oracle.quantize_rows_mx8(np.ascontiguousarray(V[0, h, :, d][None]))
            assert np.array_equal(c[0, h, d], cr[0]) and np.array_equal(s[0, h, d], sr[0])


@pytest.mark.parametrize("causal", [True, False])
def test_zero_queries_average_the_decoded_values(causal):
    """S = 0 everywhere: every P is 1, P * 2^11 = 2048 is exact in MXFP8, so
    an all-8-bit row is the plain mean of the MXFP8-decoded V over its keys."""
    w = synth.CAUSAL_MH_N8K.with_(N=256, Hq=1, Hkv=1, causal=causal)
    _, K, V = synth.generate(w)
    Q = np.zeros((1, 1, w.N, w.D), np.float16)
    nb = w.N // w.blk
    qz = oracle.Quantised(Q, K, V, mx8=True)
    rows = np.array([[0, 0, 0], [0, 0, 77], [0, 0, w.N - 1]], np.int64)
    o = oracle.attention_rows(Q, K, V, np.full((1, 1, nb, nb), 3, np.uint8), rows, w.blk, causal, w.sm_scale, qz)
    vd = oracle.dequantize_mx8(qz.v8, qz.vs8)[0, 0]           # [D, N]
    for t, (_, _, r) in enumerate(rows):
        n = r + 1 if causal else w.N
        assert np.allclose(o[t], vd[:, :n].mean(axis=1), rtol=1e-12, atol=1e-12)


def test_eight_bit_error_sits_between_fp16_and_fp4():
    w = synth.GQA_N32K.with_(N=512, Hq=4, Hkv=2)
    Q, K, V = synth.generate(w)
    rows = oracle.all_rows(w.B, w.Hq, w.N)
    nb = w.N // w.blk
    qz = oracle.Quantised(Q, K, V, mx8=True)
    ex = oracle.exact_rows(Q, K, V, rows, w.causal, w.sm_scale)
    err = {}
    for cls in (1, 3, 0):
        o = oracle.attention_rows(Q, K, V, np.full((1, w.Hq, nb, nb), cls, np.uint8), rows, w.blk, w.causal,
                                  w.sm_scale, qz)
        err[cls] = np.linalg.norm(o - ex) / np.linalg.norm(ex)
    assert err[1] < err[3] < 0.6 * err[0]
    with pytest.raises(ValueError):
        oracle.attention_rows(Q, K, V, np.full((1, w.Hq, nb, nb), 3, np.uint8), rows[:4], w.blk, w.causal,
                              w.sm_scale, oracle.Quantised(Q, K, V))
