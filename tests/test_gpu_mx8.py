"""MXFP8 copies on the GPU (through the C ABI) against the oracle: codes and
scales bit-exact (the scale layout undone by its index formula), every byte
no element maps to zero."""
import numpy as np
import pytest

import fp16_block_attention_b200 as thrift
import oracle
import synth
from gpu_helpers import shape_of, to_dev

pytestmark = pytest.mark.gpu

SHAPES = [
    synth.GQA_N32K.with_(N=640, Hq=4, Hkv=2),                    # D 128, whole tiles
    synth.CAUSAL_MH_N8K.with_(N=576, Hq=2, Hkv=2),               # D 128, last tile half full
    synth.TINY_NONCAUSAL_D64.with_(N=448, Hq=2, Hkv=1),          # D 64, ragged
    synth.BATCHED_GQA_N16K.with_(N=256, B=2, Hq=4, Hkv=2),       # batched
]
IDS = [f"{w.name}-N{w.N}-D{w.D}" for w in SHAPES]


def _check(w, x, op, H):
    sh = shape_of(w)
    xd, = to_dev(x)
    codes, scales = thrift.quantize_mxfp8(xd, op, sh)
    codes, scales = codes.cpu().numpy(), scales.cpu().numpy()
    NT = (w.N + 127) // 128
    if op == thrift.V:
        c_ref, s_ref = oracle.quantize_v_mx8(x)                         # [B,H,D,N], [B,H,D,N/32]
        assert np.array_equal(codes.reshape(c_ref.shape), c_ref)
        bh, d, g = np.meshgrid(np.arange(w.B * H), np.arange(w.D), np.arange(w.N // 32), indexing="ij")
        idx = thrift.mx8_v_scale_index(bh, d, g * 32, NT)
    else:
        c_ref, s_ref = oracle.quantize_rows_mx8(x)                      # [B,H,N,D], [B,H,N,D/32]
        assert np.array_equal(codes.reshape(c_ref.shape), c_ref)
        bh, n, g = np.meshgrid(np.arange(w.B * H), np.arange(w.N), np.arange(w.D // 32), indexing="ij")
        idx = thrift.mx8_qk_scale_index(bh, n, g, NT)
    assert np.array_equal(scales[idx].reshape(s_ref.shape), s_ref)
    used = np.zeros(scales.size, bool)
    used[idx.ravel()] = True
    assert not scales[~used].any()


@pytest.mark.parametrize("w", SHAPES, ids=IDS)
def test_mxfp8_qkv_bit_exact(w):
    Q, K, V = synth.generate(w)
    _check(w, Q, thrift.Q, w.Hq)
    _check(w, K, thrift.K, w.Hkv)
    _check(w, V, thrift.V, w.Hkv)


def test_mxfp8_special_groups():
    """Zero groups (with -0), saturation near the top of a group, fp16
    subnormals and a group whose amax is an exact power of two."""
    w = synth.TINY_NONCAUSAL_D64.with_(N=128, Hq=1, Hkv=1)
    x = np.zeros((1, 1, 128, 64), np.float64)
    x[0, 0, 1, :32] = -0.0
    x[0, 0, 2, :32] = np.linspace(-511, 511, 32)
    x[0, 0, 3, :32] = np.linspace(-2 ** -20, 2 ** -20, 32)
    x[0, 0, 4, :32] = 2.0 ** np.arange(-16, 16)
    x[0, 0, 5:, :] = np.random.default_rng(4).standard_normal((123, 64)) * 100
    x = x.astype(np.float16)
    _check(w, x, thrift.Q, 1)
    _check(w, x, thrift.V, 1)
