"""Q and K quantised and pooled in one pass, and the selection from those block
means (the fused entry points' path): bit-exact against the separate calls."""
import numpy as np
import pytest
import torch

import fp16_block_attention_b200 as thrift
import synth
from gpu_helpers import shape_of, to_dev

pytestmark = pytest.mark.gpu

CASES = [
    synth.TINY_NONCAUSAL_D64,
    synth.CAUSAL_MH_N8K.with_(N=1024, Hq=2, Hkv=2),
    synth.GQA_N32K.with_(N=2048, Hq=4, Hkv=2),
    synth.GQA_N32K.with_(N=1536 + 64, Hq=2, Hkv=1, blk=64),  # N an odd multiple of 64: a half-filled last tile
    synth.BATCHED_GQA_N16K.with_(N=1024, Hq=4, Hkv=2),
]


@pytest.mark.parametrize("w", CASES, ids=lambda w: f"{w.name}-N{w.N}-blk{w.blk}")
def test_quantize_pool_and_pooled_selection_equal_the_separate_calls(w):
    Q, K, V = synth.generate(w)
    Qd, Kd, Vd = to_dev(Q, K, V)
    sh = shape_of(w)
    q4, qs, qm = thrift.quantize_pool_nvfp4(Qd, thrift.Q, sh)
    k4, ks, km = thrift.quantize_pool_nvfp4(Kd, thrift.K, sh)
    r4, rs = thrift.quantize_nvfp4(Qd, thrift.Q, sh)
    t4, ts = thrift.quantize_nvfp4(Kd, thrift.K, sh)
    assert torch.equal(q4, r4) and torch.equal(qs, rs)
    assert torch.equal(k4, t4) and torch.equal(ks, ts)
    # block means: the pooling kernel of the decode path on K, and on Q viewed as Hq kv heads
    assert torch.equal(km, thrift.pool_keys(Kd, sh))
    shq = thrift.Shape(w.B, w.Hq, w.Hq, w.N, w.D, w.blk, w.causal, w.sm_scale)
    assert torch.equal(qm, thrift.pool_keys(Qd, shq))
    for rho in (0.0, w.rho, 0.3, 1.0):
        m1 = thrift.select_blocks_pooled(qm, km, sh, rho)
        m2 = thrift.select_blocks(Qd, Kd, sh, rho)
        assert torch.equal(m1, m2), rho
    assert thrift.last_device_error() == 0
