"""Sequence-length sweep of the gap-recovered proxy: the share of the
FP4-to-FP16 error gap that rho = 5% of FP16 block pairs recovers, on the
generator of the causal GQA workload at N = 4k .. 128k.  The abstract of
"ThriftAttention: Selective Mixed Precision for Long-Context FP4 Attention"
states that the method's advantage grows with sequence length; this sweep
looks at that shape through the proxy, on synthetic inputs.

At every length the GPU's gap on sampled rows must agree with the oracle's
within one point (the acceptance bar for the gap).  Run with -s to see the
series: one line per length with the three relative errors and both gaps,
and the gap of the vertical-line / local-window selector on the same budget
(its parity with the oracle is in test_gpu_vertical_window)."""
import numpy as np
import pytest

import fp16_block_attention_b200 as thrift
import oracle
import synth
from gpu_helpers import shape_of, to_dev

pytestmark = pytest.mark.gpu

LENGTHS = [4096, 8192, 16384, 32768, 65536, 131072]


def _rel_err(o, ex):
    return float(np.linalg.norm(o - ex) / np.linalg.norm(ex))


@pytest.mark.parametrize("N", LENGTHS)
def test_gap_recovered_by_sequence_length(N):
    w = synth.GQA_N32K.with_(N=N)
    Q, K, V = synth.generate(w)
    Qd, Kd, Vd = to_dev(Q, K, V)
    sh = shape_of(w)
    rows = synth.sample_rows(w, 48, per_block=8)
    qz = oracle.Quantised(Q, K, V)
    ex = oracle.exact_rows(Q, K, V, rows, w.causal, w.sm_scale)
    gpu, ref = {}, {}
    for rho in (0.0, w.rho, 1.0):
        o = thrift.attention_fused(Qd, Kd, Vd, sh, rho).cpu().numpy()
        assert thrift.last_device_error() == 0
        gpu[rho] = o[rows[:, 0], rows[:, 1], rows[:, 2]].astype(np.float64)
        m = oracle.select(Q, K, w.blk, w.causal, w.sm_scale, rho)
        ref[rho] = oracle.to_f16(oracle.attention_rows(Q, K, V, m, rows, w.blk, w.causal, w.sm_scale, qz)
                                 ).astype(np.float64)
    g = oracle.gap_recovered(gpu[0.0], gpu[w.rho], gpu[1.0], ex)
    r = oracle.gap_recovered(ref[0.0], ref[w.rho], ref[1.0], ex)
    # the vertical-line / local-window selector (window of one block) on the same budget
    m_vw = thrift.select_blocks_vertical_window(Qd, Kd, sh, w.rho, 1)
    o_vw = thrift.attention(Qd, Kd, Vd, m_vw, thrift.quantize_all(Qd, Kd, Vd, sh), sh).cpu().numpy()
    assert thrift.last_device_error() == 0
    g_vw = oracle.gap_recovered(gpu[0.0], o_vw[rows[:, 0], rows[:, 1], rows[:, 2]].astype(np.float64), gpu[1.0], ex)
    print(f"\ngap sweep N={N}: E(rho=0)={_rel_err(gpu[0.0], ex):.5f} E(rho={w.rho})={_rel_err(gpu[w.rho], ex):.5f} "
          f"E(rho=1)={_rel_err(gpu[1.0], ex):.5f} gap_gpu={g:.2f} gap_oracle={r:.2f} gap_vertical_window={g_vw:.2f}")
    assert abs(g - r) <= 1.0, (g, r)
