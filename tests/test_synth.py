"""The seeded input generator: reproducible, independent streams, the stated
value recipes, and correct fp16 rounding."""
import numpy as np

import synth


def test_generator_is_reproducible_and_seeded():
    w = synth.TINY_NONCAUSAL_D64.with_(N=256)
    a = synth.generate(w)
    b = synth.generate(w)
    c = synth.generate(w.with_(seed=1))
    for x, y, z in zip(a, b, c):
        assert np.array_equal(x.view(np.uint16), y.view(np.uint16))
        assert not np.array_equal(x.view(np.uint16), z.view(np.uint16))


def test_plain_normal_moments():
    w = synth.TINY_NONCAUSAL_D64.with_(N=4096, sink=False, n_heavy=0)
    Q, K, V = (a.astype(np.float64) for a in synth.generate(w))
    for x in (Q, K, V):
        assert abs(x.mean()) < 0.02 and abs(x.std() - 1) < 0.02
    assert abs(np.corrcoef(Q.ravel(), K.ravel())[0, 1]) < 0.02


def test_sink_heavy_rows_and_offsets():
    w = synth.TINY_NONCAUSAL_D64
    base = synth.generate(w.with_(sink=False, n_heavy=0))[1].astype(np.float64)
    K = synth.generate(w)[1].astype(np.float64)
    ratio = np.abs(K[0, 0]).sum(1) / np.abs(base[0, 0]).sum(1)
    assert abs(ratio[0] - 8) < 0.01
    heavy = np.where(np.abs(ratio - 4) < 0.01)[0]
    assert len(heavy) == 4 and 0 not in heavy
    assert np.sum(np.abs(ratio - 1) < 0.01) == w.N - 5
    w2 = synth.CAUSAL_MH_N8K.with_(N=2048, Hq=2, Hkv=2, sink=False)
    K2 = synth.generate(w2)[1].astype(np.float64)
    off = K2[0].mean(1)                     # per-(head, channel) offset shared by every token
    assert 1.2 < off.std() < 2.8
    assert abs((K2[0] - off[:, None, :]).std() - 1) < 0.03


def test_rank16_component_is_shared_by_q_and_k():
    w = synth.GQA_N32K.with_(N=2048, Hq=2, Hkv=1, kv_offset=False, sink=False)
    Q, K, _ = (a.astype(np.float64) for a in synth.generate(w))
    # variance per element: 1 + 16 * 3^2 / D
    assert abs(Q.var() - (1 + 16 * 9 / 128)) < 0.1
    # the shared 16-dim subspace: top-16 singular directions of Q and K coincide
    uq = np.linalg.svd(Q[0, 0], full_matrices=False)[2][:16]
    uk = np.linalg.svd(K[0, 0], full_matrices=False)[2][:16]
    assert np.linalg.svd(uq @ uk.T, compute_uv=False).min() > 0.9


def test_batches_have_independent_seeds():
    w = synth.BATCHED_GQA_N16K.with_(N=256, B=2)
    Q = synth.generate(w)[0].view(np.uint16)
    assert not np.array_equal(Q[0], Q[1])


def test_f16_rounding_matches_numpy():
    rng = np.random.default_rng(0)
    vals = np.concatenate([rng.standard_normal(3000) * 10.0 ** rng.integers(-8, 5, 3000),
                           [65504.0, 65519.0, 65520.0, 2.0 ** -24, 2.0 ** -25, 1 + 2.0 ** -11, -0.0]])
    for v in vals:
        with np.errstate(over="ignore"):
            ref = int(np.array(v).astype(np.float16).view(np.uint16))
        assert synth.f16_bits(v) == ref, v
