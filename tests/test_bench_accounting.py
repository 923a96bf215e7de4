"""Host-side accounting of bench.py (no GPU): effective FLOPs per precision
class, algorithmic bytes, and the MUFU operation count, checked against
closed forms on small masks."""
import numpy as np
import pytest

import bench
import synth


def _masks(w, seed=0):
    nb = w.N // w.blk
    rng = np.random.default_rng(seed)
    m = rng.choice(np.array([0, 1, 2, 3], np.uint8), size=(w.B, w.Hq, nb, nb))
    if w.causal:
        m &= np.tril(np.ones((nb, nb), np.uint8))[None, None] * 255
    return m


@pytest.mark.parametrize("causal", [True, False])
def test_class_flops_partition_the_dense_count(causal):
    """FLOPs of the four classes add up to the full attention count, 4 D Hq B
    times the (query, key) pairs: N^2, or N (N + 1) / 2 when causal (row r sees
    r + 1 keys)."""
    w = synth.GQA_N32K.with_(N=1024, Hq=4, Hkv=2, causal=causal)
    m = _masks(w)
    parts = [bench.pair_flops(w, m, c) for c in (0, 1, 2, 3)]
    pairs = w.N * (w.N + 1) / 2 if causal else w.N * w.N
    assert sum(parts) == pytest.approx(4.0 * w.D * pairs * w.Hq * w.B, rel=1e-12)
    assert bench.flop_split(w, m) == (parts[1], parts[0])


def test_eight_bytes_count_each_mxfp8_tile_once():
    w = synth.GQA_N32K.with_(N=512, Hq=4, Hkv=2)
    nb = w.N // w.blk
    m = np.zeros((1, 4, nb, nb), np.uint8)
    assert bench.eight_bytes(w, m) == 0
    m[0, 0, 3, 1] = 3      # head 0 (kv head 0): q tile 3, key tile 1
    m[0, 1, 3, 1] = 3      # same kv head and key tile, same query tile of another head
    m[0, 2, 2, 2] = 3      # kv head 1
    per_tile = (1 + 1 / 32) * w.blk * w.D
    # K and V tiles: (kv0, key 1), (kv1, key 2); Q tiles: (h0, 3), (h1, 3), (h2, 2)
    assert bench.eight_bytes(w, m) == pytest.approx(per_tile * (2 * 2 + 3))


def test_mufu_ops_count_exponentials_and_group_scales():
    w = synth.GQA_N32K.with_(N=512, Hq=2, Hkv=1, causal=False)
    nb = w.N // w.blk
    keys = w.N * w.N * w.Hq                       # (query, key) pairs, non-causal
    for cls, extra in ((1, 0.0), (0, 2.0 / 16), (3, 1.0 / 32)):
        m = np.full((1, w.Hq, nb, nb), cls, np.uint8)
        assert bench.mufu_ops(w, m) == pytest.approx(keys * (1 + extra), rel=1e-12)
    m = np.full((1, w.Hq, nb, nb), 2, np.uint8)   # every pair skipped: nothing to exponentiate
    assert bench.mufu_ops(w, m) == 0
