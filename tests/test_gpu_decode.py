"""Parity of the decode step on the GPU (through the C ABI) with its oracle.

The query of each (batch, query head) is the generator's query of the last
position, q = Q[:, :, N - 1], over the cache of the N keys.  Bars as for
prefill: block means bit-exact; selection masks bit-exact except for blocks
whose score lies within 1e-5 (relative) of the k-th selected score; outputs
within max-abs 2e-2 and mean-abs 1e-3 of the oracle's fp16 output (the
oracle gets the GPU's inputs and the oracle's own mask).
"""
import numpy as np
import pytest
import torch

import fp16_block_attention_b200 as thrift
import oracle
import synth
from oracle import decode
from gpu_helpers import ATOL_MAX, ATOL_MEAN, compare_o, shape_of, to_dev

pytestmark = pytest.mark.gpu

SMALL = [
    synth.GQA_N32K.with_(N=1024, Hq=4, Hkv=2),                      # GQA, 8 tiles
    synth.GQA_N32K.with_(N=128, Hq=4, Hkv=1),                       # a single key tile
    synth.BATCHED_GQA_N16K.with_(N=2048, B=2, Hq=14, Hkv=2),        # 7 heads per kv head, batched
    synth.CAUSAL_MH_N8K.with_(N=1536, Hq=2, Hkv=2, blk=128),        # one head per kv head
    synth.GQA_N32K.with_(N=896, Hq=16, Hkv=1),                      # 16 heads per kv head (the most)
    synth.GQA_N32K.with_(N=3712, B=2, Hq=32, Hkv=16),               # many units, the last chunk ragged
    synth.GQA_N32K.with_(N=4864, B=2, Hq=128, Hkv=8),               # 16 heads per kv head, two chunks per CTA
]
FULL = [synth.GQA_N32K, synth.BATCHED_GQA_N16K, synth.GQA_N128K]


def _ids(ws):
    return [f"{w.name}-N{w.N}-B{w.B}-H{w.Hq}x{w.Hkv}" for w in ws]


_cache = {}


def _data(w):
    if w not in _cache:
        if len(_cache) > 2:
            _cache.clear()
        Q, K, V = synth.generate(w)
        q = np.ascontiguousarray(Q[:, :, -1])
        _cache[w] = (Q, K, V, q)
    return _cache[w]


def _heads(w, limit=None):
    hs = [(b, h) for b in range(w.B) for h in range(w.Hq)]
    if limit is not None and len(hs) > limit:
        rng = np.random.default_rng(5)
        hs = [hs[i] for i in sorted(rng.choice(len(hs), limit, replace=False))]
    return hs


def _mask_ok(w, q, K, m_gpu, rho):
    """Masks equal except blocks within the 1e-5 band of the k-th score."""
    m_ref = decode.select(q, K, w.blk, w.sm_scale, rho, oracle.budget)
    nb = w.N // w.blk
    G = w.Hq // w.Hkv
    for b in range(w.B):
        for h in range(w.Hq):
            diff = m_gpu[b, h] != m_ref[b, h]
            if not diff.any():
                continue
            sc = decode.scores(q[b, h], K[b, h // G], w.blk, w.sm_scale)
            free = np.ones(nb, bool)
            free[[0, nb - 1]] = False
            picked = sc[(m_ref[b, h] == 1) & free]
            if picked.size == 0:
                return False
            kth = picked.min()
            if not np.all(np.abs(sc[diff] - kth) <= 1e-5 * max(abs(kth), 1e-30)):
                return False
    return True


@pytest.mark.parametrize("w", SMALL, ids=_ids(SMALL))
def test_pool_keys_bit_exact(w):
    Q, K, V, q = _data(w)
    Kd, = to_dev(K)
    km = thrift.pool_keys(Kd, shape_of(w)).cpu().numpy()
    for b in range(w.B):
        for h in range(w.Hkv):
            assert np.array_equal(km[b, h], decode.block_means(K[b, h], w.blk))


@pytest.mark.parametrize("rho", [0.0, 0.05, 0.3, 1.0])
@pytest.mark.parametrize("w", SMALL, ids=_ids(SMALL))
def test_decode_select_matches_oracle(w, rho):
    Q, K, V, q = _data(w)
    qd, Kd = to_dev(q, K)
    sh = shape_of(w)
    m = thrift.decode_select(qd, thrift.pool_keys(Kd, sh), sh, rho).cpu().numpy()
    nb = w.N // w.blk
    assert np.all(m.sum(-1) == oracle.budget(rho, nb))
    assert _mask_ok(w, q, K, m, rho)


def _check_attention(w, rho, heads):
    Q, K, V, q = _data(w)
    qd, Kd, Vd = to_dev(q, K, V)
    sh = shape_of(w)
    m_ref = decode.select(q, K, w.blk, w.sm_scale, rho, oracle.budget)
    md, = to_dev(m_ref)
    kq = thrift.quantize_kv(Kd, Vd, sh)
    o = thrift.decode_attention(qd, Kd, Vd, kq, md, sh)
    assert thrift.last_device_error() == 0
    o = o.cpu().numpy()
    ref = oracle.to_f16(decode.attention(q, K, V, m_ref, w.blk, w.sm_scale, heads))
    got = np.stack([o[b, h] for b, h in heads])
    mx, mean = compare_o(got, ref)
    assert mx <= ATOL_MAX and mean <= ATOL_MEAN, (mx, mean)


@pytest.mark.parametrize("rho", [0.0, 0.05, 0.3, 1.0])
@pytest.mark.parametrize("w", SMALL, ids=_ids(SMALL))
def test_decode_attention_matches_oracle(w, rho):
    _check_attention(w, rho, _heads(w))


@pytest.mark.parametrize("w", FULL, ids=_ids(FULL))
def test_decode_attention_matches_oracle_at_full_size(w):
    _check_attention(w, w.rho, _heads(w, limit=8))


@pytest.mark.parametrize("w", [SMALL[0], SMALL[2], SMALL[5]], ids=_ids([SMALL[0], SMALL[2], SMALL[5]]))
def test_decode_step_is_select_then_attention(w):
    Q, K, V, q = _data(w)
    qd, Kd, Vd = to_dev(q, K, V)
    sh = shape_of(w)
    km = thrift.pool_keys(Kd, sh)
    kq = thrift.quantize_kv(Kd, Vd, sh)
    o1 = thrift.decode_step(qd, Kd, Vd, kq, km, sh, 0.1)
    o2 = thrift.decode_attention(qd, Kd, Vd, kq, thrift.decode_select(qd, km, sh, 0.1), sh)
    assert thrift.last_device_error() == 0
    assert torch.equal(o1, o2)


@pytest.mark.parametrize("w", [SMALL[0], SMALL[3]], ids=_ids([SMALL[0], SMALL[3]]))
def test_decode_equals_the_prefill_last_row(w):
    """With q = Q[N - 1] and the prefill mask's last row, decode computes the
    prefill's output row N - 1 (two kernels, the same values)."""
    Q, K, V, q = _data(w)
    Qd, Kd, Vd, qd = to_dev(Q, K, V, q)
    sh = shape_of(w)
    pm = thrift.select_blocks(Qd, Kd, sh, 0.2)
    qz = thrift.quantize_all(Qd, Kd, Vd, sh)
    o_pre = thrift.attention(Qd, Kd, Vd, pm, qz, sh)[:, :, -1].cpu().numpy()
    o_dec = thrift.decode_attention(qd, Kd, Vd, qz, pm[:, :, -1].contiguous(), sh).cpu().numpy()
    assert thrift.last_device_error() == 0
    mx, mean = compare_o(o_dec.reshape(-1, w.D), o_pre.reshape(-1, w.D))
    assert mx <= ATOL_MAX and mean <= ATOL_MEAN, (mx, mean)
