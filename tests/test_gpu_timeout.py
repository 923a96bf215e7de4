"""Failure detection on the GPU: a bounded wait that runs out (no GPU fault).

Every wait inside the attention and decode kernels is bounded (thrift_set_wait_limit).
Here the wait limit is set to 1 ms and the producer of every CTA withholds the
copies of one key tile (THRIFT_TEST_WITHHOLD_TILE: its ring slot is taken but
nothing is ever copied into it, so the barrier its consumers wait on is never
completed -- a flag that nothing sets).  Each such CTA must notice within the
limit, record THRIFT_ERR_TIMEOUT in the device error word, let every role leave
its loop, drain its copies and tensor-core work and return without writing its
output; CTAs whose query tiles never reach that key tile finish normally.  The
next call in the same process, with the defaults restored, must match the
oracle.
"""
import time

import numpy as np
import pytest
import torch

import fp16_block_attention_b200 as thrift
import oracle
import synth
from gpu_helpers import ATOL_MAX, ATOL_MEAN, compare_o, shape_of, to_dev

THRIFT_ERR_TIMEOUT = 4
WITHHELD = 2  # processed key tile whose copies are withheld

CASES = [
    # (workload, selection), blk 128: the double-buffered kernel (method and skip-aware instantiations)
    (synth.GQA_N32K.with_(N=768, Hq=4, Hkv=2, rho=0.1), "method"),
    (synth.GQA_N32K.with_(N=768, Hq=4, Hkv=2, rho=0.1), "skip"),
    # blk 64: the one-pass kernel
    (synth.CAUSAL_MH_N8K.with_(N=768, Hq=2, Hkv=2, blk=64, rho=0.1), "method"),
]


def mask_of(kind, Qd, Kd, sh, w):
    if kind == "skip":
        return thrift.select_blocks_tiered(Qd, Kd, sh, w.rho, 0.3).cpu().numpy()
    return thrift.select_blocks(Qd, Kd, sh, w.rho).cpu().numpy()


def _attend(kind, Qd, Kd, Vd, sh, w, out):
    qz = thrift.quantize_all(Qd, Kd, Vd, sh)
    if kind == "skip":
        mask = thrift.select_blocks_tiered(Qd, Kd, sh, w.rho, 0.3)
        thrift.attention_tiered(Qd, Kd, Vd, mask, qz, sh, out=out)
    else:
        mask = thrift.select_blocks(Qd, Kd, sh, w.rho)
        thrift.attention(Qd, Kd, Vd, mask, qz, sh, out=out)
    return mask


@pytest.mark.gpu
@pytest.mark.parametrize("w,kind", CASES, ids=lambda c: c.name if hasattr(c, "name") else c)
def test_a_wait_that_runs_out_is_reported_and_the_next_call_is_unaffected(w, kind, monkeypatch):
    Q, K, V = synth.generate(w)
    Qd, Kd, Vd = to_dev(Q, K, V)
    sh = shape_of(w)
    assert thrift.last_device_error() == 0
    sentinel = torch.full_like(Qd, float("nan"))
    try:
        thrift.set_wait_limit(1_000_000)  # 1 ms
        monkeypatch.setenv("THRIFT_TEST_WITHHOLD_TILE", str(WITHHELD))
        torch.cuda.synchronize()
        t0 = time.perf_counter()
        out = sentinel.clone()
        _attend(kind, Qd, Kd, Vd, sh, w, out)
        status = thrift.last_device_error()  # synchronises
        elapsed = time.perf_counter() - t0
    finally:
        monkeypatch.delenv("THRIFT_TEST_WITHHOLD_TILE", raising=False)
        thrift.set_wait_limit(thrift.WAIT_LIMIT_DEFAULT_NS)
    assert status == THRIFT_ERR_TIMEOUT
    assert elapsed < 1.0, elapsed
    # A query tile is abandoned exactly when it processes more key tiles than
    # WITHHELD (key tiles are 128 wide in both kernels): its rows keep the
    # sentinel, every other row is written.
    m = mask_of(kind, Qd, Kd, sh, w)
    nt = (w.N + 127) // 128
    if kind == "skip":
        processed = np.array([[[int((m[b, h, qt, :qt + 1] != 2).sum()) for qt in range(nt)]
                               for h in range(w.Hq)] for b in range(w.B)])
    else:
        processed = np.broadcast_to(np.arange(1, nt + 1), (w.B, w.Hq, nt))
    abandoned = np.repeat(processed > WITHHELD, 128, axis=-1)[:, :, :w.N]
    assert abandoned.any() and not abandoned.all()
    untouched = np.isnan(out.cpu().numpy().astype(np.float32)).all(axis=-1)
    assert np.array_equal(untouched, abandoned)

    # the next call, with the defaults restored, is correct
    out2 = torch.empty_like(Qd)
    mask = _attend(kind, Qd, Kd, Vd, sh, w, out2)
    assert thrift.last_device_error() == 0
    rows = oracle.all_rows(w.B, w.Hq, w.N)
    m = mask.cpu().numpy()
    ref = oracle.to_f16(oracle.attention_rows(Q, K, V, m, rows, w.blk, w.causal, w.sm_scale))
    mx, mean = compare_o(out2.cpu().numpy().reshape(-1, w.D), ref)
    assert mx <= ATOL_MAX and mean <= ATOL_MEAN, (mx, mean)


def test_wait_limit_is_checked_on_the_host():
    lib = thrift.lib()
    assert lib.thrift_set_wait_limit(999) == 1
    assert lib.thrift_set_wait_limit(60_000_000_001) == 1
    assert lib.thrift_set_wait_limit(thrift.WAIT_LIMIT_DEFAULT_NS) == 0


# Decode: both passes' K producers withhold their third K tile; with a 32k
# cache every CTA of both passes takes at least three K tiles.  4, 8 and 16
# query heads per kv head: two softmax groups and a V scale copier, one group
# and a copier, one group without a copier.
DECODE_CASES = [synth.GQA_N32K.with_(Hq=8, Hkv=2), synth.GQA_N32K.with_(Hq=16, Hkv=2),
                synth.GQA_N32K.with_(Hq=32, Hkv=2)]


@pytest.mark.gpu
@pytest.mark.parametrize("w", DECODE_CASES, ids=lambda w: f"G{w.Hq // w.Hkv}")
def test_a_decode_wait_that_runs_out_is_reported_and_the_next_call_is_unaffected(w, monkeypatch):
    from oracle import decode

    Q, K, V = synth.generate(w)
    q = np.ascontiguousarray(Q[:, :, -1])
    del Q
    qd, Kd, Vd = to_dev(q, K, V)
    sh = shape_of(w)
    rho = 0.3
    m_ref = decode.select(q, K, w.blk, w.sm_scale, rho, oracle.budget)
    md, = to_dev(m_ref)
    kq = thrift.quantize_kv(Kd, Vd, sh)
    assert thrift.last_device_error() == 0
    try:
        thrift.set_wait_limit(1_000_000)  # 1 ms
        monkeypatch.setenv("THRIFT_TEST_WITHHOLD_TILE", str(WITHHELD))
        torch.cuda.synchronize()
        t0 = time.perf_counter()
        thrift.decode_attention(qd, Kd, Vd, kq, md, sh)
        status = thrift.last_device_error()  # synchronises
        elapsed = time.perf_counter() - t0
    finally:
        monkeypatch.delenv("THRIFT_TEST_WITHHOLD_TILE", raising=False)
        thrift.set_wait_limit(thrift.WAIT_LIMIT_DEFAULT_NS)
    assert status == THRIFT_ERR_TIMEOUT
    assert elapsed < 1.0, elapsed

    # the next call, with the defaults restored, is correct
    out = thrift.decode_attention(qd, Kd, Vd, kq, md, sh)
    assert thrift.last_device_error() == 0
    heads = [(0, h) for h in range(w.Hq)]
    ref = oracle.to_f16(decode.attention(q, K, V, m_ref, w.blk, w.sm_scale, heads))
    got = out.cpu().numpy().reshape(-1, w.D)
    mx, mean = compare_o(got, ref)
    assert mx <= ATOL_MAX and mean <= ATOL_MEAN, (mx, mean)
