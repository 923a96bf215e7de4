"""Pin of the oracle's NVFP4 path (no GPU).

The ThriftAttention abstract computes every block pair that the heuristic does
not pick in FP4: S from the block-scaled FP4 copies of Q and K, P encoded per
16 keys, and P V from the FP4 copy of V.  At rho = 0 every pair takes that
path.  Here that output is written out a second time in numpy, outside
``oracle.c``.  The restatement shares none of the oracle's decoders or
encoders:
  - E2M1 codes decode from the format's literal grid;
  - E4M3 scale bytes decode and encode through torch's float8_e4m3fn;
  - S is one FP64 matrix product of the decoded operands;
  - the online softmax keeps the integer running maximum block by block.
The comparison is made on a single key tile, where the output has the closed
form sum(P~ V~) / sum(P) with M = ceil(max t), and on a causal run of four
tiles.  A slip in the oracle's decoding of the Q and K codes fails the
comparison: a nibble swap, a scale taken from the neighbouring row or group,
or Q read with K's scales.
The last test plants each of these slips in the restatement and checks that
the comparison notices it.
"""
import math

import numpy as np
import pytest
import torch

import oracle

LOG2E = 1.4426950408889634073599246810019
P_LOG2 = 11

# E2M1 magnitudes by the low three bits of a code (bit 3 is the sign): the
# format's grid, 0, 0.5 (subnormal), then 1 + m/2 times 2^(e-1).
E2M1_GRID = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def e2m1_decode(codes):
    codes = np.asarray(codes, np.uint8)
    mag = E2M1_GRID[codes & 7]
    return np.where(codes & 8, -mag, mag)


def e4m3_decode(bytes_):
    b = torch.from_numpy(np.ascontiguousarray(np.asarray(bytes_, np.uint8)))
    return b.view(torch.float8_e4m3fn).to(torch.float64).numpy()


def e4m3_encode(v32):
    """Nearest E4M3 byte to FP32 values (torch's conversion, ties to even)."""
    t = torch.from_numpy(np.ascontiguousarray(np.asarray(v32, np.float32)))
    return t.to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def e2m1_round(x):
    """Nearest E2M1 value, ties to the even code, saturating at 6 (values only)."""
    a = np.abs(np.asarray(x, np.float64))
    d = np.abs(a[..., None] - E2M1_GRID)
    cand = d == d.min(axis=-1, keepdims=True)  # the nearest magnitude, or two at a tie
    even = cand & (np.arange(8) % 2 == 0)
    pick = np.where(even.any(axis=-1), np.argmax(even, axis=-1), np.argmax(cand, axis=-1))
    return np.where(np.signbit(x), -1.0, 1.0) * E2M1_GRID[pick]


def decode_rows(codes, scales):
    """NVFP4 along the last axis: element 2k in the low nibble of byte k,
    scale g covering elements 16g .. 16g + 15."""
    codes = np.asarray(codes, np.uint8)
    lo, hi = e2m1_decode(codes & 15), e2m1_decode(codes >> 4)
    vals = np.stack([lo, hi], axis=-1).reshape(codes.shape[:-1] + (2 * codes.shape[-1],))
    return vals * np.repeat(e4m3_decode(scales), 16, axis=-1)


def encode_p(P):
    """P (FP32 values) encoded at the pre-scale 2^11 per aligned 16 keys:
    scale = E4M3(fl32(amax / 6)), value = E2M1(x / scale) * scale, then / 2^11."""
    x = P.astype(np.float64).reshape(-1, 16) * 2.0 ** P_LOG2
    amax = np.abs(x).max(axis=1)
    s = e4m3_decode(e4m3_encode((amax / 6.0).astype(np.float32)))
    safe = np.where(s > 0, s, 1.0)
    q = np.where(s[:, None] > 0, e2m1_round(x / safe[:, None]) * s[:, None], 0.0)
    return q.reshape(-1) * 2.0 ** -P_LOG2


def fp4_row(Qd, Kd, Vd, r, blk, causal, sm_scale):
    """One output row at rho = 0 by the online softmax with an integer running
    maximum.  Qd [N, D] and Kd [N, D] are the decoded FP4 copies, Vd [D, N]
    the decoded copy of V along keys."""
    N = Kd.shape[0]
    c = np.float32(np.float64(sm_scale) * LOG2E)
    nblk = (r // blk + 1) if causal else N // blk
    M, l = -math.inf, 0.0
    acc = np.zeros(Vd.shape[0])
    for j in range(nblk):
        keys = np.arange(j * blk, (j + 1) * blk)
        S = Kd[keys] @ Qd[r]  # FP64
        t = (np.float32(S).astype(np.float64) * np.float64(c)).astype(np.float32)
        if causal:
            t = np.where(keys > r, np.float32(-np.inf), t)
        Mn = max(M, math.ceil(float(t.max())))
        if M != -math.inf and Mn > M:
            a = 2.0 ** (M - Mn)
            l *= a
            acc *= a
        M = Mn
        P = np.where(np.isinf(t), 0.0, np.exp2(t.astype(np.float64) - M)).astype(np.float32)
        l += float(P.astype(np.float64).sum())
        acc += encode_p(P) @ Vd[:, keys].T
    return acc / l


def _problem(seed, B, Hq, Hkv, N, D, spread):
    rng = np.random.default_rng(seed)
    # a spread of magnitudes over the channels, so groups take many scales
    mag = np.exp(rng.uniform(-spread, spread, D))
    Q = (rng.standard_normal((B, Hq, N, D)) * mag).astype(np.float16)
    K = (rng.standard_normal((B, Hkv, N, D)) * mag[::-1]).astype(np.float16)
    V = rng.standard_normal((B, Hkv, N, D)).astype(np.float16)
    return Q, K, V


def _decoded(qz, b, h, hk):
    Qd = decode_rows(qz.q4[b, h], qz.qs[b, h])
    Kd = decode_rows(qz.k4[b, hk], qz.ks[b, hk])
    Vd = decode_rows(qz.v4[b, hk], qz.vs[b, hk])  # [D, N]
    return Qd, Kd, Vd


CASES = [
    # single key tile (N = blk): the closed form
    dict(seed=11, B=1, Hq=2, Hkv=1, N=128, D=128, blk=128, causal=False, spread=1.0),
    dict(seed=12, B=1, Hq=1, Hkv=1, N=64, D=64, blk=64, causal=False, spread=1.5),
    # causal, four key tiles, GQA
    dict(seed=13, B=1, Hq=4, Hkv=2, N=512, D=128, blk=128, causal=True, spread=1.0),
    dict(seed=14, B=2, Hq=2, Hkv=1, N=256, D=64, blk=64, causal=True, spread=0.5),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"N{c['N']}-D{c['D']}-blk{c['blk']}-{'causal' if c['causal'] else 'full'}")
def test_rho_zero_rows_equal_an_independent_restatement(case):
    B, Hq, Hkv, N, D, blk, causal = (case[k] for k in ("B", "Hq", "Hkv", "N", "D", "blk", "causal"))
    Q, K, V = _problem(case["seed"], B, Hq, Hkv, N, D, case["spread"])
    sm_scale = 1.0 / math.sqrt(D)
    qz = oracle.Quantised(Q, K, V)
    nb = N // blk
    mask = np.zeros((B, Hq, nb, nb), np.uint8)  # rho = 0: every pair in FP4
    rng = np.random.default_rng(case["seed"] + 100)
    rows = [(b, h, int(r)) for b in range(B) for h in range(Hq)
            for r in sorted(set(rng.integers(0, N, 12).tolist()) | {0, N - 1, blk - 1})]
    got = oracle.attention_rows(Q, K, V, mask, rows, blk, causal, sm_scale, qz=qz)
    group = Hq // Hkv
    worst = 0.0
    for i, (b, h, r) in enumerate(rows):
        Qd, Kd, Vd = _decoded(qz, b, h, h // group)
        ref = fp4_row(Qd, Kd, Vd, r, blk, causal, sm_scale)
        err = np.abs(got[i] - ref).max() / max(1.0, np.abs(ref).max())
        worst = max(worst, err)
    assert worst <= 1e-12, worst


def test_single_tile_closed_form():
    """N = blk: O = sum_k P~_k V~_k / sum_k P_k, P = fl32(2^(t - ceil(max t)))."""
    Q, K, V = _problem(21, 1, 1, 1, 128, 128, 1.0)
    qz = oracle.Quantised(Q, K, V)
    sm_scale = 1.0 / math.sqrt(128)
    Qd, Kd, Vd = _decoded(qz, 0, 0, 0)
    c = np.float32(np.float64(sm_scale) * LOG2E)
    S = Kd @ Qd.T  # [keys, rows]
    t = (np.float32(S).astype(np.float64) * np.float64(c)).astype(np.float32)
    M = np.ceil(t.max(axis=0).astype(np.float64))
    P = np.exp2(t.astype(np.float64) - M).astype(np.float32)  # [keys, rows]
    Pt = np.stack([encode_p(P[:, r]) for r in range(128)], axis=1)
    ref = (Vd @ Pt).T / P.astype(np.float64).sum(axis=0)[:, None]
    got = oracle.attention_rows(Q, K, V, np.zeros((1, 1, 1, 1), np.uint8),
                                [(0, 0, r) for r in range(128)], 128, False, sm_scale, qz=qz)
    assert np.abs(got - ref).max() <= 1e-12 * max(1.0, np.abs(ref).max())


def test_restatement_notices_planted_decoding_slips():
    """Each plausible slip in decoding the Q and K codes moves the output far
    outside the 1e-12 bar, so the comparison above would catch it."""
    Q, K, V = _problem(31, 1, 1, 1, 256, 128, 1.0)
    qz = oracle.Quantised(Q, K, V)
    sm_scale = 1.0 / math.sqrt(128)
    rows = [(0, 0, r) for r in (5, 100, 200, 255)]
    got = oracle.attention_rows(Q, K, V, np.zeros((1, 1, 2, 2), np.uint8), rows, 128, True, sm_scale, qz=qz)

    def swap_nibbles(c):
        return ((c & 15) << 4) | (c >> 4)

    Qd, Kd, Vd = _decoded(qz, 0, 0, 0)
    slips = {
        "nibble swap in Q": (decode_rows(swap_nibbles(qz.q4[0, 0]), qz.qs[0, 0]), Kd),
        "nibble swap in K": (Qd, decode_rows(swap_nibbles(qz.k4[0, 0]), qz.ks[0, 0])),
        "Q read with K's scales": (decode_rows(qz.q4[0, 0], qz.ks[0, 0]), Kd),
        "K row read with the previous row's scales": (Qd, decode_rows(qz.k4[0, 0], np.roll(qz.ks[0, 0], 1, axis=0))),
        "Q scale of the previous 16-element group": (decode_rows(qz.q4[0, 0], np.roll(qz.qs[0, 0], 1, axis=-1)), Kd),
    }
    for name, (Qs, Ks) in slips.items():
        diff = max(np.abs(got[i] - fp4_row(Qs, Ks, Vd, r, 128, True, sm_scale)).max()
                   for i, (_, _, r) in enumerate(rows))
        assert diff > 1e-3, name
    exact = max(np.abs(got[i] - fp4_row(Qd, Kd, Vd, r, 128, True, sm_scale)).max()
                for i, (_, _, r) in enumerate(rows))
    assert exact <= 1e-12
