"""Test-side helpers for the GPU parity tests: move synthetic inputs to the
device, undo the tensor-core scale layout, and compare with the oracle."""
import numpy as np
import torch

import fp16_block_attention_b200 as thrift
import oracle
import synth

ATOL_MAX = 2e-2   # max |O_gpu - O_oracle| over the compared rows
ATOL_MEAN = 1e-3  # mean |O_gpu - O_oracle|


def shape_of(w: synth.Workload) -> thrift.Shape:
    return thrift.Shape(w.B, w.Hq, w.Hkv, w.N, w.D, w.blk, w.causal, w.sm_scale)


def to_dev(*arrs):
    return [torch.from_numpy(np.ascontiguousarray(a)).cuda() for a in arrs]


def canon_qk_scales(scales: torch.Tensor, B, H, N, D):
    """Tensor-core scale layout -> [B, H, N, D/16]."""
    s = scales.cpu().numpy()
    NT = (N + 127) // 128
    bh, n, g = np.meshgrid(np.arange(B * H), np.arange(N), np.arange(D // 16), indexing="ij")
    idx = thrift.qk_scale_index(bh, n, g, NT, D)
    return s[idx].reshape(B, H, N, D // 16)


def qk_scale_padding(scales: torch.Tensor, B, H, N, D):
    s = scales.cpu().numpy()
    NT = (N + 127) // 128
    if NT * 128 == N:
        return np.zeros(0, np.uint8)
    bh, n, g = np.meshgrid(np.arange(B * H), np.arange(N, NT * 128), np.arange(D // 16), indexing="ij")
    return s[thrift.qk_scale_index(bh, n, g, NT, D)]


def canon_v_scales(scales: torch.Tensor, B, H, N, D):
    """V scale layout -> [B, H, D, N/16]."""
    s = scales.cpu().numpy()
    NT = (N + 127) // 128
    bh, d, n16 = np.meshgrid(np.arange(B * H), np.arange(D), np.arange(N // 16), indexing="ij")
    return s[thrift.v_scale_index(bh, d, n16 * 16, NT)].reshape(B, H, D, N // 16)


def compare_o(o_gpu: np.ndarray, o_ref16: np.ndarray):
    d = np.abs(o_gpu.astype(np.float64) - o_ref16.astype(np.float64))
    return float(d.max()), float(d.mean())


def near_tie_pairs(Q, K, w, rho, kth_rel=1e-5):
    """Per head: boolean [nb, nb] of valid pairs whose oracle score lies within
    kth_rel (relative) of the k-th selected score, where GPU and oracle may differ."""
    nb = w.N // w.blk
    G = w.Hq // w.Hkv
    mask = oracle.select(Q, K, w.blk, w.causal, w.sm_scale, rho)
    out = np.zeros((w.B, w.Hq, nb, nb), bool)
    for b in range(w.B):
        for h in range(w.Hq):
            sc = oracle.pooled_scores(Q[b, h], K[b, h // G], w.blk, w.causal, w.sm_scale)
            sel = mask[b, h] == 1
            valid = ~np.isnan(sc)
            free = valid.copy()
            free[np.arange(nb), np.arange(nb)] = False
            free[:, 0] = False
            picked = sc[sel & free]
            if picked.size == 0:
                continue
            kth = picked.min()
            out[b, h] = valid & (np.abs(sc - kth) <= kth_rel * max(abs(kth), 1e-30))
    return mask, out


TIE_JITTER = 2.0 ** -19  # relative nudge of the oracle's encoded P that resolves rounding ties the other way


def compare_o_with_ties(o_rows, Q, K, V, mask, rows, blk, causal, sm_scale, qz=None):
    """compare_o against the oracle, where a row that misses ATOL_MAX is
    checked again against the oracle with its encoded P nudged by
    +-TIE_JITTER: the pages fix no exp2 accuracy, so a P within ~1e-6 of an
    E2M1 or fp16 rounding boundary may be encoded either way, and in a row
    whose weight sits on one NVFP4 key one such flip moves the output by up
    to one E2M1 step of that key's share.  Returns (max, mean, rows resolved
    by a nudge)."""
    ref = oracle.to_f16(oracle.attention_rows(Q, K, V, mask, rows, blk, causal, sm_scale, qz)).astype(np.float64)
    got = np.asarray(o_rows, np.float64)
    err = np.abs(got - ref)
    bad = np.nonzero(err.max(axis=1) > ATOL_MAX)[0]
    resolved = 0
    for i in bad:
        best = err[i]
        for j in (TIE_JITTER, -TIE_JITTER):
            alt = oracle.to_f16(oracle.attention_rows(Q, K, V, mask, rows[i:i + 1], blk, causal, sm_scale, qz,
                                                      p_jitter=j)).astype(np.float64)[0]
            e = np.abs(got[i] - alt)
            if e.max() < best.max():
                best = e
        if best.max() <= ATOL_MAX:
            resolved += 1
        err[i] = best
    return float(err.max()), float(err.mean()), resolved
