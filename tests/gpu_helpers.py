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
