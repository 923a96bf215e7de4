"""CPU oracle for selective mixed-precision (FP16 / NVFP4) block attention.

TEST INFRASTRUCTURE.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package.  It is plain C
(``oracle.c``, FP64 arithmetic, OpenMP over rows) loaded with ctypes, plus the
numpy modules ``vertical_window`` (the HyQuant-style selector), ``tiered``
(FP16 / NVFP4 / skip selection) and ``decode`` (one decode step over the
prefill's caches), and it shares no code with the CUDA library.  See
``oracle.c`` and the modules for what each function computes and which
reading of the method it takes.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SO = os.path.join(_HERE, "liboracle.so")
_lib = None

P_LOG2_DEFAULT = 11  # pre-scale exponent c of P (2^c); 0 = literal reading


class Problem(ctypes.Structure):
    _fields_ = [
        ("Q", ctypes.c_void_p), ("K", ctypes.c_void_p), ("V", ctypes.c_void_p),
        ("q4", ctypes.c_void_p), ("qs", ctypes.c_void_p), ("k4", ctypes.c_void_p), ("ks", ctypes.c_void_p),
        ("v4", ctypes.c_void_p), ("vs", ctypes.c_void_p),
        ("q8", ctypes.c_void_p), ("qs8", ctypes.c_void_p), ("k8", ctypes.c_void_p), ("ks8", ctypes.c_void_p),
        ("v8", ctypes.c_void_p), ("vs8", ctypes.c_void_p),
        ("B", ctypes.c_int), ("Hq", ctypes.c_int), ("Hkv", ctypes.c_int), ("N", ctypes.c_int),
        ("D", ctypes.c_int), ("blk", ctypes.c_int), ("causal", ctypes.c_int),
        ("sm_scale", ctypes.c_float), ("p_log2", ctypes.c_int), ("p_jitter", ctypes.c_double),
    ]


def build(force: bool = False) -> str:
    """Compile ``liboracle.so`` next to this file (gcc, OpenMP)."""
    src = os.path.join(_HERE, "oracle.c")
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(src):
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11",
                               src, "-o", _SO, "-lm"])
    return _SO


def _load():
    global _lib
    if _lib is not None:
        return _lib
    build()
    lib = ctypes.CDLL(_SO)
    vp, i32, i64, f64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_long, ctypes.c_double
    sig = {
        "orc_f16_value": ([ctypes.c_uint16], f64),
        "orc_f16_encode": ([f64], ctypes.c_uint16),
        "orc_e2m1_value": ([ctypes.c_uint8], f64),
        "orc_e2m1_encode": ([f64], ctypes.c_uint8),
        "orc_e4m3_value": ([ctypes.c_uint8], f64),
        "orc_e4m3_encode": ([f64], ctypes.c_uint8),
        "orc_e4m3_encode_direct": ([f64], ctypes.c_uint8),
        "orc_e8m0_value": ([ctypes.c_uint8], f64),
        "orc_quantize_rows": ([vp, i64, i32, vp, vp], i32),
        "orc_quantize_rows_mx8": ([vp, i64, i32, vp, vp], i32),
        "orc_quantize_v_mx8": ([vp, i64, i32, i32, vp, vp], i32),
        "orc_quantize_v": ([vp, i64, i32, i32, vp, vp], i32),
        "orc_budget": ([f64, i64], i64),
        "orc_pooled_scores": ([vp, vp, i32, i32, i32, i32, ctypes.c_float, vp], i32),
        "orc_select": ([vp, vp, i32, i32, i32, i32, i32, i32, i32, ctypes.c_float, f64, vp], i32),
        "orc_attention_rows": ([ctypes.POINTER(Problem), vp, vp, i64, vp, vp], i32),
        "orc_attention_fp4_rows": ([ctypes.POINTER(Problem), vp, i64, vp], i32),
        "orc_exact_rows": ([ctypes.POINTER(Problem), vp, i64, vp], i32),
        "orc_to_f16": ([vp, i64, vp], None),
    }
    for name, (args, res) in sig.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = res
    _lib = lib
    return lib


def _c(a):
    return np.ascontiguousarray(a)


def _bits16(a):
    a = _c(a)
    return a.view(np.uint16) if a.dtype == np.float16 else a.astype(np.uint16)


# ---- scalar formats -------------------------------------------------------
def f16_value(bits: int) -> float:
    return _load().orc_f16_value(bits)


def f16_encode(v: float) -> int:
    return int(_load().orc_f16_encode(v))


def e2m1_value(code: int) -> float:
    return _load().orc_e2m1_value(code)


def e2m1_encode(v: float) -> int:
    return int(_load().orc_e2m1_encode(v))


def e4m3_value(code: int) -> float:
    return _load().orc_e4m3_value(code)


def e4m3_encode(v: float) -> int:
    return int(_load().orc_e4m3_encode(v))


def budget(rho: float, valid: int) -> int:
    return int(_load().orc_budget(rho, valid))


# ---- NVFP4 ------------------------------------------------------------------
def quantize_rows(x):
    """NVFP4 along the last axis: returns codes [..., L/2] (u8, even element in the
    low nibble) and scales [..., L/16] (E4M3 bytes)."""
    x = _bits16(x)
    L = x.shape[-1]
    rows = x.size // L
    codes = np.empty(x.shape[:-1] + (L // 2,), np.uint8)
    scales = np.empty(x.shape[:-1] + (L // 16,), np.uint8)
    if _load().orc_quantize_rows(x.ctypes.data, rows, L, codes.ctypes.data, scales.ctypes.data):
        raise ValueError("orc_quantize_rows: length must be a multiple of 16")
    return codes, scales


def quantize_v(V):
    """NVFP4 of V [B,H,N,D] along keys: codes [B,H,D,N/2], scales [B,H,D,N/16]."""
    V = _bits16(V)
    B, H, N, D = V.shape
    codes = np.empty((B, H, D, N // 2), np.uint8)
    scales = np.empty((B, H, D, N // 16), np.uint8)
    if _load().orc_quantize_v(V.ctypes.data, B * H, N, D, codes.ctypes.data, scales.ctypes.data):
        raise ValueError("orc_quantize_v: N must be a multiple of 16")
    return codes, scales


def e4m3_encode_direct(v: float) -> int:
    return int(_load().orc_e4m3_encode_direct(float(v)))


def e8m0_value(code: int) -> float:
    return float(_load().orc_e8m0_value(int(code)))


def quantize_rows_mx8(x):
    """MXFP8 along the last axis: codes [..., L] (E4M3 bytes) and scales
    [..., L/32] (E8M0 bytes)."""
    x = _bits16(x)
    L = x.shape[-1]
    rows = x.size // L
    codes = np.empty(x.shape, np.uint8)
    scales = np.empty(x.shape[:-1] + (L // 32,), np.uint8)
    if _load().orc_quantize_rows_mx8(x.ctypes.data, rows, L, codes.ctypes.data, scales.ctypes.data):
        raise ValueError("orc_quantize_rows_mx8: length must be a multiple of 32")
    return codes, scales


def quantize_v_mx8(V):
    """MXFP8 of V [B,H,N,D] along keys: codes [B,H,D,N], scales [B,H,D,N/32]."""
    V = _bits16(V)
    B, H, N, D = V.shape
    codes = np.empty((B, H, D, N), np.uint8)
    scales = np.empty((B, H, D, N // 32), np.uint8)
    if _load().orc_quantize_v_mx8(V.ctypes.data, B * H, N, D, codes.ctypes.data, scales.ctypes.data):
        raise ValueError("orc_quantize_v_mx8: N must be a multiple of 32")
    return codes, scales


def dequantize_mx8(codes, scales):
    """Decode MXFP8 codes / scales along the last axis into float64 (test helper)."""
    codes = np.asarray(codes, np.uint8)
    vals = np.array([e4m3_value(c) for c in range(256)])[codes]
    sc = np.array([e8m0_value(e) for e in range(256)])[np.asarray(scales, np.uint8)]
    return vals * np.repeat(sc, 32, axis=-1)


def dequantize(codes, scales):
    """Decode NVFP4 codes/scales along the last axis into float64 (test helper)."""
    lut = np.array([e2m1_value(c) for c in range(16)])
    slut = np.array([e4m3_value(c) for c in range(256)])
    lo = lut[codes & 15]
    hi = lut[codes >> 4]
    vals = np.stack([lo, hi], axis=-1).reshape(codes.shape[:-1] + (codes.shape[-1] * 2,))
    s = np.repeat(slut[scales], 16, axis=-1)
    return vals * s


# ---- selection -----------------------------------------------------------------
def pooled_scores(Qh, Kh, blk, causal, sm_scale):
    """Pooled scores of one head: Qh [N,D], Kh [N,D] -> float32 [nb,nb] (NaN = invalid)."""
    Qh, Kh = _bits16(Qh), _bits16(Kh)
    N, D = Qh.shape
    nb = N // blk
    out = np.full((nb, nb), np.nan, np.float32)
    if _load().orc_pooled_scores(Qh.ctypes.data, Kh.ctypes.data, N, D, blk, int(causal),
                                 float(sm_scale), out.ctypes.data):
        raise ValueError("orc_pooled_scores rejected the shape")
    return out


def select(Q, K, blk, causal, sm_scale, rho):
    """Selection mask [B,Hq,nb,nb] (u8, 1 = FP16 pair)."""
    Q, K = _bits16(Q), _bits16(K)
    B, Hq, N, D = Q.shape
    Hkv = K.shape[1]
    nb = N // blk
    mask = np.zeros((B, Hq, nb, nb), np.uint8)
    if _load().orc_select(Q.ctypes.data, K.ctypes.data, B, Hq, Hkv, N, D, blk, int(causal),
                          float(sm_scale), float(rho), mask.ctypes.data):
        raise ValueError("orc_select rejected the shape")
    return mask


def select_tiered(Q, K, blk, causal, sm_scale, rho, sigma, rho8=0.0):
    """Mask [B,Hq,nb,nb] (u8: 1 FP16, 3 MXFP8, 0 NVFP4, 2 skip) of the tiered
    selection (``tiered``) on the pooled scores of every (batch, query head)."""
    from . import tiered
    B, Hq = Q.shape[:2]
    group = Hq // K.shape[1]
    nb = Q.shape[2] // blk
    mask = np.zeros((B, Hq, nb, nb), np.uint8)
    for b in range(B):
        for h in range(Hq):
            sc = pooled_scores(Q[b, h], K[b, h // group], blk, causal, sm_scale)
            mask[b, h] = tiered.select_head(sc, causal, rho, sigma, budget, rho8)
    return mask


def select_vertical_window(Q, K, blk, causal, sm_scale, rho, window):
    """Mask [B,Hq,nb,nb] (u8) of the vertical-line / local-window selector
    (``vertical_window``) on the pooled scores of every (batch, query head)."""
    from . import vertical_window as vw
    B, Hq = Q.shape[:2]
    group = Hq // K.shape[1]
    nb = Q.shape[2] // blk
    mask = np.zeros((B, Hq, nb, nb), np.uint8)
    for b in range(B):
        for h in range(Hq):
            sc = pooled_scores(Q[b, h], K[b, h // group], blk, causal, sm_scale)
            mask[b, h] = vw.select_head(sc, causal, rho, window, budget)
    return mask


# ---- attention -------------------------------------------------------------------
class Quantised:
    """Oracle NVFP4 copies of Q, K (along D) and V (along keys); with mx8, also
    the MXFP8 copies that 8-bit pairs (mask value 3) read."""

    def __init__(self, Q, K, V, mx8=False):
        self.q4, self.qs = quantize_rows(Q)
        self.k4, self.ks = quantize_rows(K)
        self.v4, self.vs = quantize_v(V)
        self.q8 = self.qs8 = self.k8 = self.ks8 = self.v8 = self.vs8 = None
        if mx8:
            self.q8, self.qs8 = quantize_rows_mx8(Q)
            self.k8, self.ks8 = quantize_rows_mx8(K)
            self.v8, self.vs8 = quantize_v_mx8(V)


def _problem(Q, K, V, qz, blk, causal, sm_scale, p_log2, keep, p_jitter=0.0):
    Q, K, V = _bits16(Q), _bits16(K), _bits16(V)
    keep.extend([Q, K, V])
    B, Hq, N, D = Q.shape
    Hkv = K.shape[1]
    ptrs = [None] * 6
    if qz is not None:
        arrs = [_c(qz.q4), _c(qz.qs), _c(qz.k4), _c(qz.ks), _c(qz.v4), _c(qz.vs)]
        keep.extend(arrs)
        ptrs = [a.ctypes.data for a in arrs]
    ptrs8 = [None] * 6
    if qz is not None and getattr(qz, "q8", None) is not None:
        arrs = [_c(qz.q8), _c(qz.qs8), _c(qz.k8), _c(qz.ks8), _c(qz.v8), _c(qz.vs8)]
        keep.extend(arrs)
        ptrs8 = [a.ctypes.data for a in arrs]
    return Problem(Q.ctypes.data, K.ctypes.data, V.ctypes.data, *ptrs, *ptrs8, B, Hq, Hkv, N, D, blk,
                   int(causal), float(sm_scale), int(p_log2), float(p_jitter))


def attention_rows(Q, K, V, mask, rows, blk, causal, sm_scale, qz=None, order=None,
                   p_log2=P_LOG2_DEFAULT, p_jitter=0.0):
    """Mixed-precision attention output (float64, before fp16 rounding) for rows
    [(b, h, r), ...] -> [nrows, D].  p_jitter (tests only): encode P * (1 +
    p_jitter) instead of P, to resolve E2M1 / fp16 rounding ties the other way."""
    keep = []
    if qz is None:
        qz = Quantised(Q, K, V)
    p = _problem(Q, K, V, qz, blk, causal, sm_scale, p_log2, keep, p_jitter)
    rows = _c(np.asarray(rows, np.int64).reshape(-1, 3))
    mask = _c(np.asarray(mask, np.uint8))
    out = np.empty((rows.shape[0], p.D), np.float64)
    order_arr = None
    if order is not None:
        order_arr = _c(np.asarray(order, np.int32))
    rc = _load().orc_attention_rows(ctypes.byref(p), mask.ctypes.data, rows.ctypes.data, rows.shape[0],
                                    None if order_arr is None else order_arr.ctypes.data, out.ctypes.data)
    if rc == 2:
        raise ValueError("8-bit pairs (mask 3) need Quantised(..., mx8=True)")
    if rc:
        raise ValueError("orc_attention_rows rejected the shape")
    return out


def attention_fp4_rows(Q, K, V, rows, blk, causal, sm_scale, qz=None, p_log2=P_LOG2_DEFAULT):
    """Pure-FP4 attention written directly (no mask, two passes)."""
    keep = []
    if qz is None:
        qz = Quantised(Q, K, V)
    p = _problem(Q, K, V, qz, blk, causal, sm_scale, p_log2, keep)
    rows = _c(np.asarray(rows, np.int64).reshape(-1, 3))
    out = np.empty((rows.shape[0], p.D), np.float64)
    if _load().orc_attention_fp4_rows(ctypes.byref(p), rows.ctypes.data, rows.shape[0], out.ctypes.data):
        raise ValueError("orc_attention_fp4_rows rejected the shape")
    return out


def exact_rows(Q, K, V, rows, causal, sm_scale, blk=16):
    """Exact FP64 softmax(Q K^T sm_scale) V for the given rows."""
    keep = []
    p = _problem(Q, K, V, None, blk, causal, sm_scale, 0, keep)
    rows = _c(np.asarray(rows, np.int64).reshape(-1, 3))
    out = np.empty((rows.shape[0], p.D), np.float64)
    if _load().orc_exact_rows(ctypes.byref(p), rows.ctypes.data, rows.shape[0], out.ctypes.data):
        raise ValueError("orc_exact_rows rejected the shape")
    return out


def to_f16(x):
    """Round float64 values to fp16 with the oracle's own rounding."""
    x = _c(np.asarray(x, np.float64))
    out = np.empty(x.shape, np.uint16)
    _load().orc_to_f16(x.ctypes.data, x.size, out.ctypes.data)
    return out.view(np.float16)


def all_rows(B, H, N):
    """Every (b, h, r) of a problem."""
    b, h, r = np.meshgrid(np.arange(B), np.arange(H), np.arange(N), indexing="ij")
    return np.stack([b.ravel(), h.ravel(), r.ravel()], axis=1).astype(np.int64)


def gap_recovered(o_fp4, o_mixed, o_fp16, o_exact):
    """Share (percent) of the FP4-to-FP16 error gap that the mixed output
    recovers: errors are relative Frobenius distances to the exact output."""
    def err(o):
        return np.linalg.norm(o - o_exact) / np.linalg.norm(o_exact)
    e4, em, e16 = err(o_fp4), err(o_mixed), err(o_fp16)
    return 100.0 * (e4 - em) / (e4 - e16)
