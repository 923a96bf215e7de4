"""Seeded synthetic inputs for the selective FP4/FP16 attention path.

The five named workloads follow the workload descriptions of the method's
evaluation (prefill attention on long contexts); the pages name no public
dataset for them, so these generators stand in for it.  The module draws
random numbers only: no quantisation, selection or attention arithmetic lives
here.  Both the CPU oracle (tests) and the CUDA library are fed from it.

The generator is plain C (``synth.c``) loaded with ctypes; ``build()``
compiles it with gcc.
"""
from __future__ import annotations

import ctypes
import dataclasses
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SO = os.path.join(_HERE, "libsynth.so")
_lib = None


class _Recipe(ctypes.Structure):
    _fields_ = [
        ("B", ctypes.c_int), ("Hq", ctypes.c_int), ("Hkv", ctypes.c_int),
        ("N", ctypes.c_int), ("D", ctypes.c_int),
        ("kv_offset", ctypes.c_int), ("offset_sd", ctypes.c_double),
        ("sink", ctypes.c_int), ("sink_scale", ctypes.c_double),
        ("n_heavy", ctypes.c_int), ("heavy_scale", ctypes.c_double),
        ("rank", ctypes.c_int), ("coeff_sd", ctypes.c_double),
        ("seed_per_batch", ctypes.c_int),
    ]


def build(force: bool = False) -> str:
    """Compile ``libsynth.so`` next to this file (gcc, OpenMP)."""
    src = os.path.join(_HERE, "synth.c")
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(src):
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11",
                               src, "-o", _SO, "-lm"])
    return _SO


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_SO)
        lib.synth_generate.argtypes = [ctypes.POINTER(_Recipe), ctypes.c_uint64,
                                       ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]
        lib.synth_generate.restype = ctypes.c_int
        lib.synth_f16.argtypes = [ctypes.c_double]
        lib.synth_f16.restype = ctypes.c_uint16
        lib.synth_normal.argtypes = [ctypes.c_uint64, ctypes.c_uint64]
        lib.synth_normal.restype = ctypes.c_double
        lib.synth_stream.argtypes = [ctypes.c_uint64, ctypes.c_uint32, ctypes.c_uint32, ctypes.c_uint32]
        lib.synth_stream.restype = ctypes.c_uint64
        _lib = lib
    return _lib


@dataclasses.dataclass(frozen=True)
class Workload:
    """Shape, value recipe and method parameters of one synthetic workload."""
    name: str
    B: int
    Hq: int
    Hkv: int
    N: int
    D: int
    causal: bool
    blk: int
    rho: float
    seed: int
    kv_offset: bool = False
    offset_sd: float = 2.0
    sink: bool = False
    sink_scale: float = 8.0
    n_heavy: int = 0
    heavy_scale: float = 4.0
    rank: int = 0
    coeff_sd: float = 3.0
    seed_per_batch: bool = False

    @property
    def sm_scale(self) -> float:
        return float(np.float32(1.0 / np.sqrt(self.D)))

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)

    def flops(self) -> float:
        """Effective attention flops: 4*N^2*D*Hq*B, halved when causal."""
        f = 4.0 * self.N * self.N * self.D * self.Hq * self.B
        return f / 2 if self.causal else f


# The five workloads of the method's prefill setting (names state what they are).
TINY_NONCAUSAL_D64 = Workload("tiny_noncausal_B1_H1_N1024_D64", 1, 1, 1, 1024, 64, False, 64, 0.05, 0,
                              sink=True, n_heavy=4)
CAUSAL_MH_N8K = Workload("causal_B1_H8_N8192_D128", 1, 8, 8, 8192, 128, True, 64, 0.05, 2,
                         kv_offset=True, sink=True)
GQA_N32K = Workload("causal_gqa_B1_Hq32_Hkv8_N32768_D128", 1, 32, 8, 32768, 128, True, 128, 0.05, 3,
                    kv_offset=True, sink=True, rank=16)
GQA_N128K = Workload("causal_gqa_B1_Hq32_Hkv8_N131072_D128", 1, 32, 8, 131072, 128, True, 128, 0.05, 4,
                     kv_offset=True, sink=True, rank=16, n_heavy=64)
BATCHED_GQA_N16K = Workload("causal_gqa_B4_Hq28_Hkv4_N16384_D128", 4, 28, 4, 16384, 128, True, 128, 0.05, 5,
                            kv_offset=True, rank=16, seed_per_batch=True)

WORKLOADS = [TINY_NONCAUSAL_D64, CAUSAL_MH_N8K, GQA_N32K, GQA_N128K, BATCHED_GQA_N16K]


def generate(w: Workload):
    """Return fp16 numpy arrays Q [B,Hq,N,D], K [B,Hkv,N,D], V [B,Hkv,N,D]."""
    lib = _load()
    rc = _Recipe(w.B, w.Hq, w.Hkv, w.N, w.D, int(w.kv_offset), w.offset_sd, int(w.sink), w.sink_scale,
                 w.n_heavy, w.heavy_scale, w.rank, w.coeff_sd, int(w.seed_per_batch))
    Q = np.empty((w.B, w.Hq, w.N, w.D), dtype=np.uint16)
    K = np.empty((w.B, w.Hkv, w.N, w.D), dtype=np.uint16)
    V = np.empty((w.B, w.Hkv, w.N, w.D), dtype=np.uint16)
    rc_ = lib.synth_generate(ctypes.byref(rc), ctypes.c_uint64(w.seed), Q.ctypes.data, K.ctypes.data,
                             V.ctypes.data)
    if rc_ != 0:
        raise ValueError(f"synth_generate rejected workload {w} (code {rc_})")
    return Q.view(np.float16), K.view(np.float16), V.view(np.float16)


def f16_bits(x: float) -> int:
    """The generator's own double -> fp16 rounding (exposed for its tests)."""
    return int(_load().synth_f16(float(x)))


def sample_rows(w: Workload, count: int, seed: int = 7, per_block: int | None = None):
    """Deterministic row sample (b, hq, r): rows of q-blocks {0, 1, nb/2, nb-1} of the
    first (b, hq) (all of them, or `per_block` evenly spaced ones) plus `count`
    seeded random rows spread over the heads."""
    rng = np.random.default_rng(seed)
    nb = w.N // w.blk
    step = 1 if per_block is None else max(1, w.blk // per_block)
    rows = []
    for qb in sorted({0, min(1, nb - 1), nb // 2, nb - 1}):
        for r in range(qb * w.blk, (qb + 1) * w.blk, step):
            rows.append((0, 0, r))
    for _ in range(count):
        rows.append((int(rng.integers(w.B)), int(rng.integers(w.Hq)), int(rng.integers(w.N))))
    return np.array(rows, dtype=np.int64)
