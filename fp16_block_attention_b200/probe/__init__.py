"""Tensor-pipe rate probe (``libthrift_probe.so``): a measurement helper for the
benchmark's sweep, kept out of ``libthrift.so`` and its ABI.

``mma_rate(kind, iters)`` launches one CTA per SM, each issuing ``iters``
back-to-back M = 128, N = 256 tcgen05 products of ``kind`` (0: NVFP4
``.kind::mxf4nvf4`` with K = 64, 1: fp16 ``.kind::f16`` with K = 16) from
zeroed operands into one tensor-memory accumulator; the caller times the
launch.  ``FLOP[kind]`` is the work of one product.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libthrift_probe.so")
FLOP = {0: 2 * 128 * 256 * 64, 1: 2 * 128 * 256 * 16}
_lib = None


def _load():
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with `python -m fp16_block_attention_b200.build`")
        lib = ctypes.CDLL(LIB_PATH)
        lib.thrift_probe_mma_rate.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_void_p]
        lib.thrift_probe_mma_rate.restype = ctypes.c_int
        lib.thrift_probe_last_error.argtypes = [ctypes.c_void_p]
        lib.thrift_probe_last_error.restype = ctypes.c_int
        _lib = lib
    return _lib


def lib():
    return _load()


def mma_rate(kind: int, iters: int, stream=None):
    """Launch the probe on the current device (asynchronous on `stream`)."""
    if stream is None:
        stream = torch.cuda.current_stream()
    rc = _load().thrift_probe_mma_rate(int(kind), int(iters), ctypes.c_void_p(stream.cuda_stream))
    if rc != 0:
        raise RuntimeError(f"thrift_probe_mma_rate: status {rc}")


def last_error(stream=None) -> int:
    """Synchronise and read/clear the probe's error word (0, or 4 = a bounded wait timed out)."""
    if stream is None:
        stream = torch.cuda.current_stream()
    return int(_load().thrift_probe_last_error(ctypes.c_void_p(stream.cuda_stream)))
