"""Python binding of ``libthrift.so``: selective mixed-precision (FP16 / NVFP4)
block attention on B200 (sm_100a).

Argument marshalling only: every step runs in the library's CUDA kernels.
PyTorch supplies device memory and the stream.  The functions mirror the C ABI
in ``include/thrift.h``:

    quantize_nvfp4(x, op, shape)            -> (codes, scales)
    select_blocks(Q, K, shape, rho)         -> mask [B, Hq, nb, nb] (u8, 1 = FP16 pair)
    attention(Q, K, V, mask, qz, shape)     -> O
    attention_fused(Q, K, V, shape, rho)    -> O

There is no CPU fallback: importing fails loudly when the library is missing.
"""
from __future__ import annotations

import ctypes
import dataclasses
import math
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libthrift.so")

Q, K, V = 0, 1, 2  # thrift_operand

_STATUS = {0: "ok", 1: "invalid argument", 2: "unsupported shape", 3: "CUDA runtime error",
           4: "a kernel gave up a bounded wait", 5: "workspace missing or too small"}


class ThriftError(RuntimeError):
    def __init__(self, fn: str, status: int):
        super().__init__(f"{fn}: {_STATUS.get(status, 'unknown status')} (status {status})")
        self.status = status


class CShape(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("Hq", ctypes.c_int), ("Hkv", ctypes.c_int), ("N", ctypes.c_int),
                ("D", ctypes.c_int), ("blk", ctypes.c_int), ("causal", ctypes.c_int), ("sm_scale", ctypes.c_float)]


@dataclasses.dataclass(frozen=True)
class Shape:
    B: int
    Hq: int
    Hkv: int
    N: int
    D: int
    blk: int = 128
    causal: bool = True
    sm_scale: float | None = None

    def c(self) -> CShape:
        sm = self.sm_scale if self.sm_scale is not None else 1.0 / math.sqrt(self.D)
        return CShape(self.B, self.Hq, self.Hkv, self.N, self.D, self.blk, int(self.causal), sm)

    @property
    def nb(self) -> int:
        return self.N // self.blk


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with `python -m fp16_block_attention_b200.build` "
                          "(there is no fallback path)")
    lib = ctypes.CDLL(LIB_PATH)
    vp, st, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
    psh = ctypes.POINTER(CShape)
    sig = {
        "thrift_quant_bytes": ([psh, st, ctypes.POINTER(sz), ctypes.POINTER(sz)], st),
        "thrift_quantize_nvfp4": ([vp, st, psh, vp, vp, vp], st),
        "thrift_quantize_pool_nvfp4": ([vp, st, psh, vp, vp, vp, vp], st),
        "thrift_select_blocks_pooled": ([vp, vp, psh, ctypes.c_double, vp, vp, sz, vp], st),
        "thrift_quant8_bytes": ([psh, st, ctypes.POINTER(sz), ctypes.POINTER(sz)], st),
        "thrift_quantize_mxfp8": ([vp, st, psh, vp, vp, vp], st),
        "thrift_select_workspace_bytes": ([psh, ctypes.POINTER(sz)], st),
        "thrift_select_blocks": ([vp, vp, psh, ctypes.c_double, vp, vp, sz, vp], st),
        "thrift_select_blocks_static": ([vp, vp, psh, ctypes.c_double, vp, vp], st),
        "thrift_select_blocks_vertical_window": ([vp, vp, psh, ctypes.c_double, st, vp, vp, sz, vp], st),
        "thrift_select_blocks_tiered": ([vp, vp, psh, ctypes.c_double, ctypes.c_double, ctypes.c_double, vp, vp, sz,
                                         vp], st),
        "thrift_attention": ([vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, psh, vp, vp], st),
        "thrift_attention_tiered": ([vp] * 16 + [psh, vp, vp], st),
        "thrift_fused_workspace_bytes": ([psh, ctypes.POINTER(sz)], st),
        "thrift_attention_fused": ([vp, vp, vp, psh, ctypes.c_double, vp, vp, sz, vp], st),
        "thrift_fused_tiered_workspace_bytes": ([psh, ctypes.c_double, ctypes.POINTER(sz)], st),
        "thrift_attention_fused_tiered": ([vp, vp, vp, psh, ctypes.c_double, ctypes.c_double, ctypes.c_double, vp, vp,
                                           sz, vp], st),
        "thrift_pool_keys": ([vp, psh, vp, vp], st),
        "thrift_decode_select": ([vp, vp, psh, ctypes.c_double, vp, vp], st),
        "thrift_decode_workspace_bytes": ([psh, ctypes.POINTER(sz)], st),
        "thrift_decode_attention": ([vp, vp, vp, vp, vp, vp, vp, vp, psh, vp, vp, sz, vp], st),
        "thrift_decode_step": ([vp, vp, vp, vp, vp, vp, vp, vp, psh, ctypes.c_double, vp, vp, sz, vp], st),
        "thrift_last_device_error": ([vp], st),
        "thrift_set_wait_limit": ([ctypes.c_uint64], st),
        "thrift_strerror": ([st], ctypes.c_char_p),
    }
    for name, (args, res) in sig.items():
        f = getattr(lib, name)
        f.argtypes = args
        f.restype = res
    return lib


_lib = _load()

# C-ABI symbols the header declares (checked by the tests).
EXPORTS = ("thrift_quant_bytes", "thrift_quantize_nvfp4", "thrift_quantize_pool_nvfp4", "thrift_quant8_bytes",
           "thrift_quantize_mxfp8", "thrift_select_blocks_pooled",
           "thrift_select_workspace_bytes", "thrift_select_blocks",
           "thrift_select_blocks_static", "thrift_select_blocks_vertical_window", "thrift_select_blocks_tiered",
           "thrift_attention", "thrift_attention_tiered",
           "thrift_fused_workspace_bytes",
           "thrift_attention_fused", "thrift_fused_tiered_workspace_bytes", "thrift_attention_fused_tiered",
           "thrift_pool_keys", "thrift_decode_select", "thrift_decode_workspace_bytes",
           "thrift_decode_attention", "thrift_decode_step", "thrift_last_device_error",
           "thrift_set_wait_limit", "thrift_strerror")


def lib():
    return _lib


def _check(fn: str, status: int):
    if status != 0:
        raise ThriftError(fn, status)


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else None


def _dev(t: torch.Tensor, name: str, dtype=None):
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}")
    return t


def _nbytes(t: torch.Tensor) -> int:
    return t.numel() * t.element_size()


def _guard(*specs) -> torch.device:
    """Check the tensors of one call before the library reads them.

    Each spec is (tensor, name, dtype, count, kind): a contiguous CUDA tensor
    of `dtype` (None: any) holding exactly `count` elements (kind "n"), or at
    least `count` bytes (kind "b", caller buffers); a None tensor is skipped.
    All tensors must sit on one device, which is returned: the library takes
    its stream and its static device memory from the current device, so a
    tensor on another device, or one smaller than the shape implies, would be
    read out of bounds on the GPU."""
    dev = None
    for t, name, dtype, count, kind in specs:
        if t is None:
            continue
        _dev(t, name, dtype)
        if kind == "n" and t.numel() != count:
            raise ValueError(f"{name} holds {t.numel()} elements; the shape needs {count}")
        if kind == "b" and _nbytes(t) < count:
            raise ValueError(f"{name} holds {_nbytes(t)} bytes; the shape needs at least {count}")
        if dev is None:
            dev = t.device
        elif t.device != dev:
            raise ValueError(f"{name} is on {t.device}; the call's other tensors are on {dev}")
    return dev


def _stream(stream, dev: torch.device):
    if stream is None:
        stream = torch.cuda.current_stream(dev)
    elif stream.device != dev:
        raise ValueError(f"the stream is on {stream.device}; the tensors are on {dev}")
    return ctypes.c_void_p(stream.cuda_stream)


def _counts(shape: Shape):
    """Element counts of Q (and O), K / V and the block mask for `shape`."""
    nq = shape.B * shape.Hq * shape.N * shape.D
    nk = shape.B * shape.Hkv * shape.N * shape.D
    return nq, nk, shape.B * shape.Hq * shape.nb * shape.nb


def shape_of(Q: torch.Tensor, K: torch.Tensor, blk: int = 128, causal: bool = True,
             sm_scale: float | None = None) -> Shape:
    B, Hq, N, D = Q.shape
    return Shape(B, Hq, K.shape[1], N, D, blk, causal, sm_scale)


def quant_bytes(shape: Shape, op: int):
    c, s = ctypes.c_size_t(), ctypes.c_size_t()
    _check("thrift_quant_bytes", _lib.thrift_quant_bytes(ctypes.byref(shape.c()), op, ctypes.byref(c),
                                                         ctypes.byref(s)))
    return c.value, s.value


def quantize_nvfp4(x: torch.Tensor, op: int, shape: Shape, codes=None, scales=None, stream=None):
    """NVFP4 copy of Q/K (along D) or V (along keys): (codes u8, scales u8)."""
    nq, nk, _ = _counts(shape)
    nc, ns = quant_bytes(shape, op)
    dev = _guard((x, "x", torch.float16, nq if op == Q else nk, "n"), (codes, "codes", None, nc, "b"),
                 (scales, "scales", None, ns, "b"))
    if codes is None:
        codes = torch.empty(nc, dtype=torch.uint8, device=dev)
    if scales is None:
        scales = torch.empty(ns, dtype=torch.uint8, device=dev)
    with torch.cuda.device(dev):
        _check("thrift_quantize_nvfp4", _lib.thrift_quantize_nvfp4(_ptr(x), op, ctypes.byref(shape.c()), _ptr(codes),
                                                                   _ptr(scales), _stream(stream, dev)))
    return codes, scales


def quantize_pool_nvfp4(x: torch.Tensor, op: int, shape: Shape, codes=None, scales=None, means=None, stream=None):
    """NVFP4 copy of Q or K (as quantize_nvfp4) and its FP32 block means
    [B, H, nb, D] in one pass: (codes, scales, means)."""
    if op not in (Q, K):
        raise ValueError("quantize_pool_nvfp4 takes Q or K")
    nq, nk, _ = _counts(shape)
    nc, ns = quant_bytes(shape, op)
    H = shape.Hq if op == Q else shape.Hkv
    nm = shape.B * H * shape.nb * shape.D
    dev = _guard((x, "x", torch.float16, nq if op == Q else nk, "n"), (codes, "codes", None, nc, "b"),
                 (scales, "scales", None, ns, "b"), (means, "means", torch.float32, nm, "n"))
    if codes is None:
        codes = torch.empty(nc, dtype=torch.uint8, device=dev)
    if scales is None:
        scales = torch.empty(ns, dtype=torch.uint8, device=dev)
    if means is None:
        means = torch.empty((shape.B, H, shape.nb, shape.D), dtype=torch.float32, device=dev)
    with torch.cuda.device(dev):
        _check("thrift_quantize_pool_nvfp4", _lib.thrift_quantize_pool_nvfp4(
            _ptr(x), op, ctypes.byref(shape.c()), _ptr(codes), _ptr(scales), _ptr(means), _stream(stream, dev)))
    return codes, scales, means


def quant8_bytes(shape: Shape, op: int):
    c, s = ctypes.c_size_t(), ctypes.c_size_t()
    _check("thrift_quant8_bytes", _lib.thrift_quant8_bytes(ctypes.byref(shape.c()), op, ctypes.byref(c),
                                                           ctypes.byref(s)))
    return c.value, s.value


def quantize_mxfp8(x: torch.Tensor, op: int, shape: Shape, codes=None, scales=None, stream=None):
    """MXFP8 copy of Q/K (along D) or V (along keys): (codes u8, scales u8)."""
    nq, nk, _ = _counts(shape)
    nc, ns = quant8_bytes(shape, op)
    dev = _guard((x, "x", torch.float16, nq if op == Q else nk, "n"), (codes, "codes", None, nc, "b"),
                 (scales, "scales", None, ns, "b"))
    if codes is None:
        codes = torch.empty(nc, dtype=torch.uint8, device=dev)
    if scales is None:
        scales = torch.empty(ns, dtype=torch.uint8, device=dev)
    with torch.cuda.device(dev):
        _check("thrift_quantize_mxfp8", _lib.thrift_quantize_mxfp8(_ptr(x), op, ctypes.byref(shape.c()), _ptr(codes),
                                                                   _ptr(scales), _stream(stream, dev)))
    return codes, scales


def mx8_qk_scale_index(bh, n, g, NT):
    """Byte of the MXFP8 scale of (row n, group g = d / 32) of Q or K."""
    return (bh * NT + n // 128) * 512 + (n % 32) * 16 + ((n % 128) // 32) * 4 + g


def mx8_v_scale_index(bh, d, n, NT):
    """Byte of the MXFP8 scale of (channel d, key n) of V."""
    return (bh * NT + n // 128) * 512 + (d % 32) * 16 + (d // 32) * 4 + (n % 128) // 32


def select_workspace_bytes(shape: Shape) -> int:
    n = ctypes.c_size_t()
    _check("thrift_select_workspace_bytes", _lib.thrift_select_workspace_bytes(ctypes.byref(shape.c()),
                                                                               ctypes.byref(n)))
    return n.value


def _select_args(Qt, Kt, shape: Shape, mask, ws):
    """Checks shared by the selection calls; allocates the missing mask and
    workspace (ws=False: the call takes none)."""
    nq, nk, nm = _counts(shape)
    need = select_workspace_bytes(shape) if ws is not False else 0
    dev = _guard((Qt, "Q", torch.float16, nq, "n"), (Kt, "K", torch.float16, nk, "n"),
                 (mask, "mask", torch.uint8, nm, "n"), (ws if ws is not False else None, "ws", None, need, "b"))
    if mask is None:
        mask = torch.empty((shape.B, shape.Hq, shape.nb, shape.nb), dtype=torch.uint8, device=dev)
    if ws is None:
        ws = torch.empty(need, dtype=torch.uint8, device=dev)
    return dev, mask, ws


def select_blocks(Qt: torch.Tensor, Kt: torch.Tensor, shape: Shape, rho: float, mask=None, ws=None, stream=None):
    """Selection mask [B, Hq, nb, nb] (u8): 1 = FP16 block pair."""
    dev, mask, ws = _select_args(Qt, Kt, shape, mask, ws)
    with torch.cuda.device(dev):
        _check("thrift_select_blocks", _lib.thrift_select_blocks(_ptr(Qt), _ptr(Kt), ctypes.byref(shape.c()),
                                                                 float(rho), _ptr(mask), _ptr(ws), _nbytes(ws),
                                                                 _stream(stream, dev)))
    return mask


def select_blocks_tiered(Qt: torch.Tensor, Kt: torch.Tensor, shape: Shape, rho: float, sigma: float, mask=None,
                         ws=None, stream=None, rho8: float = 0.0):
    """Tiered selection mask [B, Hq, nb, nb] (u8): 1 FP16, 3 MXFP8 (the next
    rho8 of the ranking), 0 NVFP4, 2 skipped (the lowest-ranked pairs, never
    forced, FP16 or 8-bit ones)."""
    dev, mask, ws = _select_args(Qt, Kt, shape, mask, ws)
    with torch.cuda.device(dev):
        _check("thrift_select_blocks_tiered", _lib.thrift_select_blocks_tiered(
            _ptr(Qt), _ptr(Kt), ctypes.byref(shape.c()), float(rho), float(rho8), float(sigma), _ptr(mask), _ptr(ws),
            _nbytes(ws), _stream(stream, dev)))
    return mask


def select_blocks_vertical_window(Qt: torch.Tensor, Kt: torch.Tensor, shape: Shape, rho: float, window: int,
                                  mask=None, ws=None, stream=None):
    """Selection mask [B, Hq, nb, nb] (u8) of the HyQuant-style selector: the
    local window of `window` blocks, then whole key-block columns ranked by
    the pooled attention mass they receive, on the same budget as
    select_blocks."""
    dev, mask, ws = _select_args(Qt, Kt, shape, mask, ws)
    with torch.cuda.device(dev):
        _check("thrift_select_blocks_vertical_window", _lib.thrift_select_blocks_vertical_window(
            _ptr(Qt), _ptr(Kt), ctypes.byref(shape.c()), float(rho), int(window), _ptr(mask), _ptr(ws), _nbytes(ws),
            _stream(stream, dev)))
    return mask


def select_blocks_pooled(qm: torch.Tensor, km: torch.Tensor, shape: Shape, rho: float, mask=None, ws=None,
                         stream=None):
    """select_blocks from precomputed FP32 block means (quantize_pool_nvfp4)."""
    _, _, nmask = _counts(shape)
    need = select_workspace_bytes(shape)
    dev = _guard((qm, "qm", torch.float32, shape.B * shape.Hq * shape.nb * shape.D, "n"),
                 (km, "km", torch.float32, shape.B * shape.Hkv * shape.nb * shape.D, "n"),
                 (mask, "mask", torch.uint8, nmask, "n"), (ws, "ws", None, need, "b"))
    if mask is None:
        mask = torch.empty((shape.B, shape.Hq, shape.nb, shape.nb), dtype=torch.uint8, device=dev)
    if ws is None:
        ws = torch.empty(need, dtype=torch.uint8, device=dev)
    with torch.cuda.device(dev):
        _check("thrift_select_blocks_pooled", _lib.thrift_select_blocks_pooled(
            _ptr(qm), _ptr(km), ctypes.byref(shape.c()), float(rho), _ptr(mask), _ptr(ws), _nbytes(ws),
            _stream(stream, dev)))
    return mask


SELECT_STATIC_BYTES = 16 << 20


def select_blocks_static(Qt: torch.Tensor, Kt: torch.Tensor, shape: Shape, rho: float, mask=None, stream=None):
    """Selection mask without a workspace argument: for callers that cannot
    allocate device memory (their GPU memory belongs to another allocator, or
    they are hooks with no way to allocate).  Runs on the library's static
    16 MiB scratch per device; larger selection workspaces are rejected.  Calls
    that overlap on the GPU race on the shared scratch.  (This binding still
    lets torch allocate the mask when none is given.)"""
    dev, mask, _ = _select_args(Qt, Kt, shape, mask, False)
    with torch.cuda.device(dev):
        _check("thrift_select_blocks_static", _lib.thrift_select_blocks_static(
            _ptr(Qt), _ptr(Kt), ctypes.byref(shape.c()), float(rho), _ptr(mask), _stream(stream, dev)))
    return mask


@dataclasses.dataclass
class Quantised:
    q4: torch.Tensor
    qs: torch.Tensor
    k4: torch.Tensor
    ks: torch.Tensor
    v4: torch.Tensor
    vs: torch.Tensor


def quantize_all(Qt, Kt, Vt, shape: Shape, stream=None) -> Quantised:
    q4, qs = quantize_nvfp4(Qt, Q, shape, stream=stream)
    k4, ks = quantize_nvfp4(Kt, K, shape, stream=stream)
    v4, vs = quantize_nvfp4(Vt, V, shape, stream=stream)
    return Quantised(q4, qs, k4, ks, v4, vs)


def _qz_specs(qz, shape: Shape, with_q: bool = True):
    """Guard specs of the NVFP4 copies (byte counts from thrift_quant_bytes)."""
    specs = []
    for op, names in ((Q, ("q4", "qs")), (K, ("k4", "ks")), (V, ("v4", "vs"))):
        if op == Q and not with_q:
            continue
        nc, ns = quant_bytes(shape, op)
        specs.append((getattr(qz, names[0]), names[0], None, nc, "b"))
        specs.append((getattr(qz, names[1]), names[1], None, ns, "b"))
    return specs


def _attention_args(Qt, Kt, Vt, mask, qz, shape: Shape, out, extra=()):
    nq, nk, nm = _counts(shape)
    for t, n in ((qz.q4, "q4"), (qz.qs, "qs"), (qz.k4, "k4"), (qz.ks, "ks"), (qz.v4, "v4"), (qz.vs, "vs")):
        if t is None:
            raise ValueError(f"{n} is missing")
    dev = _guard((Qt, "Q", torch.float16, nq, "n"), (Kt, "K", torch.float16, nk, "n"),
                 (Vt, "V", torch.float16, nk, "n"), (mask, "mask", torch.uint8, nm, "n"),
                 (out, "out", torch.float16, nq, "n"), *_qz_specs(qz, shape), *extra)
    if out is None:
        out = torch.empty_like(Qt)
    return dev, out


def attention(Qt, Kt, Vt, mask, qz: Quantised, shape: Shape, out=None, stream=None):
    """Mixed FP16/NVFP4 attention output O (fp16, shaped like Q)."""
    dev, out = _attention_args(Qt, Kt, Vt, mask, qz, shape, out)
    with torch.cuda.device(dev):
        _check("thrift_attention", _lib.thrift_attention(
            _ptr(Qt), _ptr(Kt), _ptr(Vt), _ptr(mask), _ptr(qz.q4), _ptr(qz.qs), _ptr(qz.k4), _ptr(qz.ks),
            _ptr(qz.v4), _ptr(qz.vs), ctypes.byref(shape.c()), _ptr(out), _stream(stream, dev)))
    return out


@dataclasses.dataclass
class Quantised8:
    """MXFP8 copies of Q, K, V (codes and scales) for 8-bit pairs."""
    q8: torch.Tensor
    qs8: torch.Tensor
    k8: torch.Tensor
    ks8: torch.Tensor
    v8: torch.Tensor
    vs8: torch.Tensor


def quantize_all_mxfp8(Qt, Kt, Vt, shape: Shape, stream=None) -> Quantised8:
    q8, qs8 = quantize_mxfp8(Qt, Q, shape, stream=stream)
    k8, ks8 = quantize_mxfp8(Kt, K, shape, stream=stream)
    v8, vs8 = quantize_mxfp8(Vt, V, shape, stream=stream)
    return Quantised8(q8, qs8, k8, ks8, v8, vs8)


def attention_tiered(Qt, Kt, Vt, mask, qz: Quantised, shape: Shape, out=None, stream=None, q8: Quantised8 = None):
    """attention() for masks that may hold 2 (skipped pairs, absent from the
    softmax) and, given the MXFP8 copies q8, 3 (8-bit pairs), as from
    select_blocks_tiered."""
    extra = []
    if q8 is not None:
        for op, names in ((Q, ("q8", "qs8")), (K, ("k8", "ks8")), (V, ("v8", "vs8"))):
            nc, ns = quant8_bytes(shape, op)
            extra += [(getattr(q8, names[0]), names[0], None, nc, "b"), (getattr(q8, names[1]), names[1], None, ns, "b")]
    dev, out = _attention_args(Qt, Kt, Vt, mask, qz, shape, out, extra)
    p8 = [None] * 6 if q8 is None else [_ptr(t) for t in (q8.q8, q8.qs8, q8.k8, q8.ks8, q8.v8, q8.vs8)]
    with torch.cuda.device(dev):
        _check("thrift_attention_tiered", _lib.thrift_attention_tiered(
            _ptr(Qt), _ptr(Kt), _ptr(Vt), _ptr(mask), _ptr(qz.q4), _ptr(qz.qs), _ptr(qz.k4), _ptr(qz.ks),
            _ptr(qz.v4), _ptr(qz.vs), *p8, ctypes.byref(shape.c()), _ptr(out), _stream(stream, dev)))
    return out


def fused_workspace_bytes(shape: Shape) -> int:
    n = ctypes.c_size_t()
    _check("thrift_fused_workspace_bytes", _lib.thrift_fused_workspace_bytes(ctypes.byref(shape.c()),
                                                                             ctypes.byref(n)))
    return n.value


def _fused_args(Qt, Kt, Vt, shape: Shape, out, ws, need):
    nq, nk, _ = _counts(shape)
    dev = _guard((Qt, "Q", torch.float16, nq, "n"), (Kt, "K", torch.float16, nk, "n"),
                 (Vt, "V", torch.float16, nk, "n"), (out, "out", torch.float16, nq, "n"), (ws, "ws", None, need, "b"))
    if out is None:
        out = torch.empty_like(Qt)
    if ws is None:
        ws = torch.empty(need, dtype=torch.uint8, device=dev)
    return dev, out, ws


def attention_fused(Qt, Kt, Vt, shape: Shape, rho: float, out=None, ws=None, stream=None):
    """Quantise, select (budget rho) and attend in one call."""
    dev, out, ws = _fused_args(Qt, Kt, Vt, shape, out, ws, fused_workspace_bytes(shape))
    with torch.cuda.device(dev):
        _check("thrift_attention_fused", _lib.thrift_attention_fused(
            _ptr(Qt), _ptr(Kt), _ptr(Vt), ctypes.byref(shape.c()), float(rho), _ptr(out), _ptr(ws), _nbytes(ws),
            _stream(stream, dev)))
    return out


def fused_tiered_workspace_bytes(shape: Shape, rho8: float = 0.0) -> int:
    n = ctypes.c_size_t()
    _check("thrift_fused_tiered_workspace_bytes", _lib.thrift_fused_tiered_workspace_bytes(
        ctypes.byref(shape.c()), float(rho8), ctypes.byref(n)))
    return n.value


def attention_fused_tiered(Qt, Kt, Vt, shape: Shape, rho: float, rho8: float = 0.0, sigma: float = 0.0, out=None,
                           ws=None, stream=None):
    """Quantise (NVFP4, and MXFP8 when rho8 > 0), select four classes (FP16
    budget rho, 8-bit budget rho8, skipped share sigma) and attend in one call."""
    dev, out, ws = _fused_args(Qt, Kt, Vt, shape, out, ws, fused_tiered_workspace_bytes(shape, rho8))
    with torch.cuda.device(dev):
        _check("thrift_attention_fused_tiered", _lib.thrift_attention_fused_tiered(
            _ptr(Qt), _ptr(Kt), _ptr(Vt), ctypes.byref(shape.c()), float(rho), float(rho8), float(sigma), _ptr(out),
            _ptr(ws), _nbytes(ws), _stream(stream, dev)))
    return out


# ---- decode ------------------------------------------------------------------
def _decode_counts(shape: Shape):
    """Element counts of q / O [B, Hq, D], the block means [B, Hkv, nb, D] and
    the decode mask [B, Hq, nb]."""
    return (shape.B * shape.Hq * shape.D, shape.B * shape.Hkv * shape.nb * shape.D, shape.B * shape.Hq * shape.nb)


def pool_keys(Kt: torch.Tensor, shape: Shape, km=None, stream=None):
    """FP32 block means of K: [B, Hkv, nb, D]."""
    _, nk, _ = _counts(shape)
    _, nkm, _ = _decode_counts(shape)
    dev = _guard((Kt, "K", torch.float16, nk, "n"), (km, "km", torch.float32, nkm, "n"))
    if km is None:
        km = torch.empty((shape.B, shape.Hkv, shape.nb, shape.D), dtype=torch.float32, device=dev)
    with torch.cuda.device(dev):
        _check("thrift_pool_keys", _lib.thrift_pool_keys(_ptr(Kt), ctypes.byref(shape.c()), _ptr(km),
                                                         _stream(stream, dev)))
    return km


def decode_select(qt: torch.Tensor, km: torch.Tensor, shape: Shape, rho: float, mask=None, stream=None):
    """Decode selection mask [B, Hq, nb] (u8, 1 = FP16 block) of q [B, Hq, D]."""
    nqd, nkm, nmask = _decode_counts(shape)
    dev = _guard((qt, "q", torch.float16, nqd, "n"), (km, "km", torch.float32, nkm, "n"),
                 (mask, "mask", torch.uint8, nmask, "n"))
    if mask is None:
        mask = torch.empty((shape.B, shape.Hq, shape.nb), dtype=torch.uint8, device=dev)
    with torch.cuda.device(dev):
        _check("thrift_decode_select", _lib.thrift_decode_select(_ptr(qt), _ptr(km), ctypes.byref(shape.c()),
                                                                 float(rho), _ptr(mask), _stream(stream, dev)))
    return mask


def decode_workspace_bytes(shape: Shape) -> int:
    n = ctypes.c_size_t()
    _check("thrift_decode_workspace_bytes", _lib.thrift_decode_workspace_bytes(ctypes.byref(shape.c()),
                                                                               ctypes.byref(n)))
    return n.value


def _decode_args(qt, Kt, Vt, kq, shape: Shape, out, ws, extra=()):
    _, nk, _ = _counts(shape)
    nqd, _, _ = _decode_counts(shape)
    for t, n in ((kq.k4, "k4"), (kq.ks, "ks"), (kq.v4, "v4"), (kq.vs, "vs")):
        if t is None:
            raise ValueError(f"{n} is missing")
    need = decode_workspace_bytes(shape)
    dev = _guard((qt, "q", torch.float16, nqd, "n"), (Kt, "K", torch.float16, nk, "n"),
                 (Vt, "V", torch.float16, nk, "n"), (out, "out", torch.float16, nqd, "n"), (ws, "ws", None, need, "b"),
                 *_qz_specs(kq, shape, with_q=False), *extra)
    if out is None:
        out = torch.empty((shape.B, shape.Hq, shape.D), dtype=torch.float16, device=dev)
    if ws is None:
        ws = torch.empty(need, dtype=torch.uint8, device=dev)
    return dev, out, ws


def decode_attention(qt, Kt, Vt, kq: "Quantised", mask, shape: Shape, out=None, ws=None, stream=None):
    """Decode output [B, Hq, D] fp16 for the given block mask; kq holds the
    NVFP4 copies of K and V (its q4 / qs fields are not read)."""
    _, _, nmask = _decode_counts(shape)
    dev, out, ws = _decode_args(qt, Kt, Vt, kq, shape, out, ws, [(mask, "mask", torch.uint8, nmask, "n")])
    with torch.cuda.device(dev):
        _check("thrift_decode_attention", _lib.thrift_decode_attention(
            _ptr(qt), _ptr(Kt), _ptr(Vt), _ptr(kq.k4), _ptr(kq.ks), _ptr(kq.v4), _ptr(kq.vs), _ptr(mask),
            ctypes.byref(shape.c()), _ptr(out), _ptr(ws), _nbytes(ws), _stream(stream, dev)))
    return out


def decode_step(qt, Kt, Vt, kq: "Quantised", km, shape: Shape, rho: float, out=None, ws=None, stream=None):
    """Selection and attention of one decode step: O [B, Hq, D] fp16."""
    _, nkm, _ = _decode_counts(shape)
    dev, out, ws = _decode_args(qt, Kt, Vt, kq, shape, out, ws, [(km, "km", torch.float32, nkm, "n")])
    with torch.cuda.device(dev):
        _check("thrift_decode_step", _lib.thrift_decode_step(
            _ptr(qt), _ptr(Kt), _ptr(Vt), _ptr(kq.k4), _ptr(kq.ks), _ptr(kq.v4), _ptr(kq.vs), _ptr(km),
            ctypes.byref(shape.c()), float(rho), _ptr(out), _ptr(ws), _nbytes(ws), _stream(stream, dev)))
    return out


def quantize_kv(Kt, Vt, shape: Shape, stream=None) -> "Quantised":
    """NVFP4 copies of K and V only (the decode cache); q4 / qs are None."""
    k4, ks = quantize_nvfp4(Kt, K, shape, stream=stream)
    v4, vs = quantize_nvfp4(Vt, V, shape, stream=stream)
    return Quantised(None, None, k4, ks, v4, vs)


def last_device_error(stream=None) -> int:
    """Synchronise and read/clear the device error word of the current device
    (or of `stream`'s device): 0 = none, 4 = a bounded wait timed out, 1 = a
    kernel met a mask byte it cannot compute."""
    dev = torch.device("cuda", torch.cuda.current_device()) if stream is None else stream.device
    with torch.cuda.device(dev):
        return int(_lib.thrift_last_device_error(_stream(stream, dev)))


WAIT_LIMIT_DEFAULT_NS = 2_000_000_000


def set_wait_limit(ns: int):
    """Bound (ns) of every wait inside the prefill attention kernels launched
    from now on (process-wide; 2 s by default)."""
    _check("thrift_set_wait_limit", _lib.thrift_set_wait_limit(int(ns)))


def qk_scale_index(bh, n, g, NT, D):
    """Byte offset of the scale of (row n, group g) in the Q/K scale layout (see thrift.h)."""
    return ((bh * NT + n // 128) * (D // 64) + g // 4) * 512 + (n % 32) * 16 + ((n % 128) // 32) * 4 + (g % 4)


def v_scale_index(bh, d, n, NT):
    """Byte offset of the scale of (channel d, key group n//16) in the V scale layout."""
    return (bh * 2 * NT + n // 64) * 512 + (d % 32) * 16 + (d // 32) * 4 + (n % 64) // 16
