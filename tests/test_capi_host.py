"""The C-ABI library loads, exports every symbol the header declares, and
rejects bad arguments on the host before any launch (no GPU needed)."""
import ctypes
import os
import re

import pytest
import torch

import fp16_block_attention_b200 as thrift

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _header_symbols():
    text = open(os.path.join(ROOT, "include", "thrift.h")).read()
    return set(re.findall(r"THRIFT_API\s+[\w\s\*]+?\b(thrift_\w+)\s*\(", text))


def test_library_exports_every_declared_symbol():
    declared = _header_symbols()
    assert declared == set(thrift.EXPORTS)
    lib = ctypes.CDLL(thrift.LIB_PATH)
    for name in declared:
        assert hasattr(lib, name), name


def _c(**kw):
    base = dict(B=1, Hq=2, Hkv=1, N=256, D=128, blk=128, causal=1, sm_scale=0.088)
    base.update(kw)
    return thrift.CShape(base["B"], base["Hq"], base["Hkv"], base["N"], base["D"], base["blk"], base["causal"],
                         base["sm_scale"])


@pytest.mark.parametrize("kw,status", [
    (dict(), 0),
    (dict(B=0), 1), (dict(N=-64), 1), (dict(Hq=3, Hkv=2), 1), (dict(causal=2), 1),
    (dict(sm_scale=float("nan")), 1), (dict(sm_scale=0.0), 1), (dict(sm_scale=-0.1), 1),
    (dict(D=96), 2), (dict(blk=32), 2), (dict(N=200), 2), (dict(N=64, blk=128), 2), (dict(N=262144), 2),
])
def test_shape_validation(kw, status):
    c, s = ctypes.c_size_t(), ctypes.c_size_t()
    assert thrift.lib().thrift_quant_bytes(ctypes.byref(_c(**kw)), 0, ctypes.byref(c), ctypes.byref(s)) == status


def test_quant_bytes_layout_sizes():
    sh = thrift.Shape(2, 4, 2, 192, 128, 64, True)
    assert thrift.quant_bytes(sh, thrift.Q) == (2 * 4 * 192 * 64, 2 * 4 * 2 * 2 * 512)
    assert thrift.quant_bytes(sh, thrift.K) == (2 * 2 * 192 * 64, 2 * 2 * 2 * 2 * 512)
    assert thrift.quant_bytes(sh, thrift.V) == (2 * 2 * 192 * 64, 2 * 2 * 4 * 512)


def test_null_pointers_and_bad_rho_are_rejected_before_launch():
    lib = thrift.lib()
    sh = ctypes.byref(_c())
    fake = ctypes.c_void_p(256)
    assert lib.thrift_quantize_nvfp4(None, 0, sh, fake, fake, None) == 1
    assert lib.thrift_quantize_nvfp4(fake, 7, sh, fake, fake, None) == 1
    assert lib.thrift_quantize_nvfp4(ctypes.c_void_p(258), 0, sh, fake, fake, None) == 1  # misaligned
    assert lib.thrift_select_blocks(fake, fake, sh, 1.5, fake, fake, 1 << 30, None) == 1
    assert lib.thrift_select_blocks(fake, fake, sh, 0.05, fake, None, 0, None) == 5
    assert lib.thrift_select_blocks(fake, fake, sh, 0.05, fake, fake, 16, None) == 5
    vw = lib.thrift_select_blocks_vertical_window
    assert vw(fake, fake, sh, 0.05, -1, fake, fake, 1 << 30, None) == 1      # negative window
    assert vw(fake, None, sh, 0.05, 2, fake, fake, 1 << 30, None) == 1
    assert vw(fake, fake, sh, -0.5, 2, fake, fake, 1 << 30, None) == 1
    assert vw(fake, fake, sh, 0.05, 2, fake, fake, 16, None) == 5
    tr = lib.thrift_select_blocks_tiered
    assert tr(fake, fake, sh, 0.05, 1.5, 0.1, fake, fake, 1 << 30, None) == 1    # rho8 out of range
    assert tr(fake, fake, sh, 0.05, 0.1, -0.1, fake, fake, 1 << 30, None) == 1   # sigma out of range
    assert tr(fake, fake, sh, 0.05, 0.1, 0.1, None, fake, 1 << 30, None) == 1
    assert tr(fake, fake, sh, 0.05, 0.1, 0.1, fake, fake, 16, None) == 5
    assert lib.thrift_quantize_mxfp8(fake, 3, sh, fake, fake, None) == 1
    assert lib.thrift_quantize_mxfp8(fake, 0, sh, None, fake, None) == 1
    ft = lib.thrift_attention_fused_tiered
    assert ft(fake, fake, fake, sh, 0.05, 1.5, 0.0, fake, fake, 1 << 30, None) == 1          # rho8 out of range
    assert ft(fake, fake, fake, sh, 0.05, 0.1, -0.5, fake, fake, 1 << 30, None) == 1         # sigma out of range
    assert ft(fake, fake, fake, ctypes.byref(_c(blk=64)), 0.05, 0.1, 0.0, fake, fake, 1 << 30, None) == 2
    assert ft(fake, fake, fake, sh, 0.05, 0.1, 0.0, fake, fake, 16, None) == 5
    assert ft(fake, None, fake, sh, 0.05, 0.0, 0.0, fake, fake, 1 << 30, None) == 1
    at = lib.thrift_attention_tiered
    assert at(*[fake] * 10, fake, None, fake, fake, fake, fake, sh, fake, None) == 1        # some copies missing
    assert at(*[fake] * 10, fake, ctypes.c_void_p(264), fake, fake, fake, fake, sh, fake, None) == 1  # misaligned
    assert at(*[fake] * 16, ctypes.byref(_c(blk=64)), fake, None) == 2                      # 8-bit needs blk 128
    args = [fake] * 10
    assert lib.thrift_attention(None, *args[:9], sh, fake, None) == 1
    assert lib.thrift_attention_fused(fake, fake, fake, sh, -0.1, fake, fake, 1 << 30, None) == 1
    assert lib.thrift_attention_fused(fake, fake, fake, sh, 0.05, fake, fake, 8, None) == 5


def test_mma_rate_probe_lives_outside_the_library_and_rejects_bad_arguments():
    from fp16_block_attention_b200 import probe
    assert not hasattr(thrift.lib(), "thrift_mma_rate_probe")
    lib = probe.lib()
    assert lib.thrift_probe_mma_rate(2, 10, None) == 1
    assert lib.thrift_probe_mma_rate(-1, 10, None) == 1
    assert lib.thrift_probe_mma_rate(0, 0, None) == 1
    assert lib.thrift_probe_mma_rate(1, (1 << 24) + 1, None) == 1


def test_workspace_sizes_cover_the_parts():
    sh = thrift.Shape(1, 4, 2, 512, 128, 64, True)
    need = thrift.fused_workspace_bytes(sh)
    parts = sum(sum(thrift.quant_bytes(sh, op)) for op in (0, 1, 2)) + 4 * 8 * 8 + thrift.select_workspace_bytes(sh)
    assert need >= parts


def test_fused_tiered_workspace_adds_the_mxfp8_copies_only_for_an_eight_bit_budget():
    sh = thrift.Shape(1, 4, 2, 1024, 128, 128, True, 0.088)
    w0, w8 = thrift.fused_tiered_workspace_bytes(sh, 0.0), thrift.fused_tiered_workspace_bytes(sh, 0.25)
    assert w0 == thrift.fused_workspace_bytes(sh)
    mx8 = sum(sum(thrift.quant8_bytes(sh, op)) for op in (thrift.Q, thrift.K, thrift.V))
    assert mx8 <= w8 - w0 <= mx8 + 6 * 256      # each part 256-byte aligned


def test_strerror_names_every_status():
    lib = thrift.lib()
    names = {lib.thrift_strerror(i).decode() for i in range(6)}
    assert len(names) == 6 and "ok" in names


@pytest.mark.parametrize("kw,status", [
    (dict(), 0), (dict(D=64), 2), (dict(blk=64), 2), (dict(Hq=32, Hkv=1), 2), (dict(Hq=16, Hkv=1), 0),
])
def test_decode_shape_validation(kw, status):
    n = ctypes.c_size_t()
    assert thrift.lib().thrift_decode_workspace_bytes(ctypes.byref(_c(**kw)), ctypes.byref(n)) == status
    if status == 0:
        assert n.value > 0


def test_decode_arguments_are_rejected_before_launch():
    lib = thrift.lib()
    sh = ctypes.byref(_c())
    fake = ctypes.c_void_p(256)
    assert lib.thrift_pool_keys(None, sh, fake, None) == 1
    assert lib.thrift_pool_keys(fake, sh, ctypes.c_void_p(260), None) == 1          # misaligned
    assert lib.thrift_decode_select(fake, fake, sh, 1.5, fake, None) == 1
    assert lib.thrift_decode_select(fake, None, sh, 0.05, fake, None) == 1
    assert lib.thrift_decode_select(fake, fake, ctypes.byref(_c(D=64)), 0.05, fake, None) == 2
    args = [fake] * 7
    assert lib.thrift_decode_attention(*args, None, sh, fake, fake, 1 << 30, None) == 1  # no mask
    assert lib.thrift_decode_attention(*args, fake, sh, fake, fake, 16, None) == 5       # workspace too small
    assert lib.thrift_decode_step(*args, fake, sh, -0.1, fake, fake, 1 << 30, None) == 1
    assert lib.thrift_decode_step(*args, fake, sh, 0.05, fake, None, 0, None) == 5


class _FakeCuda:
    """Stand-in for a CUDA tensor (no GPU here): what the binding's checks read."""

    def __init__(self, numel, dtype=torch.float16, device="cuda:0", contiguous=True):
        self._n, self.dtype, self.device, self._c = numel, dtype, torch.device(device), contiguous
        self.is_cuda = True

    def numel(self):
        return self._n

    def element_size(self):
        return torch.empty(0, dtype=self.dtype).element_size()

    def is_contiguous(self):
        return self._c


def test_binding_checks_sizes_and_devices_before_calling_the_library():
    sh = thrift.Shape(1, 4, 2, 256, 64, 64, True)
    nq, nk, nm = 4 * 256 * 64, 2 * 256 * 64, 4 * 4 * 4
    ok = [(_FakeCuda(nq), "Q", torch.float16, nq, "n"), (_FakeCuda(nk), "K", torch.float16, nk, "n"),
          (_FakeCuda(nm, torch.uint8), "mask", torch.uint8, nm, "n")]
    assert thrift._guard(*ok) == torch.device("cuda:0")
    assert thrift._counts(sh) == (nq, nk, nm)
    with pytest.raises(ValueError, match="elements"):  # an undersized Q
        thrift._guard((_FakeCuda(nq - 1), "Q", torch.float16, nq, "n"), *ok[1:])
    with pytest.raises(ValueError, match="cuda:1"):  # K on another device
        thrift._guard(ok[0], (_FakeCuda(nk, device="cuda:1"), "K", torch.float16, nk, "n"))
    with pytest.raises(ValueError, match="bytes"):  # a workspace smaller than the shape needs
        thrift._guard(ok[0], (_FakeCuda(100, torch.uint8), "ws", None, 101, "b"))
    # a float32 workspace counts bytes, not elements
    assert thrift._guard((_FakeCuda(26, torch.float32), "ws", None, 101, "b")) == torch.device("cuda:0")
    with pytest.raises(ValueError, match="float16"):
        thrift._guard((_FakeCuda(nq, torch.float32), "Q", torch.float16, nq, "n"))
    with pytest.raises(ValueError, match="contiguous"):
        thrift._guard((_FakeCuda(nq, contiguous=False), "Q", torch.float16, nq, "n"))
    with pytest.raises(ValueError, match="CUDA"):
        thrift.attention_fused(torch.zeros(nq, dtype=torch.float16), None, None, sh, 0.05)


def test_pooled_entry_points_check_their_arguments_before_launch():
    lib = thrift.lib()
    sh = ctypes.byref(_c(blk=64))
    fake = ctypes.c_void_p(256)
    assert lib.thrift_quantize_pool_nvfp4(fake, 2, sh, fake, fake, fake, None) == 1     # V cannot be pooled
    assert lib.thrift_quantize_pool_nvfp4(None, 0, sh, fake, fake, fake, None) == 1
    assert lib.thrift_quantize_pool_nvfp4(fake, 0, sh, fake, fake, ctypes.c_void_p(258), None) == 1  # misaligned means
    assert lib.thrift_select_blocks_pooled(fake, fake, sh, 1.5, fake, fake, 1 << 30, None) == 1
    assert lib.thrift_select_blocks_pooled(fake, fake, sh, 0.05, fake, fake, 8, None) == 5
