"""thrift_select_blocks_static: the selection for callers that cannot allocate
device memory (their GPU memory belongs to another allocator, or they are
hooks with no way to allocate).  It runs the selection kernels on the
library's static 16 MiB scratch array instead of a caller workspace.

This file is collected last on purpose, and the test passes both alone in a
fresh process and after the other tests: the scratch is shared by every call
and keeps the previous call's contents, which the selection kernels must
fully overwrite."""
import ctypes

import numpy as np
import pytest
import torch

import fp16_block_attention_b200 as thrift
import synth

pytestmark = pytest.mark.gpu


def _dev(*arrs):
    return [torch.from_numpy(np.ascontiguousarray(a)).cuda() for a in arrs]


def _shape(w):
    return thrift.Shape(w.B, w.Hq, w.Hkv, w.N, w.D, w.blk, w.causal, w.sm_scale)


def test_static_selection_matches_the_workspace_entry_point_on_two_calls_in_a_row():
    # Two calls in a row on different shapes: the second finds the first's data
    # in the shared scratch.  Masks are compared bit for bit (same kernels).
    for w in (synth.GQA_N32K, synth.CAUSAL_MH_N8K):
        assert thrift.select_workspace_bytes(_shape(w)) <= thrift.SELECT_STATIC_BYTES
        Q, K, _ = synth.generate(w)
        Qd, Kd = _dev(Q, K)
        sh = _shape(w)
        m_static = thrift.select_blocks_static(Qd, Kd, sh, w.rho)
        m_ws = thrift.select_blocks(Qd, Kd, sh, w.rho)
        torch.cuda.synchronize()
        assert torch.equal(m_static, m_ws), w.name
        valid = sh.nb * (sh.nb + 1) // 2
        assert int(m_static.sum()) == w.B * w.Hq * int(np.ceil(w.rho * valid - 1e-9))


def test_static_selection_rejects_shapes_beyond_the_scratch():
    big = synth.GQA_N128K
    sh = _shape(big)
    assert thrift.select_workspace_bytes(sh) > thrift.SELECT_STATIC_BYTES
    fake = ctypes.c_void_p(256)
    status = thrift.lib().thrift_select_blocks_static(fake, fake, ctypes.byref(sh.c()), 0.05, fake, None)
    assert status == 5  # THRIFT_ERR_WORKSPACE
