"""The kv-head split on the device: a rank that runs kv heads [hk0, hk1) of a
problem, with their query heads, through views of the whole tensors (pointer
offsets, no copies) gets exactly the slice of the whole problem's selection
mask and output.  This is what lets the split run without a data-path
collective; it runs the ranks' shares one after another on one GPU."""
import pytest
import torch

import bench
import fp16_block_attention_b200 as thrift
import synth
from gpu_helpers import shape_of

CASES = [
    synth.GQA_N32K.with_(N=2048, Hq=8, Hkv=4),               # blk 128, 16 key tiles
    synth.GQA_N32K.with_(N=1984, Hq=8, Hkv=4, blk=64),       # one-pass blk-64 kernel, last query tile half full
]


@pytest.mark.gpu
@pytest.mark.parametrize("w", CASES, ids=lambda w: f"N{w.N}_blk{w.blk}")
@pytest.mark.parametrize("world", [2, 4])
def test_head_share_equals_slice_of_whole_problem(w, world):
    Q, K, V = synth.generate(w)
    Qd, Kd, Vd = (torch.from_numpy(a).cuda() for a in (Q, K, V))
    sh = shape_of(w)
    whole_mask = thrift.select_blocks(Qd, Kd, sh, w.rho)
    whole = thrift.attention_fused(Qd, Kd, Vd, sh, w.rho)
    torch.cuda.synchronize()
    for r in range(world):
        (hk0, hk1), (hq0, hq1) = bench.rank_heads(w, r, world)
        q, k, v = Qd[:, hq0:hq1], Kd[:, hk0:hk1], Vd[:, hk0:hk1]
        assert q.is_contiguous() and k.is_contiguous() and v.is_contiguous()
        assert q.data_ptr() == Qd.data_ptr() + hq0 * w.N * w.D * 2
        part = bench.head_workload(w, r, world)
        psh = shape_of(part)
        mask = thrift.select_blocks(q, k, psh, w.rho)
        out = thrift.attention_fused(q, k, v, psh, w.rho)
        assert torch.equal(mask, whole_mask[:, hq0:hq1])
        assert torch.equal(out.view(torch.int16), whole[:, hq0:hq1].view(torch.int16))
    assert thrift.last_device_error() == 0
