"""The multi-rank plumbing of bench.py on CPU: two `gloo` ranks, each with its
own seeded problem of the same shape, the slowest rank's time taken by an
all-reduce max, and whole-job throughput summed over ranks.  No GPU."""
import io
import os
import socket
import sys
from contextlib import redirect_stdout

import numpy as np
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

WORLD = 2


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, port, out_dir):
    import datetime

    import torch.distributed as dist

    import bench
    import synth

    os.environ.update(RANK=str(rank), WORLD_SIZE=str(WORLD), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=WORLD,
                            timeout=datetime.timedelta(seconds=60))
    try:
        assert bench.dist_env() == (rank, WORLD, rank)
        w = bench.rank_workload(synth.TINY_NONCAUSAL_D64, rank, WORLD)
        Q, K, V = synth.generate(w)
        # per-rank "step time": rank 1 is the slow one
        ms = 2.0 + 3.0 * rank
        slowest = bench.reduce_max(ms)
        digests = [None] * WORLD
        dist.all_gather_object(digests, (w.seed, Q.shape, float(np.float64(Q.astype(np.float64).sum()))))
        value = bench.whole_job_tflops(w.flops(), slowest, WORLD)
        # the reference arm runs on rank 0 alone: other ranks return at once, printing nothing
        buf = io.StringIO()
        with redirect_stdout(buf):
            ran = bench.run_reference(type("A", (), dict(steps=1, warmup=0, ref_rows=1))) if rank == 1 else None
        np.save(os.path.join(out_dir, f"r{rank}.npy"),
                np.array([slowest, value, float(len(buf.getvalue())), float(ran is None)], np.float64))
        if rank == 0:
            import pickle
            with open(os.path.join(out_dir, "digests.pkl"), "wb") as f:
                pickle.dump(digests, f)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_weak_scaling(tmp_path):
    import pickle

    import bench
    import synth

    ctx = mp.get_context("spawn")
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, port, str(tmp_path))) for r in range(WORLD)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        if p.is_alive():
            p.kill()
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]

    r0, r1 = (np.load(tmp_path / f"r{r}.npy") for r in range(WORLD))
    # both ranks see the slowest rank's time
    assert r0[0] == r1[0] == 5.0
    # whole-job value: both ranks' work over the slowest time, identical on every rank
    flops = synth.TINY_NONCAUSAL_D64.flops()
    assert r0[1] == r1[1] == WORLD * flops / 5e-3 / 1e12
    # the reference arm did nothing on rank 1
    assert r1[2] == 0.0 and r1[3] == 1.0
    # independent problems: same shapes, different seeds and data
    digests = pickle.load(open(tmp_path / "digests.pkl", "rb"))
    (s0, shape0, sum0), (s1, shape1, sum1) = digests
    assert shape0 == shape1 and s0 != s1 and sum0 != sum1
    # one rank is the plain workload, unchanged
    assert bench.rank_workload(synth.TINY_NONCAUSAL_D64, 0, 1) is synth.TINY_NONCAUSAL_D64


def _heads_rank_main(rank, world, port, out_dir):
    import datetime

    import torch.distributed as dist

    import bench
    import synth

    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        w = synth.GQA_N32K
        (hk0, hk1), (hq0, hq1) = bench.rank_heads(w, rank, world)
        mine = bench.head_workload(w, rank, world)
        shares = [None] * world
        dist.all_gather_object(shares, (rank, hk0, hk1, hq0, hq1, mine.Hq, mine.Hkv, mine.flops()))
        # every rank computes the same whole-job FLOPs from the same slowest time
        ms = bench.reduce_max(1.0 + rank)
        value = bench.job_flops(w, world, "heads") / (ms * 1e-3) / 1e12
        if rank == 0:
            import pickle
            with open(os.path.join(out_dir, "shares.pkl"), "wb") as f:
                pickle.dump((shares, ms, value), f)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_split_one_problem_by_kv_heads(tmp_path):
    """--split heads: the ranks' kv-head ranges tile [0, Hkv) exactly, each
    carries its G query heads, and the ranks' FLOPs add up to the problem's."""
    import pickle

    import bench
    import synth

    ctx = mp.get_context("spawn")
    port = _free_port()
    procs = [ctx.Process(target=_heads_rank_main, args=(r, WORLD, port, str(tmp_path))) for r in range(WORLD)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        if p.is_alive():
            p.kill()
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    shares, ms, value = pickle.load(open(tmp_path / "shares.pkl", "rb"))
    w = synth.GQA_N32K
    G = w.Hq // w.Hkv
    assert [s[0] for s in shares] == list(range(WORLD))
    assert shares[0][1] == 0 and shares[-1][2] == w.Hkv
    assert all(a[2] == b[1] for a, b in zip(shares, shares[1:]))
    for _, hk0, hk1, hq0, hq1, hq, hkv, _f in shares:
        assert (hq0, hq1) == (hk0 * G, hk1 * G) and (hq, hkv) == (hq1 - hq0, hk1 - hk0) and hkv >= 1
    assert sum(s[7] for s in shares) == w.flops()
    assert ms == float(WORLD)
    assert value == w.flops() / (WORLD * 1e-3) / 1e12


def test_kv_head_ranges_tile_for_every_world_size():
    import pytest

    import bench
    import synth

    for w in (synth.GQA_N32K, synth.BATCHED_GQA_N16K, synth.CAUSAL_MH_N8K):
        for world in range(1, w.Hkv + 1):
            covered = []
            for r in range(world):
                (hk0, hk1), (hq0, hq1) = bench.rank_heads(w, r, world)
                assert hk1 > hk0
                covered += list(range(hk0, hk1))
            assert covered == list(range(w.Hkv))
            assert sum(bench.head_workload(w, r, world).flops() for r in range(world)) == w.flops()
        assert bench.job_flops(w, 4, "problems") == 4 * w.flops()
        with pytest.raises(ValueError):
            bench.rank_heads(w, 0, w.Hkv + 1)


def test_selection_is_separable_by_kv_head():
    """The property the split rests on: the oracle's selection of a slice of
    the kv heads (with their query heads) is that slice of the whole problem's
    selection, so the ranks' masks, and outputs, are the whole problem's."""
    import bench
    import oracle
    import synth

    w = synth.GQA_N32K.with_(N=512, Hq=8, Hkv=4)
    Q, K, _ = synth.generate(w)
    whole = oracle.select(Q, K, w.blk, w.causal, w.sm_scale, w.rho)
    for world in (2, 4):
        for r in range(world):
            (hk0, hk1), (hq0, hq1) = bench.rank_heads(w, r, world)
            part = oracle.select(np.ascontiguousarray(Q[:, hq0:hq1]), np.ascontiguousarray(K[:, hk0:hk1]),
                                 w.blk, w.causal, w.sm_scale, w.rho)
            assert np.array_equal(part, whole[:, hq0:hq1])
