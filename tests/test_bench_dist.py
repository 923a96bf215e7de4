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
