"""The multi-rank path of bench.py on CPU: two `gloo` ranks.

bench.py runs one independent system per rank (seeded by rank) with no
data-path collective; the job's time is the slowest rank's and its units are
the sum over ranks.  These tests run the same host logic — the reductions
bench.py uses and the per-rank seeding — as two processes over gloo on
127.0.0.1, so the N > 1 path is covered without GPUs.
"""
import multiprocessing as mp
import os
import socket
import sys
from datetime import timedelta

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank: int, ws: int, port: int, out):
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    import bench
    from equivariant_graph_attention_b200 import synth
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=ws, timeout=timedelta(seconds=60))
    try:
        # rank r took 10 + r ms for 100 * (r + 1) units
        res = {
            "max": bench.max_over_ranks(10.0 + rank, "cpu"),
            "sum": bench.sum_over_ranks(100.0 * (rank + 1), "cpu"),
            "rate": bench.job_rate(100.0 * (rank + 1), 10.0 + rank, "cpu"),
        }
        # every rank builds its own system: same shape, different atoms
        wl = synth.WORKLOADS["uniform64_l1_f32"]
        d = synth.make(wl, seed=rank)
        digests = [None] * ws
        dist.all_gather_object(digests, (d["pos_q"].shape, int(np.abs(d["pos_q"]).sum())))
        res["shapes_equal"] = all(x[0] == digests[0][0] for x in digests)
        res["systems_differ"] = len({x[1] for x in digests}) == ws
        dist.barrier()
        out.put((rank, res))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_reduce_like_the_bench():
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    results = dict(out.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for r in (0, 1):
        res = results[r]
        assert res["max"] == 11.0                     # slowest rank's time
        assert res["sum"] == 300.0                    # units of both ranks
        assert abs(res["rate"] - 300.0 / 0.011) < 1e-6 * res["rate"]
        assert res["shapes_equal"] and res["systems_differ"]


def test_single_process_reductions_are_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.5, "cpu") == 3.5
    assert bench.sum_over_ranks(7.0, "cpu") == 7.0
    assert bench.job_rate(50.0, 10.0, "cpu") == 5000.0
