"""The multi-rank host logic of bench.py with world size 2 over gloo on the CPU: rank setup from the
torchrun environment, the MAX-over-ranks timing collective, per-rank seeds and the whole-job rate."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, root, q):
    import sys
    sys.path.insert(0, root)
    os.environ.update({"RANK": str(rank), "LOCAL_RANK": str(rank), "WORLD_SIZE": str(world),
                       "MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    import bench
    import torch.distributed as dist
    r, w, local = bench.dist_setup("gloo")
    try:
        bench.barrier(w)
        mx = bench.max_over_ranks(10.0 + 5.0 * r, w, device="cpu")
        q.put((r, w, local, mx, bench.rank_seed(r)))
        bench.barrier(w)
    finally:
        dist.destroy_process_group()


def test_two_ranks_gloo(repo_root):
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, repo_root, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=5) for _ in range(world))
    assert [g[0] for g in got] == [0, 1]
    assert all(g[1] == world and g[2] == g[0] for g in got)
    assert all(g[3] == 15.0 for g in got)            # every rank sees the slowest rank's time
    assert got[0][4] != got[1][4]                   # ranks draw different inputs


def test_whole_job_rate_counts_all_ranks():
    import bench
    # 2 ranks, 10 steps of 1.5 TFLOP each, slowest rank 20 ms in total -> 1500 TFLOP/s
    assert abs(bench.whole_job_rate(1.5e12, 10, 2, 20.0) / 1e12 - 1500.0) < 1e-9
    assert bench.whole_job_rate(1.0, 1, 1, 1000.0) == 1.0
