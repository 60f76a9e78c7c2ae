"""The multi-rank logic of bench.py on CPU with gloo (world size 2): each rank
draws an independent batch, the timing is the max over ranks, and the job
rate counts every rank's elements over the slowest rank's time."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        from selective_state_space_42_b200 import workloads as wl
        w = wl.ScanWorkload("mp", 1, 8, 4, 2, "f32", gate=False, seed=5)
        x = wl.make_scan_inputs(w.scaled(seed=bench.rank_seed(w, rank)))["x"]
        xs = [torch.zeros_like(x) for _ in range(world)]
        dist.all_gather(xs, x)
        ms = 10.0 + 5.0 * rank
        mx = bench.max_over_ranks(ms, dist, torch.device("cpu"))
        q.put((rank, mx, not torch.equal(xs[0], xs[1]),
               bench.job_rate(w.elements, world, 3, mx)))
    finally:
        dist.destroy_process_group()


def test_two_ranks_gloo():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    for p in procs:
        if p.is_alive():
            p.kill()
            pytest.fail("rank did not finish")
        assert p.exitcode == 0
    res = sorted(q.get(timeout=5) for _ in range(world))
    for rank, mx, distinct, rate in res:
        assert mx == 15.0  # both ranks see the slowest rank's time
        assert distinct  # the ranks' batches are independent draws
        assert rate == pytest.approx(1 * 8 * 4 * 2 * 2 * 3 / 0.015)
