"""The multi-rank logic on CPU with gloo (world size 2).

bench.py: each rank draws an independent batch, the timing is the max over
ranks, and the job rate counts every rank's elements over the slowest rank's
time. Channel sharding (selective_state_space_42_b200.shard): each rank plans
selscan_fwd on its own channel slice through the C ABI (host-only planning),
the slices tile the channels exactly, and the float64 oracle run on each
rank's slice, gathered, equals the oracle on the whole layer."""
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


def _shard_worker(rank, world, port, q):
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import numpy as np
        import oracle
        import selective_state_space_42_b200 as ss
        from selective_state_space_42_b200 import shard
        from selective_state_space_42_b200 import workloads as wl
        # plans of the Mamba-2.8B layer's slices (host only, no device)
        big = wl.WORKLOADS["mamba2p8b_layer"]
        d0, d1 = shard.channel_slice(big.dim, world, rank)
        plan = ss.selscan_fwd_plan(big.batch, big.seqlen, d1 - d0, big.dstate)
        sl = torch.tensor([d0, d1])
        sls = [torch.zeros_like(sl) for _ in range(world)]
        dist.all_gather(sls, sl)
        # oracle on this rank's slice of a small layer, gathered
        w = wl.ScanWorkload("mp_shard", 2, 40, 300, 16, "f32", gate=True, seed=17)
        inp = wl.make_scan_inputs(w)
        a0, a1 = shard.channel_slice(w.dim, world, rank, tile=64)
        part = shard.shard_inputs(inp, a0, a1)
        n = lambda t: None if t is None else t.double().numpy()  # noqa: E731
        args = [n(part[k]) for k in ("x", "delta", "A", "B", "C", "D", "z", "delta_bias")]
        y, h = oracle.default().fwd(*args)
        width = torch.tensor([a1 - a0])
        widths = [torch.zeros_like(width) for _ in range(world)]
        dist.all_gather(widths, width)
        wmax = int(max(int(v) for v in widths))
        ypad = torch.zeros(w.batch, w.seqlen, wmax, dtype=torch.float64)
        ypad[:, :, :a1 - a0] = torch.from_numpy(y)
        ys = [torch.zeros_like(ypad) for _ in range(world)]
        dist.all_gather(ys, ypad)
        whole = None
        if rank == 0:
            full = [n(inp[k]) for k in ("x", "delta", "A", "B", "C", "D", "z", "delta_bias")]
            yw, _ = oracle.default().fwd(*full)
            got = np.concatenate([ys[r][:, :, :int(widths[r])].numpy() for r in range(world)],
                                 axis=2)
            whole = float(np.max(np.abs(got - yw)))
        q.put((rank, [tuple(int(v) for v in t) for t in sls], plan, whole))
    finally:
        dist.destroy_process_group()


def _spawn(target, world=2):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=target, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=180)
    for p in procs:
        if p.is_alive():
            p.kill()
            pytest.fail("rank did not finish")
        assert p.exitcode == 0
    return sorted(q.get(timeout=5) for _ in range(world))


def test_channel_sharded_plan_and_union_gloo():
    res = _spawn(_shard_worker)
    slices = res[0][1]
    assert slices == res[1][1]  # every rank sees the same split
    assert slices[0][0] == 0 and slices[-1][1] == 5120
    assert all(a[1] == b[0] for a, b in zip(slices, slices[1:]))  # no gap, no overlap
    assert all((d1 - d0) % 128 == 0 for d0, d1 in slices)
    for _, _, plan, _ in res:
        # a TMA plan per rank: one pass (1 launch) or aggregates, carry and
        # rescan (3 launches) when a rank's slice has too few tiles for the SMs
        assert plan["launches"] in (1, 3) and plan["chunks"] >= 1
    whole = [r[3] for r in res if r[3] is not None]
    assert whole == [0.0]  # the ranks' slices reproduce the whole layer exactly


def test_channel_slices_properties():
    from selective_state_space_42_b200 import shard
    for dim in (0, 1, 127, 128, 129, 300, 5120, 5121):
        for world in (1, 2, 3, 8, 64):
            sl = shard.channel_slices(dim, world)
            assert len(sl) == world
            assert sl[0][0] == 0 and sl[-1][1] == dim
            assert all(a[1] == b[0] for a, b in zip(sl, sl[1:]))
            assert all(d0 % 128 == 0 or d0 == dim for d0, _ in sl)
            tiles = [-(-(d1 - d0) // 128) for d0, d1 in sl]
            assert max(tiles) - min(tiles) <= 1  # balanced in whole tiles


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
