"""The N>1 host logic of bench.py on CPU with two gloo ranks: every rank draws
its own batch (weak scaling, no data-path collective), the step time is the
maximum over ranks, and the whole-job value counts every rank's tokens."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        from chunked_gated_delta_ckda_b200 import workloads as W
        wl = W.LAYER_FWDBWD
        w = W.Workload(**{**wl.__dict__, "seed": bench.rank_seed(wl.seed, rank)})
        x = W.make(w, B=1, T=64, H=2)
        fp = float(x["q"].float().sum())
        ms = 10.0 + 5.0 * rank                      # rank 1 is the slow one
        mx = bench.reduce_max(ms, world)
        val = bench.aggregate(32768, world, mx)
        t = torch.tensor([fp])
        gathered = [torch.zeros(1) for _ in range(world)]
        dist.all_gather(gathered, t)
        out[rank] = (mx, val, [float(g) for g in gathered])
    finally:
        dist.destroy_process_group()


def test_two_ranks_weak_scaling_and_max_timing():
    world = 2
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    for r in range(world):
        mx, val, fps = out[r]
        assert mx == 15.0                                # slowest rank's time on every rank
        assert val == pytest.approx(2 * 32768 / 0.015)   # tokens of both ranks / slowest time
        assert fps[0] != fps[1]                          # each rank its own batch


def test_single_process_helpers():
    import bench
    assert bench.reduce_max(3.5, 1) == 3.5
    assert bench.aggregate(1000, 1, 1.0) == pytest.approx(1e6)
    assert bench.rank_seed(2, 0) == 2 and bench.rank_seed(2, 3) == 3002
