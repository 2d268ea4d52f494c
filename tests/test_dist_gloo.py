"""Multi-rank host logic of the benchmark on CPU (gloo, world size 2): every rank processes
its own batch (weak scaling, no collective on the data path); the step time reported is
the max over ranks and the throughput is the whole job's."""
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


def _worker(rank, ws, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(ws), LOCAL_RANK=str(rank))
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    import workloads as W
    dist.init_process_group("gloo", rank=rank, world_size=ws)
    try:
        assert bench.dist_env() == (ws, rank, rank)
        # Each rank draws its own batch: different seeds give different data.
        x = W.make_inputs(W.TINY_F32, seed=rank)["x"]
        t = torch.tensor([float(x.sum())])
        gathered = [torch.zeros(1) for _ in range(ws)]
        dist.all_gather(gathered, t)
        distinct = len({float(g) for g in gathered}) == ws
        # Device time of the slowest rank is what the job took.
        slowest = bench.max_over_ranks(10.0 + rank, ws, device="cpu")
        bench.barrier(ws)
        q.put((rank, slowest, distinct))
    finally:
        dist.destroy_process_group()


def test_two_rank_max_time_and_weak_scaling():
    ws = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, ws, port, q)) for r in range(ws)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=5) for _ in range(ws))
    assert [r[1] for r in res] == [11.0, 11.0]
    assert all(r[2] for r in res)

    import bench
    import workloads as W
    w = W.USAGE_F32
    one, unit = bench.unit_value(w, "direct", 1e-3, 1)
    two, _ = bench.unit_value(w, "direct", 1e-3, 2)
    assert unit == "TFLOP/s" and two == pytest.approx(2 * one)
    assert one == pytest.approx(w.flops() / 1e-3 / 1e12)
