"""Host-side logic of the multi-GPU benchmark path on CPU: two gloo ranks.

Each rank runs an independent request (weak scaling, no data-path
collective); the only collective is the max of the per-rank timed device
time, and the whole-job value counts the units of every rank."""
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


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    import bench
    try:
        r, w, local = bench.dist_env()
        ms = 100.0 + 50.0 * rank          # rank 1 is the slowest
        mx = bench.max_over_ranks(ms, torch.device("cpu"))
        val = bench.weak_scaling_value(16384, 10, w, mx)
        wl = bench.wl_for_rank("glm_bf16_L128k", r)
        q.put((rank, r, w, mx, val, wl.seed, wl.L))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_ranks_max_and_weak_value():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    ps = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in ps:
        p.start()
    res = sorted(q.get(timeout=120) for _ in ps)
    for p in ps:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, r, w, mx, val, seed, L in res:
        assert (r, w) == (rank, 2)
        assert mx == 150.0                                  # max over ranks
        assert val == pytest.approx(2 * 16384 * 10 / 0.150)  # units of both ranks
        assert seed == rank and L == 131072                  # independent requests


def test_single_process_has_no_collective():
    import bench
    assert bench.max_over_ranks(3.5, torch.device("cpu")) == 3.5
    assert bench.weak_scaling_value(100, 2, 1, 1000.0) == pytest.approx(200.0)
