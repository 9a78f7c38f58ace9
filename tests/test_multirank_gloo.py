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


def _shard_worker(rank, world, port, q):
    """Each rank takes its share of every query's candidate list (a range of
    128-slot tiles), keeps that share's top k, and the ranks exchange and
    merge them through sharded.exchange_and_merge (gloo here; NCCL on GPUs).
    The merge here is a CPU restatement; the library's merge kernel is
    checked on the GPU."""
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import datetime

    import numpy as np
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    from ivf_top_key_b200 import sharded
    try:
        g = np.random.default_rng(3)              # the same data on every rank
        T, n, k = 5, 1000, 37
        scores = np.round(g.standard_normal((T, n)), 2).astype(np.float32)  # many exact ties
        ids = np.stack([g.permutation(5000)[:n] for _ in range(T)]).astype(np.int32)

        def topk(sc, idv, kk):
            order = np.lexsort((idv, -sc))[:kk]
            o_i = np.full(kk, -1, np.int32)
            o_s = np.full(kk, -np.inf, np.float32)
            o_i[:order.size], o_s[:order.size] = idv[order], sc[order]
            return o_i, o_s

        tiles = (n + 127) // 128
        t0, t1 = rank * tiles // world, (rank + 1) * tiles // world
        lo, hi = t0 * 128, min(n, t1 * 128)
        part = [topk(scores[i, lo:hi], ids[i, lo:hi], k) for i in range(T)]
        p_ids = torch.from_numpy(np.stack([p[0] for p in part]))
        p_sc = torch.from_numpy(np.stack([p[1] for p in part]))

        def cpu_merge(a_ids, a_sc, kk):
            res = [topk(a_sc[:, i].reshape(-1).numpy(), a_ids[:, i].reshape(-1).numpy(), kk)
                   for i in range(a_ids.shape[1])]
            res = [(r_i[r_i >= 0], r_s[r_i >= 0]) for r_i, r_s in res]
            out = np.full((a_ids.shape[1], kk), -1, np.int32)
            for i, (r_i, _) in enumerate(res):
                out[i, :r_i.size] = r_i
            return out

        merged = sharded.exchange_and_merge(p_ids, p_sc, k, cpu_merge)
        want = np.stack([topk(scores[i], ids[i], k)[0] for i in range(T)])
        q.put((rank, bool(np.array_equal(merged, want))))
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_ranks_sharded_exchange_gives_the_global_topk(world):
    """2 ranks split the 8 tiles of each list evenly, 3 ranks unevenly
    (2, 3 and 3 tiles)."""
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    ps = [ctx.Process(target=_shard_worker, args=(r, world, port, q)) for r in range(world)]
    for p in ps:
        p.start()
    res = sorted(q.get(timeout=120) for _ in ps)
    for p in ps:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert res == [(r, True) for r in range(world)]
