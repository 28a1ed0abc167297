"""Multi-rank host logic of bench.py on CPU (gloo, world size 2).

The decode path has no exchange step, so N GPUs run N independent replicas;
what crosses ranks is only the timing: the max over ranks and the whole-job
aggregate. These run here as two gloo processes on 127.0.0.1."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        import workloads as W
        # each rank times something different; every rank must agree on the max
        mx = bench.max_over_ranks([10.0 + rank, 5.0 - rank, 1.5])
        # replicas draw distinct data (layer index = rank)
        w = W.WORKLOADS["tiny_fp32"].with_(N=16, S_obs=2)
        _, k, _ = W.gen_layer(w, layer=rank)
        q.put((rank, mx, float(k.double().sum())))
    finally:
        dist.destroy_process_group()


def test_two_rank_max_and_distinct_replicas():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    res.sort()
    for _, mx, _ in res:
        assert mx == [11.0, 5.0, 1.5]
    assert res[0][2] != res[1][2]


def test_aggregate_is_whole_job():
    import bench
    # 2 ranks, 1 GB per rank per step, 10 ms per step (max over ranks) -> 200 GB/s
    assert bench.aggregate_gbs(2, 10**9, 10.0) == pytest.approx(200.0)
    assert bench.max_over_ranks([3.0, 4.0]) == [3.0, 4.0]   # single process: identity
