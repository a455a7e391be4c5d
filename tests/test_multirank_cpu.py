"""The multi-rank path of the benchmark on CPU (gloo, world size 2): every rank times its
own replica (weak scaling, no collective on the data path) and the job's time is the
maximum over ranks."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        mine = 10.0 + 3.5 * rank
        q.put((rank, bench.max_over_ranks(mine, dist, "cpu"), bench.rank_seed(1001, rank)))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_replica_seeds():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    assert [r[1] for r in res] == [13.5, 13.5]          # every rank sees the slowest rank's time
    assert res[0][2] != res[1][2]                       # replicas draw different inputs


def test_single_rank_is_identity():
    assert bench.max_over_ranks(4.25) == 4.25
