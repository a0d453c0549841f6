"""Multi-rank logic of bench.py on CPU (gloo, world size 2): the timed region is the max
over ranks and the value aggregates every rank's replica (weak scaling)."""
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
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    mine = [12.5, 40.0][rank]
    got = bench.max_over_ranks(mine, world, torch.device("cpu"))
    val = bench.aggregate_tokens_per_s(8, 16, world, got)
    dist.barrier()
    dist.destroy_process_group()
    q.put((rank, got, val))


def test_bench_rank_aggregation_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, got, val in res:
        assert got == 40.0                                   # max over ranks
        assert val == pytest.approx(2 * 8 * 16 / 0.040)      # both replicas' tokens


def test_single_rank_is_identity():
    import bench
    assert bench.max_over_ranks(3.0, 1, torch.device("cpu")) == 3.0
    assert bench.aggregate_tokens_per_s(8, 10, 1, 1000.0) == pytest.approx(80.0)
