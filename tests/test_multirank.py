"""The N > 1 path of bench.py on CPU: two ranks over gloo.

The scan partitions into independent sequences, so ranks never exchange data;
the only collective is the MAX of the timed region.  These tests run the same
helpers bench.py uses under torch.distributed with world_size 2 and check the
whole-job accounting (weak scaling: N ranks x their own batch / slowest time),
the per-rank input seeds, and that ranks draw different batches of the same
workload recipe.
"""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    import datetime
    import torch
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    import bench
    import s6_inputs as SI
    # each rank pretends its timed region took a different time
    local_ms = [12.0, 15.0][rank]
    mx = bench.max_over_ranks(local_ms, world, torch.device("cpu"))
    value, ms_step = bench.job_throughput(1000, world, mx, 10)
    inp = SI.scan_inputs("long_seq", Bt=1, L=8, d=16, seed=bench.rank_seed(4, rank))
    digest = float(np.asarray(inp["x"], dtype=np.float64).sum())
    bench.barrier(world)
    q.put((rank, mx, value, ms_step, digest))
    dist.destroy_process_group()


def test_two_ranks_gloo():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    # both ranks agree on the slowest time and on the job throughput
    assert res[0][1] == res[1][1] == 15.0
    assert res[0][2] == res[1][2] == pytest.approx(2 * 1000 / (1.5e-3) / 1e9)
    assert res[0][3] == 1.5
    # ranks draw different batches
    assert res[0][4] != res[1][4]


def test_single_rank_accounting():
    import bench
    assert bench.max_over_ranks(3.0, 1, None) == 3.0
    v, ms = bench.job_throughput(201326592, 1, 1660.0, 1000)
    assert ms == pytest.approx(1.66)
    assert v == pytest.approx(201326592 / 1.66e-3 / 1e9)
    assert bench.rank_seed(4, 0) == 4 and bench.rank_seed(4, 3) == 7
