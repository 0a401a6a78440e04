"""Host logic of the multi-rank bench path on CPU: world_size 2 over gloo.

Every rank quantizes its own layer (weak scaling, no collective on the data
path); the only collectives are the barrier around the timed region and the
max over ranks of the elapsed time.
"""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import datetime

    import torch.distributed as dist

    import bench
    dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    bench.barrier(world)
    t = bench.max_over_ranks(10.0 + rank, world)
    W, X, X2 = bench.make_inputs(rank, n=64, workload="q_proj_7b")
    q.put((rank, t, float(W[0, :4].sum()), int(X[0, :4].astype(np.int64).sum())))
    bench.barrier(world)
    dist.destroy_process_group()


@pytest.mark.timeout(300)
def test_two_ranks_time_max_and_distinct_layers():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=240) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert res[0][1] == res[1][1] == 11.0          # max over ranks
    assert res[0][2] != res[1][2]                  # each rank its own layer
    assert res[0][3] != res[1][3]
