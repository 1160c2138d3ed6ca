"""The multi-rank plumbing of bench.py on CPU: two gloo ranks on 127.0.0.1.

The solve itself needs no collective (replicas only); what runs on several
GPUs is the barrier, the max-over-ranks time and the whole-job value.
"""
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


ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _worker(rank, world, port, q):
    import sys
    if ROOT not in sys.path:
        sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port),
                      RANK=str(rank), WORLD_SIZE=str(world))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    import bench
    from nonlinear_rnn_paragru_b200.inputs import WORKLOADS, make_inputs
    ms = 1.0 + rank                      # rank 1 is the slow one
    bench.barrier(world)
    ms_max = bench.max_over_ranks(ms, world, device="cpu")
    w = WORKLOADS[1]
    x = make_inputs(w, seed=bench.rank_seed(rank))
    q.put((rank, ms_max, bench.weak_value(world, w.tokch, ms_max),
           float(x["u"].float().sum())))
    dist.barrier()
    dist.destroy_process_group()


def test_two_gloo_ranks_take_the_max_and_count_all_units():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(world))
    from nonlinear_rnn_paragru_b200.inputs import WORKLOADS
    for rank, ms_max, value, _ in res:
        assert ms_max == 2.0
        assert value == pytest.approx(2 * WORKLOADS[1].tokch / 2e-3)
    assert res[0][3] != res[1][3]        # independent problems per rank
