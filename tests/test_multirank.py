"""Multi-rank host logic of bench.py on CPU (gloo, world size 2).

On several GPUs every rank runs its own replica of the workload (instances are
independent, so there is no exchange step); the step time is the slowest
rank's and the job's value counts every rank's work. These tests run that
logic with two gloo ranks and no GPU.
"""

import os
import socket
import sys

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    import bench
    local_ms = [3.0, 5.0][rank]
    slowest = bench.max_over_ranks(local_ms, world)
    value = bench.job_value(2e9, world, slowest * 1e-3)
    out.put((rank, slowest, value))
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.timeout(120)
def test_two_gloo_ranks_take_the_slowest_rank_and_count_all_work():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    got = sorted(q.get(timeout=90) for _ in procs)
    for p in procs:
        p.join(timeout=30)
        assert p.exitcode == 0
    for rank, slowest, value in got:
        assert slowest == 5.0                      # max over ranks, on every rank
        assert value == pytest.approx(2 * 2e9 / 5e-3 / 1e12)  # both ranks' work / slowest time


def test_single_rank_is_its_own_maximum():
    import bench
    assert bench.max_over_ranks(7.5, 1) == 7.5
    assert bench.job_value(1e12, 1, 1.0) == pytest.approx(1.0)
