"""Multi-GPU runs are replicas: each rank decodes its own batch with no
data-path collective; only the timing is combined (max over ranks). These
tests run that host logic as two gloo ranks on the CPU."""
import os
import socket
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, per_rank_times, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import datetime
    torch.distributed.init_process_group("gloo", rank=rank, world_size=world,
                                         timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        step_s, part_s = bench.max_over_ranks(per_rank_times[rank], world, torch.device("cpu"))
        value = bench.job_throughput(1e9, world, step_s)
        q.put((rank, step_s, part_s, value))
    finally:
        torch.distributed.destroy_process_group()


def test_two_replicas_report_the_slowest_rank():
    world, port = 2, _free_port()
    times = [[2e-3, 1e-3], [3e-3, 0.5e-3]]
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank, args=(r, world, port, times, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    res = sorted(q.get(timeout=5) for _ in range(world))
    for rank, step_s, part_s, value in res:
        assert step_s == pytest.approx(3e-3) and part_s == pytest.approx(1e-3)
        # both replicas' bytes over the slowest rank's step time
        assert value == pytest.approx(2 * 1e9 / 3e-3 / 1e9)


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks([1.0, 2.0], 1, torch.device("cpu")) == [1.0, 2.0]
    assert bench.job_throughput(5e9, 1, 0.5) == pytest.approx(10.0)
