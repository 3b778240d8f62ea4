"""The benchmark's multi-rank logic on host processes (gloo, world size 2):
replicas share nothing on the data path; the only cross-rank steps are the
barrier and the max-over-ranks of the device-timed interval, and the job's
throughput counts every rank's cycles over the slowest rank's time."""
import os
import socket

import pytest
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, q):
    os.environ.update({"RANK": str(rank), "LOCAL_RANK": str(rank), "WORLD_SIZE": str(world),
                       "MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    w, r, _ = bench.setup_dist(backend="gloo")
    ms = 100.0 + 50.0 * r            # rank 1 is the slower replica
    bench.barrier(w)
    ms_max = bench.max_over_ranks(ms, w)
    q.put((r, w, ms_max, bench.job_throughput(w, 10, ms_max)))
    import torch.distributed as dist
    dist.destroy_process_group()


def test_two_replicas_report_the_slowest_rank_and_the_whole_job():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    for r, w, ms_max, value in res:
        assert w == 2 and ms_max == 150.0
        assert value == pytest.approx(2 * 10 / 0.150)


def test_single_rank_needs_no_process_group():
    assert bench.max_over_ranks(12.5, 1) == 12.5
    assert bench.job_throughput(1, 100, 50.0) == pytest.approx(2000.0)
