"""Host side of the multi-GPU path on CPU: world_size-2 gloo process groups.

The round has no exchange step, so N GPUs run N independent replicas; the
only collectives are the timing barrier and the max-over-ranks reduction of
the timed region, and the job's throughput counts every rank's rounds over
the slowest rank's time.  These tests run those host steps of bench.py with
the gloo backend (no GPU).
"""
import datetime
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    r, w, local = bench.dist_env()
    ms = [10.0, 12.5, 11.0, 9.0][rank]   # each rank's own timed region
    dist.barrier()
    ms_max = bench.max_over_ranks(ms, w, "cpu")
    value = bench.job_throughput(100, w, ms_max)
    q.put((rank, r, w, local, ms_max, value))
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 4])
def test_replica_timing_is_max_over_ranks(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    slowest = max([10.0, 12.5, 11.0, 9.0][:world])
    for rank, (rk, r, w, local, ms_max, value) in enumerate(out):
        assert (rk, r, w, local) == (rank, rank, world, rank)
        assert ms_max == slowest
        assert value == pytest.approx(world * 100 / (slowest / 1e3))


def test_single_process_defaults():
    sys.path.insert(0, ROOT)
    import bench
    for k in ("RANK", "WORLD_SIZE", "LOCAL_RANK"):
        os.environ.pop(k, None)
    assert bench.dist_env() == (0, 1, 0)
    assert bench.max_over_ranks(7.5, 1, "cpu") == 7.5
    assert bench.job_throughput(10, 1, 5.0) == pytest.approx(2000.0)
