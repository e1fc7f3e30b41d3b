"""Host side of the vocabulary-sharded build on CPU (no GPU).

  * dt_shard_range splits the vocabulary into whole 128-token tiles that
    cover it exactly once, lower ranks first, as evenly as tiles allow;
  * tree_build_sharded's wave loop, run on world_size 2 and 3 gloo process
    groups with the library calls replaced by stand-ins that write each
    rank's id and the wave into its partial block: every rank must issue
    begin, then per wave GEMM -> all-gather -> frontier, and every rank's
    frontier must see all blocks in rank order.
"""
import datetime
import os
import socket
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.parametrize("V", [512, 1000, 151936, 128 * 7 + 5])
@pytest.mark.parametrize("world", [1, 2, 3, 4, 8])
def test_shard_range_partitions_the_vocabulary(V, world):
    import draft_tree_construction_markov_b200 as dt
    T = (V + 127) // 128
    if world > T:
        pytest.skip("more ranks than tiles")
    parts = [dt.shard_range(V, world, r) for r in range(world)]
    pos = 0
    for vb, vl in parts:
        assert vb == pos and vb % 128 == 0 and vl > 0
        pos = vb + vl
    assert pos == V
    tiles = [(vl + 127) // 128 for _, vl in parts]
    assert max(tiles) - min(tiles) <= 1
    assert dt.shard_range(V, world, world) == (0, 0)   # rank outside the world


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import torch
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import draft_tree_construction_markov_b200 as dt
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    cfg = dt.shard_cfg(1, 4, 4096, 64, 2, 8, world)
    pb = dt.sharded_partials_bytes(cfg)
    log = []
    seen = []

    def begin(*a, **k):
        log.append("begin")

    def gemm(c, wave, rk, *a, **k):
        part = a[-1]
        part.fill_(0)
        part[:8].copy_(torch.tensor([rk, wave, 0, 0, 0, 0, 0, 0], dtype=torch.uint8))
        log.append(("gemm", wave))

    def frontier(c, wave, gathered, *a, **k):
        blocks = gathered.view(world, pb)
        seen.append([(int(b[0]), int(b[1])) for b in blocks])
        log.append(("frontier", wave))

    dt.sharded_build_begin, dt.sharded_build_gemm, dt.sharded_build_frontier = begin, gemm, frontier
    partials = torch.empty(pb, dtype=torch.uint8)
    gathered = torch.empty(world * pb, dtype=torch.uint8)

    def all_gather(dst, src):
        log.append("gather")
        dist.all_gather_into_tensor(dst, src)

    dt.tree_build_sharded(cfg, rank, None, None, None, None, None, None, None, None, partials,
                          gathered, all_gather)
    q.put((rank, log, seen))
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_wave_loop_gathers_in_rank_order(world):
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
    Bk = 4
    want_log = ["begin"] + [e for wv in range(Bk)
                            for e in (("gemm", wv), "gather", ("frontier", wv))]
    for rank, log, seen in out:
        assert log == want_log
        assert seen == [[(r, wv) for r in range(world)] for wv in range(Bk)]
