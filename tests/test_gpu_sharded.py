"""The vocabulary-sharded build on one GPU, its ranks emulated as one GEMM
launch per vocabulary shard writing into the gathered partial buffer (every
rank's frontier would see exactly these bytes after the all-gather).

Trees must equal the oracle's unsharded tree exactly (tokens, parents,
depths, ranks, masks, counts), keys within 1e-5, for 2 to 3 shards,
ragged shards and full size.
"""
import numpy as np
import pytest
import torch

from gen import make_workload

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import draft_tree_construction_markov_b200 as dt
    from draft_tree_construction_markov_b200 import _lib
    from tests.gpu_util import build_inputs, run_build, tree_to_host
    from tests.test_gpu_build import compare_tree


def run_sharded(w, world):
    x = build_inputs(w)
    cfg = dt.shard_cfg(w.batch, w.Bk, w.V, w.r, w.k, w.Nmax, world)
    assert cfg.ncta >= 1
    shards = [dt.shard_range(w.V, world, r) for r in range(world)]
    assert shards[0][0] == 0 and sum(n for _, n in shards) == w.V
    Bm = [x["markov_b"][vb:vb + vl].contiguous() for vb, vl in shards]
    ws = dt.workspace(dt.sharded_workspace_bytes(cfg))
    pb = dt.sharded_partials_bytes(cfg)
    gathered = torch.empty(world * pb, dtype=torch.uint8, device="cuda")
    tree = dt.Tree.empty(w.batch, w.Nmax, w.V)
    dt.sharded_build_begin(cfg, x["root_token"], x["n_budget"], x["lam"], tree, ws,
                           k_req=x["k_req"])
    for wave in range(w.Bk):
        for rank in range(world):
            dt.sharded_build_gemm(cfg, wave, rank, x["block_logits"], x["markov_a"], Bm[rank], ws,
                                  gathered[rank * pb:(rank + 1) * pb])
        dt.sharded_build_frontier(cfg, wave, gathered, x["n_budget"], x["lam"], tree, ws,
                                  calib=x["calib"], k_req=x["k_req"])
    assert dt.read_status(ws) == 0
    return tree


@pytest.mark.parametrize("name,over,world", [
    ("tiny", {}, 2),
    ("tiny", dict(V=1000, r=32, Bk=5, k=3, N=20), 3),      # ragged last shard and tile
    ("tiny", dict(V=777, r=48, Bk=6, k=5, N=40, batch=3), 2),  # 64-column node tiles
    ("qwen3_4b", {}, 2),
    ("qwen3_4b", dict(batch=4, sigma_ab=0.35), 3),
])
def test_sharded_build_equals_oracle(name, over, world):
    w = make_workload(name, seed=2, temp=0.0, **over)
    tree = run_sharded(w, world)
    ref = run_build(w, temp=0.0)
    for b in range(w.batch):
        compare_tree(w, tree, b, 0.0, w.philox_seed)
        h, r = tree_to_host(tree, b), tree_to_host(ref, b)
        assert h["n"] == r["n"] and np.array_equal(h["tokens"], r["tokens"])


def test_sharded_budgets_lambda_calibration():
    w = make_workload("tiny", seed=3, batch=5, V=1536, N=12, k=3, temp=0.0)
    w.n_budget[:] = np.array([12, 1, 0, 7, 12], np.int32)
    w.k_req[:] = np.array([3, 3, 1, 2, 1], np.int32)
    w.lam[:] = np.array([0.0, 0.0, 0.0, 0.02, 1e-4], np.float32)
    w.calib = np.array([[0.5, -0.1], [1.5, 0.2], [1.0, 0.0], [0.8, -0.3]], np.float32)
    tree = run_sharded(w, 4)
    for b in range(w.batch):
        compare_tree(w, tree, b, 0.0, w.philox_seed)


def test_sharded_argument_checks():
    w = make_workload("tiny", seed=0)
    x = build_inputs(w)
    cfg = dt.shard_cfg(w.batch, w.Bk, w.V, w.r, w.k, w.Nmax, 2)
    ws = dt.workspace(dt.sharded_workspace_bytes(cfg))
    part = torch.empty(dt.sharded_partials_bytes(cfg), dtype=torch.uint8, device="cuda")
    with pytest.raises(_lib.DtreeError) as e:   # rank outside the world
        dt.sharded_build_gemm(cfg, 0, 2, x["block_logits"], x["markov_a"], x["markov_b"], ws, part)
    assert e.value.code == _lib.DT_EINVAL
    bad = dt.shard_cfg(w.batch, w.Bk, w.V, w.r, w.k, w.Nmax, 2, ncta=3)   # 2 tiles per shard
    with pytest.raises(_lib.DtreeError) as e:
        dt.sharded_build_begin(bad, x["root_token"], x["n_budget"], x["lam"],
                               dt.Tree.empty(w.batch, w.Nmax), ws)
    assert e.value.code == _lib.DT_EUNSUPPORTED
    with pytest.raises(_lib.DtreeError) as e:
        dt.sharded_build_gemm(cfg, 0, 0, x["block_logits"], x["markov_a"], x["markov_b"], ws,
                              part[8:])   # partials not 256-byte aligned
    assert e.value.code == _lib.DT_EINVAL
