"""GPU parity of dt_tree_load_budget against the oracle (oracle/load_policy.py).

Keys and node counts are the oracle's (random sorted batches with planted
ties, and the fp32 keys of oracle-built trees); the kept node counts must be
identical for every capacity of a sweep.  An end-to-end case cuts trees the
library built itself, after checking that no cut falls on a near-tie.
"""
import numpy as np
import pytest
import torch

from gen import make_workload
from oracle import load_policy, markov_tree

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import draft_tree_construction_markov_b200 as dt
    from draft_tree_construction_markov_b200 import _lib
    from tests.gpu_util import dev, run_build


def _random_batch(g, batch, nmax, tie_every=0):
    n = g.integers(0, nmax + 1, batch)
    keys = np.zeros((batch, nmax), np.float32)
    for b in range(batch):
        k = np.sort(-np.abs(g.normal(0, 3, n[b])))[::-1].astype(np.float32)
        if tie_every and n[b] > 1:
            k[1::tie_every] = k[0::tie_every][: len(k[1::tie_every])]
            k = np.sort(k)[::-1]
        keys[b, : n[b]] = k
    return keys, n


def _gpu_budget(keys, n, plen, cap, unit):
    batch, nmax = keys.shape
    tree = dt.Tree.empty(batch, nmax)
    tree.keys.copy_(torch.from_numpy(keys))
    tree.n_nodes.copy_(torch.from_numpy(np.asarray(n, np.int32)))
    keep = torch.full((batch,), -1, dtype=torch.int32, device="cuda")
    ws = dt.workspace(dt.load_budget_workspace_bytes())
    dt.tree_load_budget(tree, cap, ws, prefix_len=None if plen is None else dev(plen.astype(np.int32)),
                        prefix_unit=unit, n_keep=keep)
    assert dt.read_status(ws) == 0
    out = tree.n_nodes.cpu().numpy()
    assert np.array_equal(out, keep.cpu().numpy())
    return out


@pytest.mark.parametrize("batch,nmax,tie,unit", [(1, 8, 0, 0), (5, 12, 2, 1000), (37, 32, 3, 512),
                                                 (64, 32, 0, 1024), (200, 64, 4, 0),
                                                 (1024, 64, 2, 700)])
def test_budget_matches_oracle_over_a_capacity_sweep(batch, nmax, tie, unit):
    g = np.random.default_rng(batch * 7 + nmax)
    keys, n = _random_batch(g, batch, nmax, tie)
    plen = g.integers(0, 8192, batch)
    w = load_policy.node_cost(plen, unit)
    total = int((n * w).sum())
    caps = sorted(set([0, 1, 2, total - 1, total, total + 5] +
                      [int(x) for x in g.integers(0, total + 1, 12)]))
    for cap in caps:
        if cap < 0:
            continue
        want = load_policy.load_budget(keys, n, plen, cap, unit)
        got = _gpu_budget(keys, n, plen, cap, unit)
        assert np.array_equal(got, want), f"capacity {cap}"


def test_budget_on_oracle_trees():
    w = make_workload("tiny", seed=4, batch=6, N=16, k=3, sigma_ab=0.35)
    trees = [markov_tree.build_tree(w.L[b], w.A, w.Bt, int(w.root[b]), w.k, w.Nmax)
             for b in range(w.batch)]
    keys = np.zeros((w.batch, w.Nmax), np.float32)
    n = np.array([t.n for t in trees])
    for b, t in enumerate(trees):
        keys[b, : t.n] = t.keys
    plen = np.array([100, 2000, 700, 4000, 50, 9000])
    for cap in range(0, int((n * load_policy.node_cost(plen, 1024)).sum()) + 2, 3):
        assert np.array_equal(_gpu_budget(keys, n, plen, cap, 1024),
                              load_policy.load_budget(keys, n, plen, cap, 1024))


def test_budget_end_to_end_on_built_trees():
    w = make_workload("tiny", seed=5, batch=8, N=16, k=3, sigma_ab=0.35)
    tree = run_build(w, temp=0.0)
    n = tree.n_nodes.cpu().numpy()
    keys = tree.keys.cpu().numpy()
    otrees = [markov_tree.build_tree(w.L[b], w.A, w.Bt, int(w.root[b]), w.k, w.Nmax)
              for b in range(w.batch)]
    okeys = np.zeros_like(keys)
    for b, t in enumerate(otrees):
        assert t.n == n[b]
        okeys[b, : t.n] = t.keys
    cap = int(n.sum()) // 2
    want = load_policy.load_budget(okeys, n, None, cap, 0)
    # the cut must not fall on a near-tie of the oracle's keys
    flat = sorted(float(okeys[b, i]) for b in range(w.batch) for i in range(n[b]))[::-1]
    c = int(want.sum())
    assert 0 < c < len(flat) and flat[c - 1] - flat[c] > 1e-4
    ws = dt.workspace(dt.load_budget_workspace_bytes())
    dt.tree_load_budget(tree, cap, ws)
    assert dt.read_status(ws) == 0
    assert np.array_equal(tree.n_nodes.cpu().numpy(), want)


def test_budget_device_and_host_checks():
    tree = dt.Tree.empty(3, 8)
    tree.n_nodes.copy_(torch.tensor([2, 9, 1], dtype=torch.int32))
    ws = dt.workspace(dt.load_budget_workspace_bytes())
    dt.tree_load_budget(tree, 100, ws)
    assert dt.read_status(ws) == _lib.DT_EDEVICE
    with pytest.raises(_lib.DtreeError) as e:
        dt.tree_load_budget(tree, -1, ws)
    assert e.value.code == _lib.DT_EINVAL
    with pytest.raises(_lib.DtreeError) as e:
        dt.tree_load_budget(tree, 5, ws[:16])
    assert e.value.code == _lib.DT_EWORKSPACE
    big = dt.Tree.empty(1025, 4)
    with pytest.raises(_lib.DtreeError) as e:
        dt.tree_load_budget(big, 5, ws)
    assert e.value.code == _lib.DT_EUNSUPPORTED
