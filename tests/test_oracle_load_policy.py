"""Pins of the load-adaptive budget (oracle/load_policy.py).

The definition is "the longest survival-ordered prefix that fits the
capacity".  It is pinned against what it must achieve rather than retyped:
with unit costs the kept set maximises the batch's total survival (expected
accepted nodes) over every choice of per-request prefixes within the budget,
found by brute force; with any costs it spends no more than the capacity,
grows monotonically with it, and keeps ancestor-closed subtrees of real
trees.  A planted mistake (keys taken in ascending order, or ties to the
higher request) breaks the optimality or ordering pins.
"""
import itertools
import math

import numpy as np
import pytest

from gen import make_workload
from oracle import load_policy, markov_tree


def _random_batch(g, batch, nmax, tie_every=0):
    n = g.integers(0, nmax + 1, batch)
    keys = np.full((batch, nmax), np.nan, np.float32)
    for b in range(batch):
        k = np.sort(-np.abs(g.normal(0, 2, n[b])))[::-1].astype(np.float32)
        if tie_every and n[b] > 1:
            k[1::tie_every] = k[0::tie_every][: len(k[1::tie_every])]
            k = np.sort(k)[::-1]
        keys[b, : n[b]] = k
    return keys, n


def test_node_cost():
    assert load_policy.node_cost([0, 1023, 1024, 5000], 1024).tolist() == [1, 1, 2, 5]
    assert load_policy.node_cost([0, 9999], 0).tolist() == [1, 1]


@pytest.mark.parametrize("seed", range(6))
def test_unit_cost_maximises_total_survival(seed):
    g = np.random.default_rng(seed)
    keys, n = _random_batch(g, 3, 5)
    for cap in range(0, int(n.sum()) + 2):
        keep = load_policy.load_budget(keys, n, np.zeros(3, np.int64), cap, 0)
        best = -1.0
        for lens in itertools.product(*[range(int(x) + 1) for x in n]):
            if sum(lens) > cap:
                continue
            s = sum(math.exp(float(keys[b, i])) for b in range(3) for i in range(lens[b]))
            best = max(best, s)
        got = sum(math.exp(float(keys[b, i])) for b in range(3) for i in range(int(keep[b])))
        assert abs(got - best) < 1e-12 * max(1.0, best)
        assert keep.sum() == min(cap, n.sum())


def test_capacity_extremes_and_ties():
    g = np.random.default_rng(7)
    keys, n = _random_batch(g, 5, 8, tie_every=2)
    P = np.array([0, 500, 1500, 3000, 40], np.int64)
    w = load_policy.node_cost(P, 1000)
    total = int((n * w).sum())
    assert np.array_equal(load_policy.load_budget(keys, n, P, total, 1000), n)
    assert np.array_equal(load_policy.load_budget(keys, n, P, 10 ** 9, 1000), n)
    assert load_policy.load_budget(keys, n, P, 0, 1000).sum() == 0
    # equal keys across requests go to the lower request first
    k2 = np.array([[-1.0, -2.0], [-1.0, -2.0]], np.float32)
    assert load_policy.load_budget(k2, [2, 2], [0, 0], 1, 0).tolist() == [1, 0]
    assert load_policy.load_budget(k2, [2, 2], [0, 0], 3, 0).tolist() == [2, 1]


@pytest.mark.parametrize("seed", range(4))
def test_costs_respected_and_monotone(seed):
    g = np.random.default_rng(100 + seed)
    keys, n = _random_batch(g, 7, 10, tie_every=3)
    P = g.integers(0, 5000, 7)
    w = load_policy.node_cost(P, 1024)
    prev = np.zeros(7, np.int64)
    for cap in range(0, int((n * w).sum()) + 3):
        keep = load_policy.load_budget(keys, n, P, cap, 1024)
        assert (keep >= 0).all() and (keep <= n).all()
        assert int((keep * w).sum()) <= cap
        assert (keep >= prev).all()
        prev = keep
        # maximal: the best excluded node (in survival order) does not fit
        rest = [(-float(keys[b, keep[b]]), b) for b in range(7) if keep[b] < n[b]]
        if rest:
            _, b = min(rest)
            assert int((keep * w).sum()) + int(w[b]) > cap


def test_kept_nodes_form_subtrees_of_real_trees():
    w = make_workload("tiny", seed=2, batch=4, N=12, k=3)
    trees = [markov_tree.build_tree(w.L[b], w.A, w.Bt, int(w.root[b]), w.k, w.Nmax)
             for b in range(w.batch)]
    keys = np.zeros((w.batch, w.Nmax), np.float32)
    n = np.array([t.n for t in trees])
    for b, t in enumerate(trees):
        keys[b, : t.n] = t.keys
    P = np.array([100, 2000, 700, 4000])
    for cap in (0, 3, 9, 20, 40, 200):
        keep = load_policy.load_budget(keys, n, P, cap, 1024)
        for b, t in enumerate(trees):
            kept = set(range(int(keep[b])))
            assert all(int(t.parents[i]) in kept | {-1} for i in kept)
