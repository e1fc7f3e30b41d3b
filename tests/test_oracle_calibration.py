"""Pins of the calibration fit (oracle/calibration.py).

  * logging: a hand-built tree and walk give exactly the expected triples;
  * consistency of the maximum-likelihood fit: outcomes drawn from a known
    (alpha*, beta*) are fitted back to it within a grid step, and outcomes
    drawn from the drafter's own probabilities give the identity (1, 0);
  * the likelihood at the chosen point is the maximum of a brute-force scan
    over a finer grid restricted to the same points, and flat likelihoods
    resolve to the smallest alpha, then the smallest beta;
  * a depth without data, or with fewer than min_samples edges, keeps the
    identity.
A planted sign error in the likelihood (log p for rejections) or a swapped
(alpha, beta) would miss the recovery pins.
"""
import numpy as np
import pytest

from oracle import calibration
from oracle.markov_tree import Tree

GRID = dict(a0=0.0, da=1 / 16, na=33, b0=-1.0, db=1 / 16, nb=25)   # alpha 0..2, beta -1..0.5


def _tree(parents, depths, keys):
    n = len(parents)
    return Tree(tokens=np.arange(n, dtype=np.int32), parents=np.asarray(parents, np.int32),
                depths=np.asarray(depths, np.int32), ranks=np.zeros(n, np.int32),
                keys=np.asarray(keys, np.float32), keys64=np.asarray(keys, np.float64),
                anc=np.zeros(n, np.uint64), expansions={}, margins=[])


def test_log_pairs_hand_built():
    # root -> 0, 1; 0 -> 2, 3; 1 -> 4; 2 -> 5.  The walk accepts 0 then stops.
    t = _tree([-1, -1, 0, 0, 1, 2], [1, 1, 2, 2, 2, 3],
              [-0.25, -1.5, -0.75, -2.0, -1.75, -1.0])
    depth, ell, y = calibration.log_pairs(t, [0])
    assert depth.tolist() == [1, 1, 2, 2, -1, -1]
    assert y[:4].tolist() == [1, 0, 0, 0]
    assert ell[:4].tolist() == [-0.25, -1.5, -0.5, -1.75]


def _draw(g, n, alpha, beta):
    ell = g.uniform(-5.0, 0.0, n).astype(np.float32)
    p = np.exp(np.minimum(0.0, alpha * ell.astype(np.float64) + beta))
    return ell, (g.random(n) < p).astype(np.int8)


@pytest.mark.parametrize("alpha,beta", [(0.75, -0.25), (1.5, 0.0), (0.5, -0.5)])
def test_fit_recovers_the_generating_calibration(alpha, beta):
    g = np.random.default_rng(int(alpha * 100 + beta * 10) + 7)
    ell, y = _draw(g, 60000, alpha, beta)
    depth = np.full(ell.size, 2, np.int32)
    cal, _ = calibration.fit(depth, ell, y, 3, **GRID)
    assert abs(cal[1, 0] - alpha) <= 2 * GRID["da"] + 1e-12
    assert abs(cal[1, 1] - beta) <= 2 * GRID["db"] + 1e-12
    # depths 1 and 3 have no data: identity
    assert cal[0].tolist() == [1.0, 0.0] and cal[2].tolist() == [1.0, 0.0]


def test_drafter_probabilities_fit_the_identity():
    g = np.random.default_rng(3)
    ell, y = _draw(g, 60000, 1.0, 0.0)
    cal, _ = calibration.fit(np.ones(ell.size, np.int32), ell, y, 1, **GRID)
    assert abs(cal[0, 0] - 1.0) <= 2 * GRID["da"] and abs(cal[0, 1]) <= 2 * GRID["db"]


def test_fit_is_the_grid_maximum_and_breaks_ties_low():
    g = np.random.default_rng(11)
    ell, y = _draw(g, 500, 0.8, -0.2)
    depth = np.ones(ell.size, np.int32)
    cal, ll = calibration.fit(depth, ell, y, 1, **GRID)
    scan = [(calibration.log_likelihood(GRID["a0"] + i * GRID["da"], GRID["b0"] + j * GRID["db"],
                                        ell, y), i, j)
            for i in range(GRID["na"]) for j in range(GRID["nb"])]
    top = max(s[0] for s in scan)
    assert ll[0] == top
    first = min((i, j) for s, i, j in scan if s == top)
    assert cal[0].tolist() == [GRID["a0"] + first[0] * GRID["da"], GRID["b0"] + first[1] * GRID["db"]]
    # every outcome accepted with l in [-1, 0]: the likelihood is 0 wherever
    # alpha * l + beta >= 0 for all l, first reached at alpha 0, beta 0
    ell1 = np.linspace(-1, 0, 50).astype(np.float32)
    cal1, ll1 = calibration.fit(np.ones(50, np.int32), ell1, np.ones(50, np.int8), 1, **GRID)
    assert ll1[0] == 0.0 and cal1[0].tolist() == [0.0, 0.0]


def test_min_samples_keeps_the_identity():
    g = np.random.default_rng(21)
    ell, y = _draw(g, 2000, 0.7, -0.3)
    depth = np.concatenate([np.ones(1990, np.int32), np.full(10, 2, np.int32)])
    full, _ = calibration.fit(depth, ell, y, 2, **GRID)
    cut, ll = calibration.fit(depth, ell, y, 2, **GRID, min_samples=11)
    assert np.array_equal(cut[0], full[0])            # 1990 edges: fitted as before
    assert cut[1].tolist() == [1.0, 0.0] and np.isnan(ll[1])
    same, _ = calibration.fit(depth, ell, y, 2, **GRID, min_samples=10)
    assert np.array_equal(same, full)
