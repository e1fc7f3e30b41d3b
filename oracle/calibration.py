"""Calibration of the edge-acceptance estimate from logged verification
outcomes.

Test infrastructure: the plain CPU definitions the library's dt_calib_log
and dt_calib_fit are checked against; nothing on the product path imports
them.

Sources:
  * TreeSpark article, "core idea": the Markov head's parent-conditioned
    probability is calibrated into an estimate of the edge's acceptance, and
    path survival (the product of those estimates) drives the tree.  The
    pages name calibration but give neither its form nor how it is fitted.

Readings fixed here:
  * the form is the one the tree build uses: for a child at depth d with
    drafter log-probability l (the order statistic of its rank),
    c_d(l) = min(0, alpha_d * l + beta_d), estimate exp(c_d(l)), alpha_d >= 0;
  * logged data: every round verified greedily on a tree built with the
    identity calibration (1, 0) yields, for every child of a node the walk
    reached (the root and each accepted node), the triple (depth, l, y) with
    l = key(child) - key(parent) in fp32 (exactly the child's log-probability
    up to that one rounding) and y = 1 iff the walk accepted the child;
  * fit: per depth, the grid point (alpha_i = a0 + i*da, beta_j = b0 + j*db)
    with the largest Bernoulli log-likelihood
        sum_y=1 c(l) + sum_y=0 log(1 - exp(c(l)))
    (ties to the smaller i, then the smaller j); a depth with fewer than
    min_samples logged edges (at least one) keeps the identity (1, 0): a
    handful of edges at a deep level would otherwise fit an estimate of 1.
"""
from __future__ import annotations

import numpy as np


def log_pairs(tree, path):
    """(depth, l, y) for every child of a reached node; -1 depth = not logged.

    tree: oracle Tree (fp32 keys in pop order); path: accepted node indices.
    Returns arrays of length tree.n in node order.
    """
    n = tree.n
    reached = set(int(i) for i in path)
    depth = np.full(n, -1, np.int32)
    ell = np.zeros(n, np.float32)
    y = np.zeros(n, np.int8)
    keys = tree.keys.astype(np.float32)
    for i in range(n):
        p = int(tree.parents[i])
        if p >= 0 and p not in reached:
            continue
        kp = np.float32(0.0) if p < 0 else keys[p]
        depth[i] = tree.depths[i]
        ell[i] = np.float32(keys[i] - kp)
        y[i] = 1 if i in reached else 0
    return depth, ell, y


def log_likelihood(alpha, beta, ell, y):
    """Bernoulli log-likelihood of outcomes y under exp(min(0, alpha*l + beta))."""
    x = np.minimum(0.0, alpha * np.asarray(ell, np.float64) + beta)
    y = np.asarray(y, bool)
    with np.errstate(divide="ignore"):
        return float(x[y].sum() + np.log1p(-np.exp(x[~y])).sum())


def fit(depth, ell, y, Bk, a0, da, na, b0, db, nb, min_samples=1):
    """(Bk, 2) fitted (alpha, beta) per child depth 1..Bk, and the (Bk,)
    maximal log-likelihoods (nan where a depth keeps the identity)."""
    depth = np.asarray(depth)
    out = np.tile(np.array([1.0, 0.0]), (Bk, 1))
    best_ll = np.full(Bk, np.nan)
    for d in range(1, Bk + 1):
        m = depth == d
        if m.sum() < max(1, min_samples):
            continue
        best = None
        for i in range(na):
            a = a0 + i * da
            for j in range(nb):
                b = b0 + j * db
                ll = log_likelihood(a, b, np.asarray(ell)[m], np.asarray(y)[m])
                if best is None or ll > best[0]:
                    best = (ll, a, b)
        out[d - 1] = best[1:]
        best_ll[d - 1] = best[0]
    return out, best_ll
