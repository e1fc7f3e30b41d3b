"""Acceptance walk over a verified draft tree.

Sources:
  * TreeSpark article, introduction: draft-then-verify with an accept/reject
    rule that leaves the output distribution equal to the target's
    (Leviathan et al. 2023).
  * TreeSpark article, "lossless decoding" section: siblings sampled without
    replacement and residuals matched in recursive rejection keep the output
    exact at every temperature.
  * PCTree summary, "setup" paragraph: greedy verification.

Readings fixed here:
  * T = 0: follow the child whose token is the target argmax (ties to the
    lower token id); the bonus is that argmax at the node where it stops.
  * T > 0, at node u with p = softmax(t_u / T) and draft q = q_u, children in
    rank order (their sampling order): accept x iff U < p(x) / q(x); on
    rejection p <- max(p - q, 0) / sum (left unchanged if that sum is 0) and
    q <- q with x removed, renormalised.  With no child accepted, or at a
    leaf, the bonus is argmax_x p(x) / E_x with E_x = -log U'_x (an
    exponential race, i.e. a draw from p), ties to the lower id.
  * coins use Philox purpose 1 (counter word 1 = candidate node index), the
    race purpose 2 (counter word 1 = stop node + 1, root = 0).
"""
from __future__ import annotations

from typing import Callable, Optional

import numpy as np

from . import philox
from .markov_tree import Tree


def greedy_walk(tree: Tree, t_rows):
    """Greedy acceptance; t_rows[0] = root row, t_rows[i + 1] = node i."""
    path = []
    node = -1
    while True:
        a = int(np.argmax(t_rows[node + 1]))          # first maximum = lower id
        nxt = [c for c in tree.children(node) if tree.tokens[c] == a]
        if not nxt:
            return path, a
        node = int(nxt[0])
        path.append(node)


def softmax(x):
    x = np.asarray(x, np.float64)
    e = np.exp(x - x.max())
    return e / e.sum()


Coin = Callable[[int, float], bool]
Race = Callable[[int, np.ndarray], int]


def stochastic_walk(tree: Tree, t_rows, temp, seed=0, offset=0, request=0,
                    coin: Optional[Coin] = None, race: Optional[Race] = None,
                    q_rows=None, margins=None):
    """Recursive residual rejection with without-replacement siblings.

    ``q_rows`` maps a row (0 = root, i + 1 = node i) to its draft
    distribution; by default the tree's own expansions are used.  ``coin`` and
    ``race`` replace the Philox draws (exact-enumeration tests).
    """
    if q_rows is None:
        q_rows = {r: e.q for r, e in tree.expansions.items()}

    def philox_coin(node, ratio):
        u = float(philox.uniforms(seed, offset, philox.PURPOSE_COIN, request,
                                  node, 0, np.zeros(1, np.int64))[0])
        if margins is not None:
            margins.append(("coin", abs(u - ratio) / max(ratio, 1e-30), node))
        return u < ratio

    def philox_race(stop, p):
        V = p.size
        U = philox.uniforms(seed, offset, philox.PURPOSE_BONUS, request,
                            stop + 1, 0, np.arange(V))
        score = p / (-np.log(U))
        best = int(np.argmax(score))
        if margins is not None and V > 1:
            two = np.sort(score)[-2:]
            margins.append(("race", (two[1] - two[0]) / max(two[1], 1e-300), stop))
        return best

    coin = coin or philox_coin
    race = race or philox_race
    path = []
    node = -1
    while True:
        p = softmax(np.asarray(t_rows[node + 1], np.float64) / temp)
        accepted = None
        kids = tree.children(node)
        if kids.size:
            q = np.array(q_rows[node + 1], np.float64, copy=True)
            for c in kids:
                x = int(tree.tokens[c])
                if coin(int(c), float(p[x] / q[x])):
                    accepted = int(c)
                    break
                r = np.maximum(p - q, 0.0)
                z = r.sum()
                if z > 0:
                    p = r / z
                q[x] = 0.0
                q = q / q.sum()
        if accepted is None:
            return path, int(race(node, p))
        path.append(accepted)
        node = accepted


def emitted_tokens(tree: Tree, path, bonus):
    return [int(tree.tokens[i]) for i in path] + [int(bonus)]
