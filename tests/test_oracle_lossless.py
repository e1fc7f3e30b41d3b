"""Exact losslessness of the oracle's stochastic round, by enumeration.

TreeSpark article, "lossless decoding" section: sampling siblings without
replacement and matching residuals in recursive rejection keep the output
distribution equal to the target's at every temperature.

The oracle's own build and walk run with every random decision replaced by
a scripted choice: the ordered sibling draw (Plackett-Luce probabilities),
each acceptance coin (min(1, p/q) and its complement) and the bonus draw
(the residual's probabilities).  Enumerating every decision sequence gives the
exact law of the emitted tokens, which must equal the target's conditional
distributions to 1e-12.  A deliberately wrong key rule (siblings ranked by the
sampled token's own probability) must fail the same check.
"""
import itertools
import math

import numpy as np
import pytest
import scipy.stats

from gen import make_workload
from oracle import accept, markov_tree


class Script:
    def __init__(self, prefix):
        self.prefix = list(prefix)
        self.taken = []
        self.options = []       # per decision: indices with non-zero probability
        self.prob = 1.0

    def choose(self, probs):
        nz = [i for i, p in enumerate(probs) if p > 0]
        pos = len(self.taken)
        i = self.prefix[pos] if pos < len(self.prefix) else nz[0]
        self.taken.append(i)
        self.options.append(nz)
        self.prob *= probs[i]
        return i


def enumerate_law(run):
    out = []
    stack = [[]]
    while stack:
        prefix = stack.pop()
        sc = Script(prefix)
        res = run(sc)
        out.append((res, sc.prob))
        for pos in range(len(prefix), len(sc.taken)):
            for alt in sc.options[pos]:
                if alt != sc.taken[pos]:
                    stack.append(sc.taken[:pos] + [alt])
    return out


def pl_prob(q, order):
    p, rest = 1.0, 1.0
    for x in order:
        p *= q[x] / rest
        rest -= q[x]
    return p


def make_run(L, A, Bt, root, k, N, temp, lam, tgt, key_mode="order_stat", calib=None):
    V = L.shape[1]

    def run(sc):
        def sampler(ranks, s, lse, kk):
            q = np.exp(s - lse)
            orders = list(itertools.permutations(range(V), kk))
            i = sc.choose([pl_prob(q, o) for o in orders])
            return np.array(orders[i])

        t = markov_tree.build_tree(L, A, Bt, root, k, N, temp=temp, lam=lam,
                                   calib=calib, sampler=sampler, key_mode=key_mode)
        rows = [tgt[(0, root)]] + [tgt[(int(t.depths[i]), int(t.tokens[i]))] for i in range(t.n)]

        def coin(node, ratio):
            a = min(1.0, ratio)
            return sc.choose([a, 1.0 - a]) == 0

        def race(node, p):
            return sc.choose(list(p))

        path, bonus = accept.stochastic_walk(t, np.array(rows), temp, coin=coin, race=race)
        return tuple(int(t.tokens[i]) for i in path), int(bonus)

    return run


def max_law_error(law, tgt, root, temp):
    """max |P(next | accepted context) - p_target(next | context)| over contexts."""
    cond, tot = {}, {}
    for (acc, bonus), pr in law:
        for i in range(len(acc) + 1):
            ctx = acc[:i]
            nxt = acc[i] if i < len(acc) else bonus
            cond.setdefault(ctx, {}).setdefault(nxt, 0.0)
            cond[ctx][nxt] += pr
            tot[ctx] = tot.get(ctx, 0.0) + pr
    total = sum(pr for _, pr in law)
    assert abs(total - 1.0) < 1e-12
    err = 0.0
    for ctx, dist in cond.items():
        if tot[ctx] < 1e-9:
            continue
        key = (len(ctx), ctx[-1] if ctx else root)
        p = accept.softmax(np.asarray(tgt[key]) / temp)
        for y in range(p.size):
            err = max(err, abs(dist.get(y, 0.0) / tot[ctx] - p[y]))
    return err


def _case(V, Bk, seed, r=2):
    w = make_workload("tiny", seed=seed, V=V, Bk=Bk, r=r)
    g = np.random.default_rng(seed + 100)
    tgt = {(d, x): 2.0 * g.standard_normal(V) for d in range(Bk + 1) for x in range(V)}
    return w.L[0].astype(np.float64) * 0.5, w.A, w.Bt, int(w.root[0]), tgt


@pytest.mark.parametrize("V,k,Bk,N,temp,lam", [
    (3, 2, 2, 3, 0.5, 0.0),
    (3, 2, 2, 3, 1.0, 0.0),
    (3, 2, 2, 4, 2.0, 0.0),
    (3, 3, 2, 4, 1.0, 0.05),
    (4, 2, 2, 3, 1.0, 0.0),
])
def test_round_is_lossless(V, k, Bk, N, temp, lam):
    L, A, Bt, root, tgt = _case(V, Bk, seed=V * 10 + N)
    law = enumerate_law(make_run(L, A, Bt, root, k, N, temp, lam, tgt))
    assert max_law_error(law, tgt, root, temp) < 1e-12


def test_lossless_with_calibration():
    L, A, Bt, root, tgt = _case(3, 2, seed=77)
    calib = np.array([[0.5, -0.1], [2.0, 0.3]], np.float32)
    law = enumerate_law(make_run(L, A, Bt, root, 2, 3, 1.0, 0.0, tgt, calib=calib))
    assert max_law_error(law, tgt, root, 1.0) < 1e-12


def _negative_control_inputs():
    V = 3
    L = np.log(np.array([[0.6, 0.3, 0.1]]))        # Bk = 1: root children only
    A = np.zeros((V, 2))
    Bt = np.zeros((V, 2))
    tgt = {(0, 0): np.zeros(V), (1, 0): np.zeros(V), (1, 1): np.zeros(V), (1, 2): np.zeros(V)}
    return L, A, Bt, 0, tgt


def test_order_statistic_keys_pass_own_q_keys_fail():
    L, A, Bt, root, tgt = _negative_control_inputs()
    good = enumerate_law(make_run(L, A, Bt, root, 2, 2, 1.0, 0.2, tgt))
    assert max_law_error(good, tgt, root, 1.0) < 1e-12
    bad = enumerate_law(make_run(L, A, Bt, root, 2, 2, 1.0, 0.2, tgt, key_mode="own_q"))
    assert max_law_error(bad, tgt, root, 1.0) > 1e-3


def test_two_token_counter_example_closed_form():
    """V={a,b}, q=(.7,.3), p=(.5,.5): keeping a sibling only when q(x) >= .5 gives P(a)=.65."""
    L = np.log(np.array([[0.7, 0.3]]))
    A, Bt = np.zeros((2, 1)), np.zeros((2, 1))
    tgt = {(0, 0): np.zeros(2), (1, 0): np.zeros(2), (1, 1): np.zeros(2)}
    bad = enumerate_law(make_run(L, A, Bt, 0, 1, 1, 1.0, 0.5, tgt, key_mode="own_q"))
    pa = sum(pr for (acc, b), pr in bad if (acc[0] if acc else b) == 0)
    assert abs(pa - 0.65) < 1e-12
    good = enumerate_law(make_run(L, A, Bt, 0, 1, 1, 1.0, 0.5, tgt))
    pa = sum(pr for (acc, b), pr in good if (acc[0] if acc else b) == 0)
    assert abs(pa - 0.5) < 1e-12


@pytest.mark.parametrize("temp", [0.6, 1.0, 2.0])
def test_philox_round_chi_square(temp):
    """Monte-Carlo with the real Philox draws on the V=512 toy round."""
    from gen import target_rows
    w = make_workload("tiny", seed=21, temp=temp)
    R = 1500
    rows_cache = {}

    def row(d, x):
        if (d, x) not in rows_cache:
            rows_cache[(d, x)] = target_rows(w, 0, np.array([d]), np.array([x]))[0]
        return rows_cache[(d, x)]

    first = np.zeros(w.V)
    for off in range(R):
        t = markov_tree.build_tree(w.L[0], w.A, w.Bt, w.root[0], w.k, w.Nmax, temp=temp,
                                   seed=5, offset=off)
        rows = np.stack([row(0, int(w.root[0]))] +
                        [row(int(t.depths[i]), int(t.tokens[i])) for i in range(t.n)])
        path, bonus = accept.stochastic_walk(t, rows, temp, seed=5, offset=off)
        first[accept.emitted_tokens(t, path, bonus)[0]] += 1
    p = accept.softmax(row(0, int(w.root[0])) / temp)
    exp_ = R * p
    big = exp_ >= 5
    obs = np.append(first[big], first[~big].sum())
    ex = np.append(exp_[big], exp_[~big].sum())
    if ex[-1] == 0:
        obs, ex = obs[:-1], ex[:-1]
    assert scipy.stats.chisquare(obs, ex * obs.sum() / ex.sum()).pvalue > 0.01
