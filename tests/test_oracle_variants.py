"""Pins of the baseline tree variants (oracle/variants.py).

Each variant is checked against a plain restatement of its definition that
does not go through the conditioning override:
  * chain: a loop of argmax steps z = L[d] + A[c] . B^T;
  * marginal-ranked tree: the method on a Markov head whose A is all zeros;
  * Shared-Markov tree: the method with A = 0 on block logits that already
    hold the chain's Markov rows, L'[d] = L[d] + A[c_d] . B^T, which is the
    "one distribution per depth, reused by every sibling" definition;
plus invariants (same-depth nodes share their children; the rank-0 path of
the Shared-Markov tree is the greedy chain) and acceptance-length special
cases.  A planted mistake in the conditioning (using the parent instead of
the chain token, or a depth off by one) fails the Shared-Markov pin.
"""
import numpy as np
import pytest

from gen import make_workload, target_rows
from oracle import markov_tree, variants


def _small(seed, **over):
    c = dict(V=512, batch=2, Bk=5, k=3, N=12, r=16, sigma_ab=0.35, logit_dtype="f32",
             plant=("margin", 3.0, 1.0))
    c.update(over)
    w = make_workload("tiny", seed=seed, **c)
    return w, w.A.astype(np.float64), w.Bt.astype(np.float64)


def _argmax_chain(L, A, Bt, root, n):
    out, c = [], int(root)
    for d in range(n):
        z = L[d] + Bt @ A[c]
        c = int(np.argmax(z))  # first maximum = lower token id
        out.append(c)
    return out


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_greedy_chain_is_an_argmax_loop(seed):
    w, A, Bt = _small(seed)
    for b in range(w.batch):
        L = w.L[b].astype(np.float64)
        got = variants.greedy_chain(L, A, Bt, int(w.root[b]), w.Bk)
        assert list(got) == _argmax_chain(L, A, Bt, w.root[b], w.Bk)
        t = variants.variant_tree("chain", L, A, Bt, int(w.root[b]), w.k, w.Nmax)
        assert t.n == w.Bk and list(t.depths) == list(range(1, w.Bk + 1))
        assert list(t.tokens) == list(got)


def _same(a, b):
    assert a.n == b.n
    for f in ("tokens", "parents", "depths", "ranks"):
        assert np.array_equal(getattr(a, f), getattr(b, f)), f
    assert np.allclose(a.keys64, b.keys64, atol=1e-12, rtol=0)


@pytest.mark.parametrize("seed,temp", [(0, 0.0), (1, 0.0), (2, 0.8)])
def test_marginal_tree_is_the_method_without_a_markov_term(seed, temp):
    w, A, Bt = _small(seed)
    for b in range(w.batch):
        L = w.L[b].astype(np.float64)
        kw = dict(temp=temp, seed=5, request=b)
        got = variants.variant_tree("marginal", L, A, Bt, int(w.root[b]), w.k, w.Nmax, **kw)
        want = markov_tree.build_tree(L, np.zeros_like(A), Bt, int(w.root[b]), w.k, w.Nmax, **kw)
        _same(got, want)


@pytest.mark.parametrize("seed,temp,N", [(0, 0.0, 12), (1, 0.0, 3), (2, 0.7, 12), (3, 0.0, 40)])
def test_shared_markov_is_one_distribution_per_depth(seed, temp, N):
    w, A, Bt = _small(seed, N=N)
    for b in range(w.batch):
        L = w.L[b].astype(np.float64)
        root = int(w.root[b])
        chain = _argmax_chain(L, A, Bt, root, min(w.Bk, N))
        cond = [root] + chain
        Lp = np.array([L[d] + Bt @ A[cond[d]] if d < len(cond) else L[d] for d in range(w.Bk)])
        kw = dict(temp=temp, seed=9, request=b)
        got = variants.variant_tree("shared_markov", L, A, Bt, root, w.k, N, **kw)
        want = markov_tree.build_tree(Lp, np.zeros_like(A), Bt, root, w.k, N, **kw)
        _same(got, want)


def test_shared_markov_pin_catches_parent_conditioning():
    # negative control: the method itself (parent-conditioned) differs from the
    # Shared-Markov tree on these inputs, so the pin above can tell them apart
    w, A, Bt = _small(0)
    diff = 0
    for b in range(w.batch):
        L = w.L[b].astype(np.float64)
        s = variants.variant_tree("shared_markov", L, A, Bt, int(w.root[b]), w.k, w.Nmax)
        p = variants.variant_tree("pctree", L, A, Bt, int(w.root[b]), w.k, w.Nmax)
        diff += int(s.n != p.n or not np.array_equal(s.tokens, p.tokens))
    assert diff > 0


@pytest.mark.parametrize("variant", ["marginal", "shared_markov"])
def test_same_depth_nodes_share_children(variant):
    w, A, Bt = _small(4, N=30)
    for b in range(w.batch):
        L = w.L[b].astype(np.float64)
        t = variants.variant_tree(variant, L, A, Bt, int(w.root[b]), w.k, w.Nmax)
        by_depth = {}
        for row, e in t.expansions.items():
            by_depth.setdefault(e.depth, set()).add(tuple(e.children.tolist()))
        assert all(len(v) == 1 for v in by_depth.values())


def test_shared_markov_rank0_path_is_the_chain():
    w, A, Bt = _small(5, N=30)
    for b in range(w.batch):
        L = w.L[b].astype(np.float64)
        root = int(w.root[b])
        t = variants.variant_tree("shared_markov", L, A, Bt, root, w.k, w.Nmax)
        node, path = -1, []
        while True:
            kids = [c for c in t.children(node) if t.ranks[c] == 0]
            if not kids:
                break
            node = int(kids[0])
            path.append(int(t.tokens[node]))
        chain = _argmax_chain(L, A, Bt, root, w.Bk)
        assert path == chain[: len(path)] and len(path) == w.Bk


def test_acceptance_length_special_cases():
    w, A, Bt = _small(6)
    L = w.L[0].astype(np.float64)
    root = int(w.root[0])
    t = variants.variant_tree("chain", L, A, Bt, root, w.k, w.Nmax)
    V = w.V
    # target rows whose argmax is the chain's next token: all Bk accepted + bonus
    rows = np.zeros((t.n + 1, V))
    nxt = list(t.tokens) + [7]
    for i, tok in enumerate(nxt):
        rows[i, tok] = 1.0
    assert variants.acceptance_length(t, rows) == w.Bk + 1
    # target disagrees at depth 3: depths 1, 2 accepted, then the bonus
    rows[2] = 0.0
    rows[2, (nxt[2] + 1) % V] = 1.0
    assert variants.acceptance_length(t, rows) == 3
    # disagreement at the root: only the bonus token
    rows[0] = 0.0
    rows[0, (nxt[0] + 1) % V] = 1.0
    assert variants.acceptance_length(t, rows) == 1


def test_greedy_acceptance_is_the_longest_matching_path():
    # brute force over root-to-node paths: the greedy walk accepts the deepest
    # node whose every edge is the target argmax after its parent
    w, A, Bt = _small(7, N=30)
    for b in range(w.batch):
        L = w.L[b].astype(np.float64)
        t = variants.variant_tree("pctree", L, A, Bt, int(w.root[b]), w.k, w.Nmax)
        rows = target_rows(w, b, np.concatenate([[0], t.depths]),
                           np.concatenate([[w.root[b]], t.tokens])).astype(np.float64)
        am = rows.argmax(axis=1)
        best = 0
        for i in range(t.n):
            node, ok = i, True
            while node >= 0:
                par = int(t.parents[node])
                ok &= int(t.tokens[node]) == int(am[par + 1])
                node = par
            if ok:
                best = max(best, int(t.depths[i]))
        assert variants.acceptance_length(t, rows) == best + 1
