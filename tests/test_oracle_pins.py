"""Pins of the CPU oracle against facts fixed outside the oracle itself.

* Philox4x32-10 known answers (Random123 publication).
* k = 1 collapses the tree to the greedy chain (PCTree summary, "k=4, N=32"
  paragraph).
* Top-N by path probability is what best-first selects (brute force over
  every node of a tiny k-ary tree, and over the full vocabulary).
* Library routines: log-sum-exp (scipy), attention (torch SDPA).
* Special cases of acceptance: target equal to draft.
"""
import itertools
import math
import os

import numpy as np
import pytest
import scipy.special
import torch

from gen import make_workload, target_rows
from oracle import accept, markov_tree, philox, verify_attn

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def test_philox_known_answers():
    rows = [l.split() for l in open(os.path.join(GOLDEN, "philox4x32_10_kat.txt"))
            if l.strip() and not l.startswith("#")]
    assert len(rows) == 3
    for r in rows:
        v = [int(x, 16) for x in r]
        out = philox.philox4x32_10(*v[:6])
        assert [int(o) for o in out] == v[6:]


def test_uniforms_open_interval_and_lanes():
    xs = np.arange(4096)
    u = philox.uniforms(7, 3, 0, 5, 11, 13, xs)
    assert np.all(u > 0) and np.all(u < 1)
    # the four tokens sharing a counter read its four output words
    words = philox.philox4x32_10((0 >> 2) | (5 << 18), 11, 13, 3, 7, 0)
    assert np.allclose(u[:4], [philox.uniform_from_word(w) for w in words])
    assert abs(u.mean() - 0.5) < 0.02


def test_lse_matches_library():
    g = np.random.default_rng(1)
    for T in (0.0, 0.6, 1.0, 2.0):
        z = 5 * g.standard_normal(1000)
        s, lse = markov_tree.scaled_logits(z, T)
        assert np.allclose(s, z / (T if T > 0 else 1.0))
        assert abs(lse - scipy.special.logsumexp(z / (T if T > 0 else 1.0))) < 1e-12


def _z_fp32(w, d, tok, b=0):
    """Drafter logits computed by torch fp32 (exact on the dyadic grid)."""
    A = torch.from_numpy(w.A[tok])
    B = torch.from_numpy(w.Bt)
    return (torch.from_numpy(w.L[b, d]) + B @ A).numpy().astype(np.float64)


@pytest.mark.parametrize("name,over", [("tiny", {}), ("qwen3_4b", {"V": 4096})])
def test_k1_is_greedy_chain(name, over):
    w = make_workload(name, seed=3, **over)
    t = markov_tree.build_tree(w.L[0], w.A, w.Bt, w.root[0], k=1, N=w.Bk + 3)
    chain, tok = [], int(w.root[0])
    for d in range(w.Bk):
        tok = int(np.argmax(_z_fp32(w, d, tok)))
        chain.append(tok)
    assert t.tokens.tolist() == chain
    assert t.parents.tolist() == list(range(-1, w.Bk - 1))
    assert t.depths.tolist() == list(range(1, w.Bk + 1))
    assert t.ranks.tolist() == [0] * w.Bk


def _brute_force_nodes(w, k, Bk):
    """Every node of the k-ary candidate tree with its path log-probability."""
    nodes = []  # (logp, depth, path_ranks, token)

    def rec(tok, d, logp, ranks):
        if d == Bk:
            return
        z = _z_fp32(w, d, tok)
        lq = z - scipy.special.logsumexp(z)
        order = np.lexsort((np.arange(z.size), -z))[:k]
        for j, x in enumerate(order):
            nodes.append((logp + lq[x], d + 1, ranks + (j,), int(x)))
            rec(int(x), d + 1, logp + lq[x], ranks + (j,))

    rec(int(w.root[0]), 0, 0.0, ())
    return nodes


@pytest.mark.parametrize("V,k,Bk,N", [(512, 2, 4, 8), (512, 2, 4, 30), (6, 6, 3, 40), (6, 6, 3, 258)])
def test_best_first_equals_brute_force_top_n(V, k, Bk, N):
    w = make_workload("tiny", seed=5, V=V, Bk=Bk)
    t = markov_tree.build_tree(w.L[0], w.A, w.Bt, w.root[0], k=k, N=min(N, 64))
    nodes = _brute_force_nodes(w, k, Bk)
    assert len(nodes) == sum(k ** i for i in range(1, Bk + 1))
    nodes.sort(key=lambda n: (-n[0], n[1]))
    want = {(n[2], n[3]) for n in nodes[:min(N, 64)]}
    got = {(t.path_ranks(i), int(t.tokens[i])) for i in range(t.n)}
    assert got == want
    # keys are the path log-probabilities (identity calibration)
    lp = {n[2]: n[0] for n in nodes}
    for i in range(t.n):
        assert abs(t.keys64[i] - lp[t.path_ranks(i)]) < 1e-9


def test_tree_invariants_and_order():
    w = make_workload("qwen3_4b", seed=1, V=2048)
    t = markov_tree.build_tree(w.L[0], w.A, w.Bt, w.root[0], k=4, N=32)
    assert t.n == 32
    for i in range(t.n):
        p = t.parents[i]
        assert p < i                                   # topological pop order
        assert t.depths[i] == (1 if p < 0 else t.depths[p] + 1)
        assert t.anc[i] == ((0 if p < 0 else int(t.anc[p])) | (1 << i))
        if p >= 0:
            assert t.keys64[i] <= t.keys64[p]
    assert np.all(np.diff(t.keys64) <= 0)              # pop order is sorted
    # siblings included form a rank prefix
    for u in range(-1, t.n):
        r = t.ranks[t.children(u)].tolist()
        assert r == list(range(len(r)))


def test_lambda_stops_and_calibration_monotone():
    w = make_workload("qwen3_4b", seed=2, V=2048)
    full = markov_tree.build_tree(w.L[0], w.A, w.Bt, w.root[0], k=4, N=64)
    lam = 0.05
    t = markov_tree.build_tree(w.L[0], w.A, w.Bt, w.root[0], k=4, N=64, lam=lam)
    want = [i for i in range(full.n) if np.float32(full.keys64[i]) >= np.float32(math.log(lam))]
    assert t.n == len(want) and t.tokens.tolist() == full.tokens[:t.n].tolist()
    calib = np.tile(np.array([[0.5, -0.25]], np.float32), (w.Bk, 1))
    tc = markov_tree.build_tree(w.L[0], w.A, w.Bt, w.root[0], k=4, N=16, calib=calib)
    for i in range(tc.n):
        p = tc.parents[i]
        e = tc.expansions[p + 1]
        lq = float(e.logq[tc.ranks[i]])
        step = min(0.0, 0.5 * lq - 0.25)
        base = 0.0 if p < 0 else tc.keys64[p]
        assert abs(tc.keys64[i] - (base + step)) < 1e-12


def test_single_node_budget():
    w = make_workload("tiny", seed=4)
    t = markov_tree.build_tree(w.L[0], w.A, w.Bt, w.root[0], k=2, N=1)
    assert t.n == 1 and t.tokens[0] == int(np.argmax(_z_fp32(w, 0, int(w.root[0]))))


def _rows_for_tree(w, t, b=0):
    d = np.concatenate([[0], t.depths]).astype(np.int64)
    prev = np.concatenate([[w.root[b]], t.tokens]).astype(np.int64)
    return target_rows(w, b, d, prev)


def test_greedy_accept_target_equals_draft_takes_argmax_chain():
    w = make_workload("tiny", seed=6)
    t = markov_tree.build_tree(w.L[0], w.A, w.Bt, w.root[0], k=2, N=8)
    rows = np.stack([_z_fp32(w, 0, int(w.root[0]))] +
                    [_z_fp32(w, min(int(t.depths[i]), w.Bk - 1), int(t.tokens[i])) for i in range(t.n)])
    path, bonus = accept.greedy_walk(t, rows)
    # the accepted path follows rank-0 children while they exist
    node, want = -1, []
    while True:
        kids = t.children(node)
        if kids.size == 0 or t.ranks[kids[0]] != 0:
            break
        node = int(kids[0])
        want.append(node)
    assert path == want
    assert bonus == int(np.argmax(rows[path[-1] + 1 if path else 0]))


def test_stochastic_accept_target_equals_draft_accepts_first_siblings():
    w = make_workload("tiny", seed=7, temp=1.0)
    t = markov_tree.build_tree(w.L[0], w.A, w.Bt, w.root[0], k=2, N=8, temp=1.0, seed=9)
    rows = np.zeros((t.n + 1, w.V))
    rows[0] = markov_tree.node_logits(w.L[0, 0], w.A[w.root[0]], w.Bt)
    for i in range(t.n):
        rows[i + 1] = markov_tree.node_logits(w.L[0, min(int(t.depths[i]), w.Bk - 1)],
                                              w.A[t.tokens[i]], w.Bt)
    path, _ = accept.stochastic_walk(t, rows, 1.0, seed=9)
    node, want = -1, []
    while t.children(node).size:
        node = int(t.children(node)[0])
        want.append(node)
    assert path == want


@pytest.mark.parametrize("n_rows", [1, 5])
def test_attention_chain_is_causal_sdpa(n_rows):
    w = make_workload("tiny", seed=8)
    q, kp, vp, kt, vt = __import__("gen").attention_inputs(w, n_rows, 0)
    n = n_rows - 1
    anc = np.array([(1 << (i + 1)) - 1 for i in range(n)], np.uint64)   # chain
    out = verify_attn.tree_attention(q, kp, vp, kt, vt, anc, n, 1 / math.sqrt(w.d))
    # causal SDPA over prefix + tree rows equals chain-masked attention
    P = kp.shape[0]
    K = torch.from_numpy(np.concatenate([kp, kt], 0)).double().permute(1, 0, 2)
    Vv = torch.from_numpy(np.concatenate([vp, vt], 0)).double().permute(1, 0, 2)
    Q = torch.from_numpy(q).double().permute(1, 0, 2)
    mask = torch.ones(n_rows, P + n_rows, dtype=torch.bool).tril(P)
    ref = torch.nn.functional.scaled_dot_product_attention(Q, K, Vv, attn_mask=mask)
    assert np.allclose(out, ref.permute(1, 0, 2).numpy(), atol=1e-10)


def test_attention_tree_mask_matches_sdpa_mask():
    w = make_workload("tiny", seed=9)
    t = markov_tree.build_tree(w.L[0], w.A, w.Bt, w.root[0], k=2, N=8)
    q, kp, vp, kt, vt = __import__("gen").attention_inputs(w, t.n + 1, 0)
    out = verify_attn.tree_attention(q, kp, vp, kt, vt, t.anc, t.n, 0.125)
    P, R = kp.shape[0], t.n + 1
    mask = torch.zeros(R, P + R, dtype=torch.bool)
    mask[:, :P] = True
    mask[:, P] = True
    for i in range(t.n):
        mask[i + 1, P + 1 + i] = True
        p = t.parents[i]
        while p >= 0:
            mask[i + 1, P + 1 + p] = True
            p = t.parents[p]
    K = torch.from_numpy(np.concatenate([kp, kt], 0)).double().permute(1, 0, 2)
    Vv = torch.from_numpy(np.concatenate([vp, vt], 0)).double().permute(1, 0, 2)
    Q = torch.from_numpy(q).double().permute(1, 0, 2)
    ref = torch.nn.functional.scaled_dot_product_attention(Q, K, Vv, attn_mask=mask, scale=0.125)
    assert np.allclose(out, ref.permute(1, 0, 2).numpy(), atol=1e-10)


def test_gumbel_siblings_follow_plackett_luce():
    """First two sampled siblings at the root follow sampling without replacement."""
    V = 5
    s = np.log(np.array([0.4, 0.25, 0.2, 0.1, 0.05]))
    counts = {}
    R = 20000
    for off in range(R):
        kids = markov_tree.gumbel_top_k(s, 2, 11, off, 0, ())
        counts[tuple(kids)] = counts.get(tuple(kids), 0) + 1
    q = np.exp(s)
    exp_, obs = [], []
    for a, b in itertools.permutations(range(V), 2):
        exp_.append(R * q[a] * q[b] / (1 - q[a]))
        obs.append(counts.get((a, b), 0))
    chi = scipy.stats.chisquare(obs, exp_)
    assert chi.pvalue > 0.001
