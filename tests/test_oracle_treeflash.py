"""Pins of the TreeFlash oracle (TreeFlash explainer, method sections 1-3).

* RMSNorm and SiLU against torch's library routines.
* Zero-initialised approximator (section 3): h' = h, so every modified
  distribution equals the plain drafter's softmax (scipy) and the tree keys
  are sums of plain log-softmax values.
* Stage 1 has exactly M unique tokens per depth; stage 2 needs
  1 + (gamma - 1) * M <= M * gamma evaluations, whatever the budget
  (section 2).
* The selected tree equals the brute-force top-B by path probability over
  the candidate tree (top-M children; only tokens of S_depth expand).
"""
import itertools

import numpy as np
import pytest
import scipy.special
import torch

from oracle import treeflash


def _inputs(seed=0, V=16, D=8, Dff=8, gamma=3):
    g = np.random.default_rng(seed)
    return dict(
        h=g.standard_normal((gamma, D)), E=0.5 * g.standard_normal((V, D)),
        w_norm_h=1 + 0.1 * g.standard_normal(D), w_norm_e=1 + 0.1 * g.standard_normal(D),
        W_gate=g.standard_normal((Dff, 2 * D)) / np.sqrt(2 * D),
        W_up=g.standard_normal((Dff, 2 * D)) / np.sqrt(2 * D),
        W_down=g.standard_normal((D, Dff)) / np.sqrt(Dff),
        W_lm=2 * g.standard_normal((V, D)) / np.sqrt(D), root=3)


def test_rmsnorm_and_silu_match_torch():
    g = np.random.default_rng(1)
    x, w = g.standard_normal((5, 7)), g.standard_normal(7)
    ref = torch.nn.functional.rms_norm(torch.from_numpy(x), (7,), torch.from_numpy(w), eps=1e-6)
    assert np.allclose(treeflash.rmsnorm(x, w), ref.numpy(), atol=1e-12)
    assert np.allclose(treeflash.silu(x), torch.nn.functional.silu(torch.from_numpy(x)).numpy(),
                       atol=1e-12)


def test_zero_down_projection_is_plain_drafter():
    x = _inputs(2)
    x["W_down"] = np.zeros_like(x["W_down"])
    M, B = 3, 10
    tree, sets, dist = treeflash.treeflash_tree(x["h"], x["E"], x["root"], M, B, x["w_norm_h"],
                                                x["w_norm_e"], x["W_gate"], x["W_up"],
                                                x["W_down"], x["W_lm"])
    base = [scipy.special.log_softmax(x["W_lm"] @ x["h"][i]) for i in range(len(x["h"]))]
    for (d, prev), (s, lse) in dist.items():
        assert np.allclose(s - lse, base[d - 1], atol=1e-12)
    for i in range(tree.n):
        want, node = 0.0, i
        while node >= 0:
            want += base[tree.depths[node] - 1][tree.tokens[node]]
            node = tree.parents[node]
        assert abs(tree.keys64[i] - want) < 1e-9


@pytest.mark.parametrize("M,gamma", [(2, 3), (4, 5)])
def test_stage_counts(M, gamma):
    x = _inputs(3, gamma=gamma)
    sets = treeflash.stage1_sets(x["h"], x["W_lm"], M)
    assert all(len(set(s.tolist())) == M for s in sets) and len(sets) == gamma
    for budget in (1, 5, 50):
        _, _, dist = treeflash.treeflash_tree(x["h"], x["E"], x["root"], M, budget, x["w_norm_h"],
                                              x["w_norm_e"], x["W_gate"], x["W_up"],
                                              x["W_down"], x["W_lm"])
        assert len(dist) == 1 + (gamma - 1) * M <= M * gamma


@pytest.mark.parametrize("seed,M,B", [(4, 2, 5), (5, 3, 12), (6, 2, 14)])
def test_tree_is_brute_force_top_b(seed, M, B):
    x = _inputs(seed)
    tree, sets, dist = treeflash.treeflash_tree(x["h"], x["E"], x["root"], M, B, x["w_norm_h"],
                                                x["w_norm_e"], x["W_gate"], x["W_up"],
                                                x["W_down"], x["W_lm"])
    gamma = len(x["h"])
    # enumerate the candidate tree with independently recomputed distributions
    W = x["W_lm"]
    nodes = []

    def logq(d, prev):
        hp = treeflash.ar_approximator(x["h"][d - 1], x["E"][prev], x["w_norm_h"], x["w_norm_e"],
                                       x["W_gate"], x["W_up"], x["W_down"])
        return scipy.special.log_softmax(W @ hp)

    def rec(d, prev, lp, path):
        if d > gamma:
            return
        if d > 1 and prev not in set(sets[d - 2].tolist()):
            return
        lq = logq(d, prev)
        kids = np.lexsort((np.arange(lq.size), -lq))[:M]
        for x_ in kids:
            nodes.append((lp + lq[x_], d, path + (int(x_),)))
            rec(d + 1, int(x_), lp + lq[x_], path + (int(x_),))

    rec(1, x["root"], 0.0, ())
    nodes.sort(key=lambda n: (-n[0], n[1]))
    want = {n[2] for n in nodes[:B]}
    got = set()
    for i in range(tree.n):
        path, node = [], i
        while node >= 0:
            path.append(int(tree.tokens[node]))
            node = tree.parents[node]
        got.add(tuple(reversed(path)))
    assert got == want


def test_bf16_store_matches_torch_rounding():
    """bf16_rne is round-to-nearest-even on the fp32 value (torch's bfloat16 cast)."""
    g = np.random.default_rng(7)
    x = np.concatenate([g.standard_normal(4000) * 10.0 ** g.integers(-3, 4, 4000),
                        # exact halfway cases between two bf16 neighbours
                        (np.arange(1, 200, dtype=np.float64) * 2 + 1) * 2.0 ** -8])
    want = torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(treeflash.bf16_rne(x), want)


def test_bf16_store_stays_within_bf16_error():
    x = _inputs(8, D=16, Dff=16)
    plain = treeflash.ar_approximator(x["h"][0], x["E"][2], x["w_norm_h"], x["w_norm_e"],
                                      x["W_gate"], x["W_up"], x["W_down"])
    stored = treeflash.ar_approximator(x["h"][0], x["E"][2], x["w_norm_h"], x["w_norm_e"],
                                       x["W_gate"], x["W_up"], x["W_down"],
                                       store=treeflash.bf16_rne)
    assert np.all(treeflash.bf16_rne(stored) == stored)  # h' itself is stored in bf16
    assert np.max(np.abs(stored - plain)) <= 0.05 * np.max(np.abs(plain))
    assert not np.array_equal(stored, plain)
