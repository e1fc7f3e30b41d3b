"""Baseline draft-tree variants and the accepted-tokens-per-round study.

Test infrastructure: the plain CPU definition that the library's variant
builds are checked against; nothing on the product path imports it.

Sources:
  * PCTree summary ("From Chains to Trees: Parent-Conditioned Drafting"),
    "k=4, N=32" paragraph: k = 1 collapses the tree to the drafter's greedy
    chain.
  * Same summary, Shared-Markov paragraph: the control tree first walks the
    greedy chain, then gives every node of a depth the distribution that the
    chain computed at that depth, whatever the node's own token.
  * Same summary, mechanism-isolation paragraph and results table: acceptance
    length per verification round, ordered chain < Shared-Markov < PCTree on
    the same drafter weights.

Readings fixed here:
  * "marginal-ranked tree": the block logits alone rank the children (no
    Markov term at all), so every node of a depth has the same children.
  * the Shared-Markov chain is greedy (T = 0) whatever the tree's temperature,
    has min(Bk, N) nodes, and conditions depth 0 on the root token; depth d
    >= 1 uses the chain's depth-d token.
  * acceptance length of a round = accepted draft tokens + 1 (the bonus
    token the target emits where the walk stops).
"""
from __future__ import annotations

import numpy as np

from .accept import greedy_walk, stochastic_walk
from .markov_tree import Tree, build_tree

VARIANTS = ("pctree", "chain", "marginal", "shared_markov")


def greedy_chain(L, A, Bt, root_token, length):
    """Tokens of the drafter's greedy chain, depths 1..length (k = 1 tree)."""
    t = build_tree(L, A, Bt, root_token, 1, length, temp=0.0)
    order = np.argsort(t.depths, kind="stable")
    return t.tokens[order].astype(np.int64)


def cond_tokens(variant, L, A, Bt, root_token, N):
    """Per-depth conditioning tokens of a variant (None = the node's own token)."""
    Bk = np.asarray(L).shape[0]
    if variant in ("pctree", "chain"):
        return None
    if variant == "marginal":
        return [-1] * Bk
    if variant == "shared_markov":
        chain = greedy_chain(L, A, Bt, root_token, min(Bk, N))
        cond = [int(root_token)] + [int(c) for c in chain[: Bk - 1]]
        return cond + [-1] * (Bk - len(cond))
    raise ValueError(f"unknown variant {variant!r}")


def variant_tree(variant, L, A, Bt, root_token, k, N, **kw) -> Tree:
    """The draft tree of ``variant`` for one request (keyword arguments as
    ``build_tree``; the chain uses k = 1)."""
    cond = cond_tokens(variant, L, A, Bt, root_token, N)
    if variant == "chain":
        k = 1
    return build_tree(L, A, Bt, root_token, k, N, cond_tokens=cond, **kw)


def acceptance_length(tree: Tree, t_rows, temp=0.0, **walk_kw):
    """Accepted draft tokens + 1 for one verified round of ``tree``."""
    if temp > 0:
        path, _ = stochastic_walk(tree, t_rows, temp, **walk_kw)
    else:
        path, _ = greedy_walk(tree, t_rows)
    return len(path) + 1
