"""TreeFlash round: SwiGLU AR-approximator over a one-shot drafter block, then
a draft tree chosen from the modified distributions.

Sources (TreeFlash explainer):
  * method section 1: h'_{t+i} = h_{t+i} + SwiGLU(h~_{t+i} :: e_{t+i-1}), with
    h~ the normalised drafter hidden state and e the normalised input
    embedding of the previous token.
  * method section 2: stage 1 builds a top-M tree from the unmodified drafter
    distributions, with exactly M unique tokens per depth; stage 2 evaluates
    the approximator on that tree's nodes, M * gamma parallel evaluations
    independent of the budget B; the final tree is chosen from the modified
    distributions by OPT-Tree.
  * method section 3: the approximator starts from zero (the model then
    equals the plain drafter), which the tests use as a pin.

Readings fixed here:
  * "normalised" = RMSNorm x / sqrt(mean(x^2) + eps) * w with eps = 1e-6;
    SwiGLU(x) = W_down (silu(W_gate x) * (W_up x)), silu(x) = x * sigmoid(x);
    no final norm before the LM head: logits = W_lm h'.
  * depth i (1..gamma) uses drafter position i; S_i = top-M tokens of the
    stage-1 logits W_lm h_i (ties to the lower id).
  * stage 2 evaluates q'_1(. | root) and q'_i(. | t) for every t in S_{i-1}.
  * OPT-Tree (named, not defined, on the page): maximising the expected
    accepted length over a candidate tree is taking the B nodes of highest
    path probability, i.e. best-first by cumulative log q' under the same
    total order as the Markov tree (key desc, depth asc, parent index asc,
    rank asc).  Candidates are the top-M children of a node; a node whose
    token is outside S_depth has no evaluated distribution and is a leaf.
  * temperature 0: tokens by top-M of the logits, survival from T = 1.
  * `store` (optional) is applied where a bf16 network stores an activation
    that feeds the next GEMM: x, silu(g) * u and h'.  With store=bf16_rne the
    oracle takes its top-M decisions on the same bf16 activations as a bf16
    kernel; store=None is the plain fp64 definition.
"""
from __future__ import annotations

import heapq

import numpy as np

from .markov_tree import Tree, f32, scaled_logits, top_k_desc

EPS = 1e-6


def rmsnorm(x, w, eps=EPS):
    x = np.asarray(x, np.float64)
    return x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps) * np.asarray(w, np.float64)


def silu(x):
    return x / (1.0 + np.exp(-x))


def bf16_rne(x):
    """Round to float32, then to bfloat16 (round to nearest, ties to even); fp64 out."""
    u = np.asarray(x, np.float64).astype(np.float32).view(np.uint32).astype(np.uint64)
    u = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16) << 16
    return u.astype(np.uint32).view(np.float32).astype(np.float64)


def ar_approximator(h, e_prev, w_norm_h, w_norm_e, W_gate, W_up, W_down, store=None):
    """h' = h + W_down(silu(W_gate x) * (W_up x)), x = [rms(h) :: rms(e_prev)]."""
    keep = store if store is not None else (lambda v: v)
    x = keep(np.concatenate([rmsnorm(h, w_norm_h), rmsnorm(e_prev, w_norm_e)], axis=-1))
    g = np.asarray(W_gate, np.float64) @ x
    u = np.asarray(W_up, np.float64) @ x
    act = keep(silu(g) * u)
    return keep(np.asarray(h, np.float64) + np.asarray(W_down, np.float64) @ act)


def stage1_sets(h, W_lm, M):
    """S_i (i = 1..gamma): the M best tokens of W_lm h_i; returns list of arrays
    (the gamma matrix-vector products as one matrix product W_lm [h_1 ... h_gamma])."""
    W = np.asarray(W_lm, np.float64)
    Z = W @ np.asarray(h, np.float64).T
    return [top_k_desc(Z[:, i], M) for i in range(len(h))]


def stage2_distributions(h, E, root, sets, w_norm_h, w_norm_e, W_gate, W_up, W_down, W_lm,
                         store=None):
    """{(depth, prev): (s, lse)} for depth 1 (prev = root) and every prev in S_{depth-1}.

    The LM head of every evaluation is one column of a single matrix product
    W_lm [h'_1 ... h'_n] (the same dot products as one matrix-vector product
    per evaluation, read with one pass over W_lm)."""
    W = np.asarray(W_lm, np.float64)
    out = {}
    evals = [(1, int(root))] + [(i, int(t)) for i in range(2, len(h) + 1) for t in sets[i - 2]]
    H = np.stack([ar_approximator(h[d - 1], E[prev], w_norm_h, w_norm_e, W_gate, W_up, W_down,
                                  store) for d, prev in evals], axis=1)
    Z = W @ H
    for j, (d, prev) in enumerate(evals):
        out[(d, prev)] = scaled_logits(Z[:, j], 0.0)
    return out


def treeflash_tree(h, E, root, M, budget, w_norm_h, w_norm_e, W_gate, W_up, W_down, W_lm,
                   store=None):
    """Best-first top-`budget` tree over the stage-2 distributions of one request."""
    gamma = len(h)
    sets = stage1_sets(h, W_lm, M)
    dist = stage2_distributions(h, E, root, sets, w_norm_h, w_norm_e, W_gate, W_up, W_down, W_lm,
                                store)
    in_set = [set(int(t) for t in s) for s in sets]

    heap = []

    def push_children(depth, prev, parent_idx, parent_key):
        if (depth + 1, prev) not in dist:
            return
        s, lse = dist[(depth + 1, prev)]
        kids = top_k_desc(s, M)
        for j, x in enumerate(kids):
            key = parent_key + (s[x] - lse)
            heapq.heappush(heap, ((-f32(key), depth + 1, parent_idx, j), key, int(x)))

    push_children(0, int(root), -1, 0.0)
    tokens, parents, depths, ranks, keys, anc = [], [], [], [], [], []
    while len(tokens) < budget and heap:
        (negk, d, p, j), key, tok = heapq.heappop(heap)
        i = len(tokens)
        tokens.append(tok)
        parents.append(p)
        depths.append(d)
        ranks.append(j)
        keys.append(key)
        anc.append((0 if p < 0 else anc[p]) | (1 << i))
        if d < gamma and tok in in_set[d - 1]:
            push_children(d, tok, i, key)
    tree = Tree(tokens=np.asarray(tokens, np.int32), parents=np.asarray(parents, np.int32),
                depths=np.asarray(depths, np.int32), ranks=np.asarray(ranks, np.int32),
                keys=np.asarray(keys).astype(np.float32), keys64=np.asarray(keys, np.float64),
                anc=np.asarray(anc, np.uint64), expansions={}, margins=[])
    return tree, sets, dist
