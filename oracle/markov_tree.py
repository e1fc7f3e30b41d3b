"""Parent-conditioned node distributions and the best-first budget-N draft tree.

Sources (the pages give no formulas for these steps; the plain readings taken
are listed with each function):
  * PCTree summary, DSpark paragraph: one parallel backbone forward yields a
    block of logits, and a light Markov head biases that block by the previous
    token.  Reading: z_u = L[depth(u)] + A[tok(u)] . B^T (low rank r), row d of
    the block gives the distribution of the children of a depth-d node.
  * PCTree summary, "k=4, N=32" paragraph: the chain is unrolled into a
    budget-limited tree sharing the block logits; k=1 collapses it to the
    greedy chain.
  * TreeSpark article, "core idea" section: the Markov head's parent-
    conditioned distribution is calibrated into an edge-acceptance estimate;
    path survival drives best-first expansion and per-round stopping.
  * TreeSpark article, "lossless" section: siblings are sampled without
    replacement.

Readings fixed here (the pages leave each of these open):
  * temperature: s = z / T for T > 0; at T = 0 tokens are the top-k of z and
    the survival estimate uses T = 1.
  * calibration of child depth d: c_d(l) = min(0, alpha_d * l + beta_d),
    identity = (1, 0); alpha_d >= 0 keeps it monotone.
  * a child of rank j (0-based) gets key S(parent) + c(logq_(j)), where
    logq_(j) is the j-th largest log-probability of the parent's distribution
    (an order statistic), never the sampled token's own probability.
  * candidates are popped in the total order (key desc, depth asc, parent
    index asc, rank asc); popping stops at N nodes or at the first key with
    exp(key) < lambda, decided in fp32 as key >= fp32(log(lambda)).
  * at T > 0 siblings are the Gumbel-top-k of s + G, G = -log(-log U) with
    Philox uniforms (purpose 0, counter words 1-2 = the node's path id).
"""
from __future__ import annotations

import dataclasses
import heapq
import math
from typing import Callable, Optional

import numpy as np

from . import philox

NEG_INF = float("-inf")


def node_logits(L_row, A_row, Bt):
    """z[x] = L[x] + sum_rho A_row[rho] * Bt[x, rho], in fp64 (exact inputs)."""
    return np.asarray(L_row, np.float64) + np.asarray(Bt, np.float64) @ np.asarray(A_row, np.float64)


def scaled_logits(z, temp):
    """s = z / T_r with T_r = T if T > 0 else 1, and log-sum-exp of s."""
    t_r = temp if temp > 0 else 1.0
    s = np.asarray(z, np.float64) / t_r
    m = float(s.max())
    lse = m + math.log(float(np.exp(s - m).sum()))
    return s, lse


def top_k_desc(values, k):
    """Indices of the k largest values, largest first, ties to the lower index."""
    values = np.asarray(values)
    order = np.lexsort((np.arange(values.size), -values))
    return order[:k]


def calibrate(logq, child_depth, calib):
    """c_d(l) = min(0, alpha_d * l + beta_d); calib is (Bk, 2) or None (identity)."""
    if calib is None:
        return min(0.0, logq)
    a, b = (float(v) for v in calib[child_depth - 1])
    return min(0.0, a * logq + b)


def lambda_threshold(lam):
    """fp32 threshold on keys: include a node iff key >= fp32(log(lambda))."""
    if lam <= 0.0:
        return NEG_INF
    return float(np.float32(math.log(float(lam))))


def f32(x):
    return float(np.float32(x))


def gumbel_top_k(s, k, seed, offset, request, ranks, margins=None):
    """Ordered k siblings sampled without replacement from softmax(s).

    Gumbel-top-k: the k largest s_x + G_x with G_x = -log(-log U_x) are a
    without-replacement sample in sampling order (Kool, van Hoof, Welling 2019).
    """
    V = s.size
    pid = philox.path_id(ranks)
    U = philox.uniforms(seed, offset, philox.PURPOSE_SIBLINGS, request,
                        pid & 0xFFFFFFFF, pid >> 32, np.arange(V))
    g = s + (-np.log(-np.log(U)))
    idx = top_k_desc(g, min(k + 1, V))
    if margins is not None and idx.size > 1:
        vals = g[idx]
        gaps = np.abs(np.diff(vals)) / np.maximum(1.0, np.abs(vals[:-1]))
        margins.append(("gumbel_order", float(gaps.min()), tuple(ranks)))
    return idx[:k]


@dataclasses.dataclass
class Expansion:
    """What expanding one node (or the root) produced."""
    row: int                  # 0 = root, i + 1 = node i
    depth: int
    token: int
    lse: float
    logq: np.ndarray          # (k,) order statistics s_(j) - lse
    children: np.ndarray      # (k,) child tokens in rank order
    q: Optional[np.ndarray]   # (V,) fp64 draft distribution (T > 0 only)


@dataclasses.dataclass
class Tree:
    tokens: np.ndarray        # (n,) int32
    parents: np.ndarray       # (n,) int32, -1 = root
    depths: np.ndarray        # (n,) int32, 1..Bk
    ranks: np.ndarray         # (n,) int32, 0-based sibling rank
    keys: np.ndarray          # (n,) float32 cumulative calibrated log-survival
    keys64: np.ndarray        # (n,) float64
    anc: np.ndarray           # (n,) uint64, bit j = node j is ancestor-or-self
    expansions: dict          # row -> Expansion (rows that were expanded)
    margins: list             # (kind, relative margin, context)

    @property
    def n(self):
        return int(self.tokens.size)

    def children(self, node):
        """Children of ``node`` (-1 = root) in rank order."""
        idx = np.nonzero(self.parents == node)[0]
        return idx[np.argsort(self.ranks[idx], kind="stable")]

    def path_ranks(self, node):
        out = []
        while node >= 0:
            out.append(int(self.ranks[node]))
            node = int(self.parents[node])
        return tuple(reversed(out))


Sampler = Callable[[tuple, np.ndarray, float, int], np.ndarray]


def build_tree(L, A, Bt, root_token, k, N, temp=0.0, lam=0.0, calib=None,
               seed=0, offset=0, request=0, sampler: Optional[Sampler] = None,
               key_mode="order_stat", cond_tokens=None) -> Tree:
    """Sequential best-first construction of one request's draft tree.

    L: (Bk, V) block logits of this request; A, Bt: (V, r) Markov factors.
    ``sampler(ranks, s, lse, k)`` may replace the Philox Gumbel draw (used by
    the exact-enumeration tests).  ``key_mode="own_q"`` is a deliberately
    wrong variant (keys from the sampled token's own probability) that the
    tests use as a negative control; the method uses ``"order_stat"``.

    ``cond_tokens`` (length Bk) replaces the parent token in the Markov term
    for the baseline variants of the PCTree summary's mechanism-isolation
    paragraph: every node at depth d draws its children from
    L[d] + A[cond_tokens[d]] . B^T, or from L[d] alone where the entry is -1.
    None (the method) conditions each node on its own token.
    """
    L = np.asarray(L)
    Bk, V = L.shape
    if not 1 <= k <= V:
        raise ValueError("need 1 <= k <= V")
    if calib is not None and np.any(np.asarray(calib)[:, 0] < 0):
        raise ValueError("calibration slopes must be >= 0")
    thr = lambda_threshold(lam)
    margins: list = []
    expansions: dict = {}

    if cond_tokens is not None and len(cond_tokens) != Bk:
        raise ValueError("cond_tokens needs one entry per block row")

    def markov_row(depth, token):
        if cond_tokens is None:
            return A[token]
        c = int(cond_tokens[depth])
        return np.zeros(A.shape[1]) if c < 0 else A[c]

    def expand(row, depth, token, ranks):
        z = node_logits(L[depth], markov_row(depth, token), Bt)
        s, lse = scaled_logits(z, temp)
        order = top_k_desc(s, k)
        logq = s[order] - lse
        if temp > 0:
            if sampler is None:
                kids = gumbel_top_k(s, k, seed, offset, request, ranks, margins)
            else:
                kids = np.asarray(sampler(ranks, s, lse, k))
            q = np.exp(s - lse)
        else:
            kids = order
            q = None
        if key_mode == "own_q":
            logq = s[kids] - lse
        e = Expansion(row, depth, int(token), lse, logq, np.asarray(kids, np.int64), q)
        expansions[row] = e
        return e

    heap = []

    def push_children(e, parent_idx, parent_key64, ranks):
        for j in range(k):
            key64 = parent_key64 + calibrate(float(e.logq[j]), e.depth + 1, calib)
            item = (-f32(key64), e.depth + 1, parent_idx, j)
            heapq.heappush(heap, (item, key64, int(e.children[j]), ranks + (j,)))

    root_e = expand(0, 0, int(root_token), ())
    push_children(root_e, -1, 0.0, ())

    tokens, parents, depths, ranks_l, keys64, anc = [], [], [], [], [], []
    while len(tokens) < N and heap:
        item, key64, tok, ranks = heapq.heappop(heap)
        negk, depth, parent_idx, j = item
        if not (-negk >= thr):
            margins.append(("lambda", abs(key64 - thr) / max(1.0, abs(thr)), ranks))
            break
        if thr != NEG_INF:
            margins.append(("lambda", abs(key64 - thr) / max(1.0, abs(thr)), ranks))
        i = len(tokens)
        tokens.append(tok)
        parents.append(parent_idx)
        depths.append(depth)
        ranks_l.append(j)
        keys64.append(key64)
        anc.append((0 if parent_idx < 0 else anc[parent_idx]) | (1 << i))
        if depth < Bk:
            e = expand(i + 1, depth, tok, ranks)
            push_children(e, i, key64, ranks)

    # decision margins between neighbours of the final order, including the
    # best rejected candidate; exact fp64 ties are settled by the tie rule
    rest = sorted(heap)[:1]
    seq = keys64 + [r[1] for r in rest]
    for a, b in zip(seq[:-1], seq[1:]):
        if a != b:
            margins.append(("key_order", abs(a - b) / max(1.0, abs(a)), None))

    n = len(tokens)
    if n > 64:
        raise ValueError("ancestor bitmask holds at most 64 nodes")
    return Tree(
        tokens=np.asarray(tokens, np.int32), parents=np.asarray(parents, np.int32),
        depths=np.asarray(depths, np.int32), ranks=np.asarray(ranks_l, np.int32),
        keys=np.asarray(keys64, np.float64).astype(np.float32),
        keys64=np.asarray(keys64, np.float64),
        anc=np.asarray(anc, np.uint64), expansions=expansions, margins=margins)
