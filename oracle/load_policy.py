"""Load-adaptive tree budget: one survival signal allocates a round's
verification capacity over the requests of a batch.

Test infrastructure: the plain CPU definition the library's
dt_tree_load_budget is checked against; nothing on the product path imports
it.

Sources:
  * TreeSpark article, "core idea": the load-adaptive serving policy sizes the
    trees by the current load, with the same calibrated path survival that
    drives expansion and stopping.
  * TreeSpark article, "measured gains": as load rises the trees shrink back
    toward the chain.

Readings fixed here (the pages give no formula):
  * a verified node of request i costs w_i = 1 + floor(P_i / prefix_unit)
    units (P_i its prefix length: the verification forward reads the prefix
    for each node; prefix_unit = 0 makes every node cost 1); a round has a
    capacity of C units;
  * the nodes of the batch are ordered by survival, i.e. (fp32 key desc,
    request asc, pop index asc), and the batch keeps the longest prefix of
    that order whose total cost is <= C.  Within a request the order is its
    own pop order, so every request keeps a prefix of its tree (ancestor
    closed); high load cuts each tree back to its most likely nodes.
"""
from __future__ import annotations

import numpy as np


def node_cost(prefix_len, prefix_unit):
    """Cost in units of one verified node of each request."""
    p = np.asarray(prefix_len, np.int64)
    if prefix_unit <= 0:
        return np.ones_like(p)
    return 1 + p // int(prefix_unit)


def load_budget(keys, n_nodes, prefix_len, capacity, prefix_unit):
    """Nodes each request keeps.

    keys: (batch, >= max n) fp32 keys in pop order; n_nodes: (batch,).
    """
    keys = np.asarray(keys, np.float32)
    n_nodes = np.asarray(n_nodes, np.int64)
    if prefix_len is None:  # no prefix lengths: every node costs one unit
        prefix_len = np.zeros(len(n_nodes), np.int64)
    w = node_cost(prefix_len, prefix_unit)
    order = sorted(((-float(keys[b, i]), b, i) for b in range(len(n_nodes))
                    for i in range(int(n_nodes[b]))))
    keep = np.zeros(len(n_nodes), np.int64)
    used = 0
    for _, b, _ in order:
        if used + int(w[b]) > capacity:
            break
        used += int(w[b])
        keep[b] += 1
    return keep
