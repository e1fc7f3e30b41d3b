"""Tree-masked grouped-query attention for verifying every draft node at once.

Source: TreeSpark article, introduction (the target checks all tree nodes in a
single forward pass); PCTree summary, "setup" paragraph (SDPA attention).
The mask is the plain reading of "each node sees the committed prefix, the
root and its own ancestors":

  out[i, h] = sum_j softmax_j(scale * q[i, h] . k[j, h // g] + M[i, j]) v[j, h // g]

rows i: 0 = root, i >= 1 = node i-1; columns: the request's prefix (all
allowed), then tree row 0 (the root, allowed for every row) and tree row
j' + 1 (allowed for row i >= 1 iff bit j' of anc[i - 1] is set).
"""
import numpy as np


def allowed_tree_columns(anc, n, i):
    """Tree columns (0 = root, j + 1 = node j) row i may attend to."""
    cols = [0]
    if i >= 1:
        bits = int(anc[i - 1])
        cols += [j + 1 for j in range(n) if (bits >> j) & 1]
    return cols


def tree_attention(q, k_prefix, v_prefix, k_tree, v_tree, anc, n, scale):
    """fp64 attention of one request.

    q: (n_rows, Hq, d); k/v_prefix: (P, Hkv, d); k/v_tree: (n_rows, Hkv, d);
    rows beyond n + 1 are ignored.  Returns (n + 1, Hq, d) float64.
    """
    q = np.asarray(q, np.float64)
    kp, vp = np.asarray(k_prefix, np.float64), np.asarray(v_prefix, np.float64)
    kt, vt = np.asarray(k_tree, np.float64), np.asarray(v_tree, np.float64)
    Hq, Hkv = q.shape[1], kp.shape[1]
    g = Hq // Hkv
    out = np.zeros((n + 1, Hq, q.shape[2]))
    for i in range(n + 1):
        cols = allowed_tree_columns(anc, n, i)
        for h in range(Hq):
            kv = h // g
            keys = np.concatenate([kp[:, kv], kt[cols, kv]], 0)
            vals = np.concatenate([vp[:, kv], vt[cols, kv]], 0)
            sc = scale * (keys @ q[i, h])
            w = np.exp(sc - sc.max())
            out[i, h] = (w / w.sum()) @ vals
    return out
