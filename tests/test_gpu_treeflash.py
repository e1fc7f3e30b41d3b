"""TreeFlash round on the GPU (dt_treeflash_build) against the oracle.

The oracle runs with its bf16 store hook, so both sides take their top-M and
selection decisions on the same bf16 activations (x, silu(g) * u, h').  The
remaining differences are fp32 accumulation order and rare one-ulp rounding
flips of those activations, far below the decision margins of the chosen
seeds; the test asserts those margins (> 1e-3) before it demands equality.
Tree structure is compared exactly, keys within 1e-3.
"""
import numpy as np
import pytest
import torch

from gen import treeflash_inputs
from oracle import treeflash
from oracle.markov_tree import top_k_desc

pytestmark = pytest.mark.gpu

CASES = [  # seed, V, D, Dff, gamma, M, budget, batch
    (1, 1024, 128, 128, 5, 3, 10, 2),
    (3, 1536, 128, 64, 4, 2, 8, 2),
    (4, 4096, 192, 128, 8, 4, 16, 2),
    (6, 1000, 128, 64, 5, 3, 9, 2),   # ragged last vocabulary tile
    (8, 1000, 64, 64, 5, 3, 9, 2),    # D smaller than one weight tile
]


def _oracle(x, b, M, budget):
    return treeflash.treeflash_tree(x["h"][b], x["E"], int(x["root"][b]), M, budget,
                                    x["w_norm_h"], x["w_norm_e"], x["W_gate"], x["W_up"],
                                    x["W_down"], x["W_lm"], store=treeflash.bf16_rne)


def _min_margin(x, b, M, tree, sets, dist):
    """Smallest gap at any top-M or selection decision of request b."""
    W = x["W_lm"].astype(np.float64)
    gaps = []
    for i in range(x["h"].shape[1]):
        v = np.sort(W @ x["h"][b][i].astype(np.float64))[::-1]
        gaps.append(v[M - 1] - v[M])
    for s, _ in dist.values():
        v = np.sort(s)[::-1]
        gaps.append(v[M - 1] - v[M])
    keys = []

    def push(d, prev, k0):
        if (d + 1, prev) in dist:
            s, l = dist[(d + 1, prev)]
            keys.extend(k0 + s[t] - l for t in top_k_desc(s, M))

    push(0, int(x["root"][b]), 0.0)
    for i in range(tree.n):
        push(int(tree.depths[i]), int(tree.tokens[i]), float(tree.keys64[i]))
    if len(keys) > 1:
        gaps.append(np.min(np.diff(np.sort(keys))))
    return min(gaps)


@pytest.mark.parametrize("seed,V,D,Dff,gamma,M,budget,batch", CASES)
def test_treeflash_tree_matches_oracle(seed, V, D, Dff, gamma, M, budget, batch):
    import draft_tree_construction_markov_b200 as dt

    x = treeflash_inputs(seed, V=V, D=D, Dff=Dff, positions=gamma, batch=batch)
    bf = torch.bfloat16
    cu = lambda a, t=None: torch.from_numpy(np.ascontiguousarray(a)).cuda().to(t or torch.float32)
    out = dt.Tree.empty(batch, budget, V, stochastic=False)
    ws = dt.workspace(dt.treeflash_workspace_bytes(batch, gamma, D, Dff, V, M, budget))
    dt.treeflash_build(cu(x["h"], bf), cu(x["E"], bf), cu(x["w_norm_h"]), cu(x["w_norm_e"]),
                       cu(x["W_gate"], bf), cu(x["W_up"], bf), cu(x["W_down"], bf),
                       cu(x["W_lm"], bf), torch.from_numpy(x["root"]).cuda(), M=M,
                       budget=budget, out=out, ws=ws)
    assert dt.read_status(ws) == 0
    for b in range(batch):
        tree, sets, dist = _oracle(x, b, M, budget)
        assert _min_margin(x, b, M, tree, sets, dist) > 1e-3
        n = int(out.n_nodes[b])
        assert n == tree.n
        g = lambda t: t[b, :n].cpu().numpy()
        assert np.array_equal(g(out.tokens), tree.tokens)
        assert np.array_equal(g(out.parents), tree.parents)
        assert np.array_equal(g(out.depths), tree.depths)
        assert np.array_equal(g(out.ranks), tree.ranks)
        assert np.array_equal(g(out.anc).astype(np.uint64), tree.anc)
        assert np.allclose(g(out.keys), tree.keys64, atol=1e-3, rtol=0)


def test_treeflash_rejects_bad_shapes():
    import draft_tree_construction_markov_b200 as dt
    from draft_tree_construction_markov_b200 import _lib

    x = treeflash_inputs(1, V=1024, D=128, Dff=128, positions=5, batch=2)
    bf = torch.bfloat16
    cu = lambda a, t=None: torch.from_numpy(np.ascontiguousarray(a)).cuda().to(t or torch.float32)
    out = dt.Tree.empty(2, 10, 1024, stochastic=False)
    ws = dt.workspace(dt.treeflash_workspace_bytes(2, 5, 128, 128, 1024, 3, 10))
    args = [cu(x["h"], bf), cu(x["E"], bf), cu(x["w_norm_h"]), cu(x["w_norm_e"]),
            cu(x["W_gate"], bf), cu(x["W_up"], bf), cu(x["W_down"], bf), cu(x["W_lm"], bf),
            torch.from_numpy(x["root"]).cuda()]
    with pytest.raises(_lib.DtreeError) as e:
        dt.treeflash_build(*args, M=17, budget=10, out=out, ws=ws)
    assert e.value.code == _lib.DT_EUNSUPPORTED
    with pytest.raises(_lib.DtreeError) as e:
        dt.treeflash_build(*args, M=3, budget=10, out=out, ws=ws[:64])
    assert e.value.code == _lib.DT_EWORKSPACE
