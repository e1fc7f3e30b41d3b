"""GPU parity of the baseline tree variants (dt_tree_build_ex) and of the
acceptance study against the oracle (oracle/variants.py).

Trees must match the oracle's exactly (tokens, parents, depths, ranks,
ancestor masks, node counts); keys within 1e-5.  The acceptance lengths
the library's greedy walk gives on these trees must equal the oracle's.
"""
import ctypes

import numpy as np
import pytest
import torch

from gen import make_workload
from oracle import variants

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import draft_tree_construction_markov_b200 as dt
    from draft_tree_construction_markov_b200 import _lib
    from tests.gpu_util import BF16, build_inputs, dev, target_for_tree, tree_to_host

VARIANTS = ["pctree", "chain", "marginal", "shared_markov"]


def run_variant(w, variant, temp, seed=None):
    x = build_inputs(w)
    tree = dt.Tree.empty(w.batch, w.Nmax, w.V, stochastic=temp > 0)
    ws = dt.workspace(dt.build_workspace_bytes(w.batch, w.Bk, w.V, w.r, w.k, w.Nmax))
    dt.tree_build(x["block_logits"], x["markov_a"], x["markov_b"], x["root_token"],
                  x["n_budget"], x["lam"], k=w.k, Nmax=w.Nmax, temp=temp, out=tree, ws=ws,
                  calib=x["calib"], k_req=x["k_req"],
                  philox_seed=w.philox_seed if seed is None else seed, variant=variant)
    assert dt.read_status(ws) == 0
    return tree


_F64 = {}


def oracle_variant(w, variant, b, temp, seed=None):
    if _F64.get("w") is not w:   # fp64 copies of the Markov factors, once per workload
        _F64.update(w=w, A=w.A.astype(np.float64), Bt=w.Bt.astype(np.float64))
    return variants.variant_tree(
        variant, w.L[b], _F64["A"], _F64["Bt"], int(w.root[b]), int(w.k_req[b]), int(w.n_budget[b]),
        temp=temp, lam=float(w.lam[b]), calib=w.calib,
        seed=w.philox_seed if seed is None else seed, request=b)


def compare(w, tree, variant, b, temp):
    o = oracle_variant(w, variant, b, temp)
    h = tree_to_host(tree, b)
    ties = [m for m in o.margins if m[1] < 1e-5]
    msg = f"{variant} request {b}: near-ties {ties[:5]}"
    assert h["n"] == o.n, msg
    for f in ("tokens", "parents", "depths", "ranks", "anc"):
        assert np.array_equal(h[f], getattr(o, f)), f"{f}: {msg}"
    np.testing.assert_allclose(h["keys"], o.keys64, rtol=1e-5, atol=1e-5)
    if temp > 0 and o.n > 0:
        q = tree.draft_q[b].cpu().numpy()
        for r in [0] + [i + 1 for i in range(o.n) if o.depths[i] < w.Bk]:
            ref = o.expansions[r].q
            big = ref > 1e-30
            np.testing.assert_allclose(q[r].astype(np.float64)[big], ref[big], rtol=1e-5, atol=0)
    return o


CASES = [
    ("tiny", dict(sigma_ab=0.35), 0.0),
    ("tiny", dict(sigma_ab=0.35), 1.0),
    ("tiny", dict(V=1000, r=32, Bk=5, k=3, N=20, sigma_ab=0.35), 0.0),   # ragged vocab tile
    ("tiny", dict(V=1000, r=32, Bk=5, k=3, N=20, sigma_ab=0.35), 0.8),
    ("tiny", dict(V=777, r=48, Bk=6, k=5, N=40), 0.0),                   # 64-column node tiles
    ("tiny", dict(V=700, r=320, Bk=4, k=3, N=40), 0.0),                  # rows through H (TMA)
    ("tiny", dict(V=700, r=320, Bk=4, k=3, N=40), 0.9),
]


@pytest.mark.parametrize("variant", VARIANTS)
@pytest.mark.parametrize("name,over,temp", CASES)
def test_variant_tree_parity(variant, name, over, temp):
    for seed in (0, 1):
        w = make_workload(name, seed=seed, temp=temp, **over)
        tree = run_variant(w, variant, temp)
        for b in range(w.batch):
            compare(w, tree, variant, b, temp)


@pytest.mark.parametrize("variant", VARIANTS)
def test_variant_batch_budgets_lambda_calibration(variant):
    w = make_workload("tiny", seed=3, batch=5, V=600, N=12, k=3, sigma_ab=0.35)
    w.n_budget[:] = np.array([12, 1, 0, 7, 12], np.int32)
    w.k_req[:] = np.array([3, 3, 1, 2, 1], np.int32)
    w.lam[:] = np.array([0.0, 0.0, 0.0, 0.02, 1e-4], np.float32)
    w.calib = np.array([[0.5, -0.1], [1.5, 0.2], [1.0, 0.0], [0.8, -0.3]], np.float32)
    tree = run_variant(w, variant, 0.0)
    for b in range(w.batch):
        compare(w, tree, variant, b, 0.0)


@pytest.mark.parametrize("variant", VARIANTS)
def test_variant_full_vocabulary(variant):
    # the qwen3_4b-shaped round at full size, one request
    w = make_workload("qwen3_4b", seed=2, sigma_ab=0.35)
    tree = run_variant(w, variant, 0.0)
    compare(w, tree, variant, 0, 0.0)


def test_shared_markov_stochastic_block16():
    w = make_workload("qwen3_8b", seed=1, sigma_ab=0.35, N=24)
    tree = run_variant(w, "shared_markov", w.temp)
    compare(w, tree, "shared_markov", 0, w.temp)


def test_acceptance_lengths_match_oracle():
    w = make_workload("qwen3_4b", seed=5, V=4096, batch=6, Bk=16, N=32, sigma_ab=0.35)
    for variant in VARIANTS:
        tree = run_variant(w, variant, 0.0)
        tgt = np.zeros((w.batch, w.Nmax + 1, w.V), np.float32)
        orc = []
        for b in range(w.batch):
            o = compare(w, tree, variant, b, 0.0)
            tgt[b] = target_for_tree(w, b, o.depths, o.tokens)
            orc.append(variants.acceptance_length(o, tgt[b, : o.n + 1].astype(np.float64)))
        acc = torch.empty(w.batch, w.Bk, dtype=torch.int32, device="cuda")
        nacc = torch.empty(w.batch, dtype=torch.int32, device="cuda")
        bonus = torch.empty(w.batch, dtype=torch.int32, device="cuda")
        ws = dt.workspace(dt.accept_workspace_bytes(w.batch, w.Nmax, w.V))
        dt.tree_accept(dev(tgt, BF16), tree, w.Bk, 0.0, acc, nacc, bonus, ws)
        assert dt.read_status(ws) == 0
        assert (nacc.cpu().numpy() + 1).tolist() == orc, variant


def test_unknown_variant_is_rejected():
    w = make_workload("tiny", seed=0)
    x = build_inputs(w)
    tree = dt.Tree.empty(w.batch, w.Nmax, w.V)
    ws = dt.workspace(dt.build_workspace_bytes(w.batch, w.Bk, w.V, w.r, w.k, w.Nmax))
    st = tree.c_struct()
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    code = _lib.lib.dt_tree_build_ex(
        p(x["block_logits"]), _lib.DT_F32, p(x["markov_a"]), p(x["markov_b"]), w.r, None,
        p(x["root_token"]), p(x["n_budget"]), None, p(x["lam"]), w.batch, w.Bk, w.V, w.k,
        w.Nmax, 0.0, 0, 0, 7, ctypes.byref(st), p(ws), ws.numel(), _lib.stream_ptr())
    assert code == _lib.DT_EINVAL
