"""GPU parity of the Markov-head GEMM and of tree_build against the CPU oracle.

Tree structure (tokens, parents, depths, ranks, ancestor masks, node counts)
must be bit-exact; keys and draft probabilities agree within 1e-5 relative.
When an integer output differs, the oracle's decision margins are printed so
that a near-tie is reported, never silently excused.
"""
import numpy as np
import pytest
import torch

from gen import make_workload
from oracle import markov_tree

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import draft_tree_construction_markov_b200 as dt
    from tests.gpu_util import BF16, build_inputs, dev, run_build, tree_to_host


@pytest.mark.parametrize("name,over", [
    ("tiny", {}),
    ("tiny", dict(V=1000, r=32, Bk=5)),
    ("qwen3_4b", {}),
])
def test_markov_logits_exact(name, over):
    w = make_workload(name, seed=1, **over)
    x = build_inputs(w)
    g = np.random.default_rng(0)
    n = 40
    req = np.zeros(n, np.int32)
    depth = g.integers(0, w.Bk, n).astype(np.int32)
    tok = g.integers(0, w.V, n).astype(np.int32)
    out = torch.empty(n, w.V, dtype=torch.float32, device="cuda")
    ws = dt.workspace(dt._lib.lib.dt_markov_logits_workspace_bytes(n, w.V, w.r))
    dt.markov_logits(x["block_logits"], x["markov_a"], x["markov_b"], dev(req), dev(depth),
                     dev(tok), out, ws)
    assert dt.read_status(ws) == 0
    z = out.cpu().numpy()
    for i in range(n):
        ref = markov_tree.node_logits(w.L[0, depth[i]], w.A[tok[i]], w.Bt)
        # dyadic inputs: the fp32 tensor-core result is exact
        assert np.array_equal(z[i].astype(np.float64), ref), f"row {i}"


def _oracle_tree(w, b, temp, seed, offset=0):
    return markov_tree.build_tree(
        w.L[b], w.A, w.Bt, int(w.root[b]), int(w.k_req[b]), int(w.n_budget[b]), temp=temp,
        lam=float(w.lam[b]), calib=w.calib, seed=seed, offset=offset, request=b)


def _near_ties(o, lim=1e-5):
    return [m for m in o.margins if m[1] < lim]


def compare_tree(w, tree, b, temp, seed, offset=0):
    o = _oracle_tree(w, b, temp, seed, offset)
    h = tree_to_host(tree, b)
    ties = _near_ties(o)
    msg = f"request {b}: near-ties {ties[:5]}"
    assert h["n"] == o.n, msg
    assert np.array_equal(h["tokens"], o.tokens), msg
    assert np.array_equal(h["parents"], o.parents), msg
    assert np.array_equal(h["depths"], o.depths), msg
    assert np.array_equal(h["ranks"], o.ranks), msg
    assert np.array_equal(h["anc"], o.anc), msg
    np.testing.assert_allclose(h["keys"], o.keys64, rtol=1e-5, atol=1e-5)
    if temp > 0 and o.n > 0:   # an empty tree needs (and gets) no draft rows
        q = tree.draft_q[b].cpu().numpy()
        rows = [0] + [i + 1 for i in range(o.n) if o.depths[i] < w.Bk]
        for r in rows:
            ref = o.expansions[r].q
            got = q[r].astype(np.float64)
            # 1e-5 relative on every probability above 1e-30 (fp32 range)
            big = ref > 1e-30
            np.testing.assert_allclose(got[big], ref[big], rtol=1e-5, atol=0)
    return o


CASES = [
    ("tiny", {}, 0.0),
    ("tiny", {}, 1.0),
    ("tiny", dict(V=1000, r=32, Bk=5, k=3, N=20), 0.0),   # ragged last vocab tile
    ("tiny", dict(V=1000, r=32, Bk=5, k=3, N=20), 0.8),
    ("tiny", dict(V=777, r=48, Bk=6, k=5, N=40), 0.0),    # N > 32: 64-column tiles
    ("tiny", dict(V=777, r=48, Bk=6, k=5, N=40), 1.3),
    ("qwen3_4b", {}, 0.0),
    ("qwen3_8b", {}, 0.6),
]


# every case fits both ways of running the waves: one persistent launch, or
# one GEMM + frontier launch pair per wave
PATHS = ["persistent", "waves"]


@pytest.mark.parametrize("path", PATHS)
@pytest.mark.parametrize("name,over,temp", CASES)
@pytest.mark.parametrize("seed", [0, 1])
def test_tree_build_parity(name, over, temp, seed, path):
    w = make_workload(name, seed=seed, temp=temp, **over)
    tree = run_build(w, temp=temp, seed=w.philox_seed, path=path)
    for b in range(w.batch):
        compare_tree(w, tree, b, temp, w.philox_seed)


@pytest.mark.parametrize("path", PATHS)
@pytest.mark.parametrize("temp", [0.0, 1.0])
def test_batch_budgets_lambda_calibration(temp, path):
    w = make_workload("tiny", seed=3, batch=5, V=600, N=12, k=3, temp=temp)
    w.n_budget[:] = np.array([12, 1, 0, 7, 12], np.int32)
    w.k_req[:] = np.array([3, 3, 1, 2, 1], np.int32)
    w.lam[:] = np.array([0.0, 0.0, 0.0, 0.02, 1e-4], np.float32)
    w.calib = np.array([[0.5, -0.1], [1.5, 0.2], [1.0, 0.0], [0.8, -0.3]], np.float32)
    tree = run_build(w, temp=temp, path=path)
    for b in range(w.batch):
        compare_tree(w, tree, b, temp, w.philox_seed)


def test_persistent_build_rejects_what_it_cannot_hold():
    # batch * Nmax above 64 never runs persistently: forced, the call is refused
    w = make_workload("tiny", seed=0, batch=3, N=30)
    x = build_inputs(w)
    tree = dt.Tree.empty(w.batch, w.Nmax)
    ws = dt.workspace(dt.build_workspace_bytes(w.batch, w.Bk, w.V, w.r, w.k, w.Nmax))
    dt.set_build_path("persistent")
    try:
        with pytest.raises(dt.DtreeError) as e:
            dt.tree_build(x["block_logits"], x["markov_a"], x["markov_b"], x["root_token"],
                          x["n_budget"], x["lam"], k=w.k, Nmax=w.Nmax, temp=0.0, out=tree, ws=ws)
        assert e.value.code == dt._lib.DT_EUNSUPPORTED
    finally:
        dt.set_build_path("auto")
    tree = run_build(w, temp=0.0)   # "auto" runs it as waves
    for b in range(w.batch):
        compare_tree(w, tree, b, 0.0, 0)


@pytest.mark.parametrize("name", ["tiny", "qwen3_4b"])
def test_persistent_build_wait_runs_out(name):
    """A CTA that never reaches the first grid barrier: every wait gives up
    after the test's 1 ms limit, the call reports DT_ETIMEOUT, and the next
    build on the same stream and workspace is exact again."""
    w = make_workload(name, seed=2)
    x = build_inputs(w)
    tree = dt.Tree.empty(w.batch, w.Nmax)
    ws = dt.workspace(dt.build_workspace_bytes(w.batch, w.Bk, w.V, w.r, w.k, w.Nmax))
    args = (x["block_logits"], x["markov_a"], x["markov_b"], x["root_token"], x["n_budget"],
            x["lam"])
    dt.set_build_path("persistent")
    try:
        dt.set_build_wait_test(0, 1_000_000)
        dt.tree_build(*args, k=w.k, Nmax=w.Nmax, temp=0.0, out=tree, ws=ws)
        assert dt.read_status(ws) == dt._lib.DT_ETIMEOUT
        tree2 = dt.Tree.empty(w.batch, w.Nmax)
        dt.tree_build(*args, k=w.k, Nmax=w.Nmax, temp=0.0, out=tree2, ws=ws)
        assert dt.read_status(ws) == 0
    finally:
        dt.set_build_wait_test(-1, 0)
        dt.set_build_path("auto")
    compare_tree(w, tree2, 0, 0.0, 0)


def test_k1_is_greedy_chain_on_gpu():
    w = make_workload("qwen3_4b", seed=4, k=1, N=10)
    tree = run_build(w, temp=0.0)
    h = tree_to_host(tree, 0)
    assert h["n"] == w.Bk
    assert h["parents"].tolist() == list(range(-1, w.Bk - 1))
    compare_tree(w, tree, 0, 0.0, 0)


def test_rejects_bad_arguments_without_launch():
    w = make_workload("tiny", seed=0)
    x = build_inputs(w)
    tree = dt.Tree.empty(1, w.Nmax)
    ws = dt.workspace(dt.build_workspace_bytes(1, w.Bk, w.V, w.r, w.k, w.Nmax))
    with pytest.raises(dt.DtreeError) as e:
        dt.tree_build(x["block_logits"], x["markov_a"], x["markov_b"], x["root_token"],
                      x["n_budget"], x["lam"], k=w.k, Nmax=65, temp=0.0, out=tree, ws=ws)
    assert e.value.code == dt._lib.DT_EUNSUPPORTED
    with pytest.raises(dt.DtreeError) as e:
        dt.tree_build(x["block_logits"], x["markov_a"], x["markov_b"], x["root_token"],
                      x["n_budget"], x["lam"], k=w.k, Nmax=w.Nmax, temp=0.0, out=tree,
                      ws=ws[:100])
    assert e.value.code == dt._lib.DT_EWORKSPACE
    with pytest.raises(dt.DtreeError) as e:   # T > 0 needs draft_q
        dt.tree_build(x["block_logits"], x["markov_a"], x["markov_b"], x["root_token"],
                      x["n_budget"], x["lam"], k=w.k, Nmax=w.Nmax, temp=1.0, out=tree, ws=ws)
    assert e.value.code == dt._lib.DT_EINVAL


def test_device_range_check_sets_status():
    w = make_workload("tiny", seed=0)
    w.n_budget[:] = 99          # beyond Nmax: clamped on device, status reported
    tree = dt.Tree.empty(1, w.Nmax)
    x = build_inputs(w)
    ws = dt.workspace(dt.build_workspace_bytes(1, w.Bk, w.V, w.r, w.k, w.Nmax))
    dt.tree_build(x["block_logits"], x["markov_a"], x["markov_b"], x["root_token"],
                  x["n_budget"], x["lam"], k=w.k, Nmax=w.Nmax, temp=0.0, out=tree, ws=ws)
    assert dt.read_status(ws) == dt._lib.DT_EDEVICE
    assert int(tree.n_nodes[0]) == w.Nmax
