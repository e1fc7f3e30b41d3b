"""GPU parity of dt_calib_log and dt_calib_fit against the oracle
(oracle/calibration.py).

Logging is compared exactly on oracle-built trees and oracle walks.  The fit
is compared exactly on seeded samples; where a grid point differs, the test
requires the two points' oracle log-likelihoods to agree within 1e-9
relative (a tie up to fp64 rounding, both maxima are correct).  An
end-to-end case logs and fits rounds the library built and walked itself.
"""
import numpy as np
import pytest
import torch

from gen import make_workload, target_rows
from oracle import accept, calibration, markov_tree

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import draft_tree_construction_markov_b200 as dt
    from draft_tree_construction_markov_b200 import _lib
    from tests.gpu_util import BF16, dev, run_build, target_for_tree

GRID = (0.0, 1 / 16, 33, -1.0, 1 / 16, 25)


def _gpu_fit(depth, ell, y, Bk, grid=GRID, min_samples=1):
    cal = torch.empty(Bk, 2, dtype=torch.float32, device="cuda")
    ll = torch.empty(Bk, dtype=torch.float64, device="cuda")
    ws = dt.workspace(dt.calib_workspace_bytes(Bk, grid[2], grid[5]))
    dt.calib_fit(dev(np.asarray(depth, np.int32)), dev(np.asarray(ell, np.float32)),
                 dev(np.asarray(y, np.int8)), Bk, grid, cal, ws, loglik=ll,
                 min_samples=min_samples)
    assert dt.read_status(ws) == 0
    return cal.cpu().numpy(), ll.cpu().numpy()


def _check_fit(depth, ell, y, Bk, grid=GRID, min_samples=1):
    got, got_ll = _gpu_fit(depth, ell, y, Bk, grid, min_samples)
    want, want_ll = calibration.fit(depth, ell, y, Bk, *grid, min_samples=min_samples)
    for d in range(Bk):
        if np.isnan(want_ll[d]):
            assert np.isnan(got_ll[d]) and got[d].tolist() == [1.0, 0.0]
            continue
        m = np.asarray(depth) == d + 1
        if not np.array_equal(got[d], want[d].astype(np.float32)):
            # both points must be maxima up to fp64 rounding
            at = calibration.log_likelihood(float(got[d, 0]), float(got[d, 1]),
                                            np.asarray(ell)[m], np.asarray(y)[m])
            assert abs(at - want_ll[d]) <= 1e-9 * max(1.0, abs(want_ll[d])), (d, got[d], want[d])
        if np.isfinite(want_ll[d]):
            assert abs(got_ll[d] - want_ll[d]) <= 1e-9 * max(1.0, abs(want_ll[d]))


@pytest.mark.parametrize("seed,n,Bk,min_samples", [(0, 500, 3, 1), (1, 5000, 7, 1),
                                                    (2, 20000, 16, 1), (3, 1, 2, 1),
                                                    (4, 3000, 16, 190)])
def test_fit_matches_oracle(seed, n, Bk, min_samples):
    g = np.random.default_rng(seed)
    depth = g.integers(0, Bk + 2, n).astype(np.int32)   # includes ignored depths 0, Bk+1
    a_true = g.uniform(0.3, 1.8, Bk + 2)
    b_true = g.uniform(-0.8, 0.3, Bk + 2)
    ell = g.uniform(-6, 0, n).astype(np.float32)
    p = np.exp(np.minimum(0, a_true[depth] * ell + b_true[depth]))
    y = (g.random(n) < p).astype(np.int8)
    _check_fit(depth, ell, y, Bk, min_samples=min_samples)


def test_fit_degenerate_outcomes():
    ell = np.linspace(-3, 0, 300).astype(np.float32)
    depth = np.concatenate([np.ones(150, np.int32), np.full(150, 2, np.int32)])
    y = np.concatenate([np.ones(150, np.int8), np.zeros(150, np.int8)])
    _check_fit(depth, ell, y, 4)              # depth 3, 4 without samples
    _check_fit(np.zeros(0, np.int32), np.zeros(0, np.float32), np.zeros(0, np.int8), 2)


def _oracle_rounds(w):
    trees, paths, rows = [], [], []
    for b in range(w.batch):
        t = markov_tree.build_tree(w.L[b], w.A, w.Bt, int(w.root[b]), w.k, w.Nmax)
        r = target_for_tree(w, b, t.depths, t.tokens)
        path, _ = accept.greedy_walk(t, r[: t.n + 1].astype(np.float64))
        trees.append(t)
        paths.append(path)
        rows.append(r)
    return trees, paths, np.stack(rows)


def test_log_matches_oracle_on_oracle_trees():
    w = make_workload("tiny", seed=6, batch=8, N=16, k=3, sigma_ab=0.35)
    trees, paths, _ = _oracle_rounds(w)
    tree = dt.Tree.empty(w.batch, w.Nmax)
    acc = torch.full((w.batch, w.Bk), -1, dtype=torch.int32, device="cuda")
    nacc = torch.zeros(w.batch, dtype=torch.int32, device="cuda")
    for b, (t, pth) in enumerate(zip(trees, paths)):
        for nm in ("tokens", "parents", "depths", "ranks"):
            getattr(tree, nm)[b, : t.n] = torch.from_numpy(getattr(t, nm).astype(np.int32))
        tree.keys[b, : t.n] = torch.from_numpy(t.keys)
        tree.n_nodes[b] = t.n
        acc[b, : len(pth)] = torch.tensor(pth, dtype=torch.int32)
        nacc[b] = len(pth)
    depth = torch.empty(w.batch, w.Nmax, dtype=torch.int32, device="cuda")
    ell = torch.empty(w.batch, w.Nmax, dtype=torch.float32, device="cuda")
    y = torch.empty(w.batch, w.Nmax, dtype=torch.int8, device="cuda")
    ws = dt.workspace(dt.calib_workspace_bytes())
    dt.calib_log(tree, acc, nacc, w.Bk, depth, ell, y, ws)
    assert dt.read_status(ws) == 0
    for b, (t, pth) in enumerate(zip(trees, paths)):
        dd, ll, yy = calibration.log_pairs(t, pth)
        assert np.array_equal(depth[b, : t.n].cpu().numpy(), dd)
        assert np.array_equal(ell[b, : t.n].cpu().numpy().view(np.uint32), ll.view(np.uint32))
        assert np.array_equal(y[b, : t.n].cpu().numpy(), yy)
        assert (depth[b, t.n:].cpu().numpy() == -1).all()


def test_log_and_fit_end_to_end():
    w = make_workload("qwen3_4b", seed=7, V=4096, batch=32, Bk=7, N=32, sigma_ab=0.35)
    tree = run_build(w, temp=0.0)
    trees, paths, rows = _oracle_rounds(w)
    for b, t in enumerate(trees):
        assert int(tree.n_nodes[b]) == t.n
        assert np.array_equal(tree.tokens[b, : t.n].cpu().numpy(), t.tokens)
    acc = torch.empty(w.batch, w.Bk, dtype=torch.int32, device="cuda")
    nacc = torch.empty(w.batch, dtype=torch.int32, device="cuda")
    bonus = torch.empty(w.batch, dtype=torch.int32, device="cuda")
    ws_a = dt.workspace(dt.accept_workspace_bytes(w.batch, w.Nmax, w.V))
    dt.tree_accept(dev(rows, BF16), tree, w.Bk, 0.0, acc, nacc, bonus, ws_a)
    assert dt.read_status(ws_a) == 0
    depth = torch.empty(w.batch, w.Nmax, dtype=torch.int32, device="cuda")
    ell = torch.empty(w.batch, w.Nmax, dtype=torch.float32, device="cuda")
    y = torch.empty(w.batch, w.Nmax, dtype=torch.int8, device="cuda")
    ws = dt.workspace(dt.calib_workspace_bytes(w.Bk, GRID[2], GRID[5]))
    dt.calib_log(tree, acc, nacc, w.Bk, depth, ell, y, ws)
    assert dt.read_status(ws) == 0
    od, ol, oy = [], [], []
    for b, (t, pth) in enumerate(zip(trees, paths)):
        assert nacc[b].item() == len(pth)
        dd, ll, yy = calibration.log_pairs(t, pth)
        assert np.array_equal(depth[b, : t.n].cpu().numpy(), dd)
        assert np.array_equal(y[b, : t.n].cpu().numpy(), yy)
        np.testing.assert_allclose(ell[b, : t.n].cpu().numpy(), ll, rtol=0, atol=1e-5)
        od.append(dd); ol.append(ll); oy.append(yy)
    cal = torch.empty(w.Bk, 2, dtype=torch.float32, device="cuda")
    ll_gpu = torch.empty(w.Bk, dtype=torch.float64, device="cuda")
    dt.calib_fit(depth.reshape(-1), ell.reshape(-1), y.reshape(-1), w.Bk, GRID, cal, ws,
                 loglik=ll_gpu)
    assert dt.read_status(ws) == 0
    od, ol, oy = np.concatenate(od), np.concatenate(ol), np.concatenate(oy)
    want, want_ll = calibration.fit(od, ol, oy, w.Bk, *GRID)
    got = cal.cpu().numpy()
    for d in range(w.Bk):
        if np.isnan(want_ll[d]):
            assert got[d].tolist() == [1.0, 0.0]
            continue
        m = od == d + 1
        at = calibration.log_likelihood(float(got[d, 0]), float(got[d, 1]), ol[m], oy[m])
        # the GPU fitted l values within 1e-5 of the oracle's: its point is a
        # maximum of the oracle's likelihood up to that perturbation
        assert at >= want_ll[d] - 1e-3 * max(1.0, abs(want_ll[d]))


def test_calib_argument_checks():
    ws = dt.workspace(dt.calib_workspace_bytes(2, 4, 4))
    cal = torch.empty(2, 2, dtype=torch.float32, device="cuda")
    z = lambda tt: torch.zeros(4, dtype=tt, device="cuda")
    with pytest.raises(_lib.DtreeError) as e:
        dt.calib_fit(z(torch.int32), z(torch.float32), z(torch.int8), 2, (-1.0, 0.1, 4, 0, 0.1, 4),
                     cal, ws)
    assert e.value.code == _lib.DT_EINVAL
    with pytest.raises(_lib.DtreeError) as e:
        dt.calib_fit(z(torch.int32), z(torch.float32), z(torch.int8), 2, (0, 0.1, 2048, 0, 0.1, 1024),
                     cal, ws)
    assert e.value.code == _lib.DT_EUNSUPPORTED
    with pytest.raises(_lib.DtreeError) as e:
        dt.calib_fit(z(torch.int32), z(torch.float32), z(torch.int8), 2, (0, 0.1, 64, 0, 0.1, 64),
                     cal, ws)
    assert e.value.code == _lib.DT_EWORKSPACE
