"""GPU parity of tree_accept and tree_verify_attn against the CPU oracle, plus
the sampling-distribution test over 1e6 seeded rounds."""
import math

import numpy as np
import pytest
import scipy.stats
import torch

from gen import make_workload, target_rows
from oracle import accept, markov_tree, verify_attn

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import draft_tree_construction_markov_b200 as dt
    from tests.gpu_util import (BF16, attn_device_inputs, build_inputs, dev, run_build,
                                target_for_tree, tree_to_host)


def _accept_gpu(w, tree, tgt, temp, seed, offset=0):
    acc = torch.empty(w.batch, w.Bk, dtype=torch.int32, device="cuda")
    nacc = torch.empty(w.batch, dtype=torch.int32, device="cuda")
    bonus = torch.empty(w.batch, dtype=torch.int32, device="cuda")
    ws = dt.workspace(dt.accept_workspace_bytes(w.batch, w.Nmax, w.V))
    dt.tree_accept(tgt, tree, w.Bk, temp, acc, nacc, bonus, ws, philox_seed=seed,
                   philox_offset=offset)
    assert dt.read_status(ws) == 0
    return acc.cpu().numpy(), nacc.cpu().numpy(), bonus.cpu().numpy()


ACCEPT_CASES = [
    ("tiny", {}, 0.0),
    ("tiny", {}, 1.0),
    ("tiny", dict(V=1000, r=32, Bk=5, k=3, N=20), 0.7),
    ("tiny", dict(V=1000, r=32, Bk=5, k=3, N=20, batch=3), 2.0),
    ("tiny", dict(V=777, r=48, Bk=6, k=5, N=40), 1.3),  # V % 4 != 0: the walk's scalar path
    ("qwen3_4b", {}, 0.0),
    ("qwen3_8b", {}, 0.6),
]


@pytest.mark.parametrize("name,over,temp", ACCEPT_CASES)
@pytest.mark.parametrize("seed", [0, 1, 2])
def test_accept_parity(name, over, temp, seed):
    w = make_workload(name, seed=seed, temp=temp, **over)
    tree = run_build(w, temp=temp)
    rows = []
    otrees = []
    for b in range(w.batch):
        o = markov_tree.build_tree(w.L[b], w.A, w.Bt, int(w.root[b]), int(w.k_req[b]),
                                   int(w.n_budget[b]), temp=temp, seed=w.philox_seed, request=b)
        h = tree_to_host(tree, b)
        assert np.array_equal(h["tokens"], o.tokens) and np.array_equal(h["parents"], o.parents)
        otrees.append(o)
        rows.append(target_for_tree(w, b, o.depths, o.tokens))
    tdt = BF16 if w.logit_dtype == "bf16" else torch.float32
    tgt = dev(np.stack(rows), tdt)
    acc, nacc, bonus = _accept_gpu(w, tree, tgt, temp, seed=77, offset=5)
    for b, o in enumerate(otrees):
        r = rows[b][: o.n + 1].astype(np.float64)
        margins = []
        if temp == 0:
            path, bon = accept.greedy_walk(o, r)
        else:
            path, bon = accept.stochastic_walk(o, r, temp, seed=77, offset=5, request=b,
                                               margins=margins)
        near = [m for m in margins if m[1] < 1e-5]
        assert nacc[b] == len(path), (b, near)
        assert acc[b, : nacc[b]].tolist() == path, (b, near)
        assert np.all(acc[b, nacc[b]:] == -1)
        assert bonus[b] == bon, (b, near)


def _attn_case(w, temp=0.0):
    tree = run_build(w, temp=temp)
    x = attn_device_inputs(w, None)
    out = torch.zeros_like(x["q"])
    ws = dt.workspace(dt.verify_workspace_bytes(w.batch, w.Nmax, w.Hq, w.Hkv, w.d,
                                                int(w.prefix_len.max())))
    dt.tree_verify_attn(x["q"], x["k_prefix"], x["v_prefix"], x["prefix_start"], x["prefix_len"],
                        int(w.prefix_len.max()), x["k_tree"], x["v_tree"], tree.anc,
                        tree.n_nodes, x["scale"], out, ws)
    assert dt.read_status(ws) == 0
    got = out.float().cpu().numpy()
    qs, kps, vps, kts, vts = x["host"]
    for b in range(w.batch):
        h = tree_to_host(tree, b)
        ref = verify_attn.tree_attention(qs[b], kps[b], vps[b], kts[b], vts[b], h["anc"], h["n"],
                                         x["scale"])
        tol = 2e-2 if w.attn_dtype == "bf16" else 1e-4
        np.testing.assert_allclose(got[b, : h["n"] + 1], ref, atol=tol, rtol=0)


@pytest.mark.parametrize("name,over", [
    ("tiny", {}),
    ("tiny", dict(V=600, N=20, P=100, attn_dtype="bf16")),
    ("tiny", dict(V=600, N=20, P=77, Hq=8, Hkv=2, d=128, attn_dtype="bf16", batch=3)),
    ("qwen3_4b", {}),
    ("qwen3_8b", dict(temp=0.0)),
])
def test_verify_attn_parity(name, over):
    w = make_workload(name, seed=2, **over)
    _attn_case(w)


def test_verify_attn_ragged_prefixes():
    w = make_workload("tiny", seed=5, V=600, N=16, P=300, Hq=8, Hkv=2, d=64,
                      attn_dtype="bf16", batch=4)
    w.prefix_len[:] = np.array([1, 300, 129, 64], np.int32)
    _attn_case(w)


@pytest.mark.parametrize("temp", [0.6, 1.0, 2.0])
def test_emitted_tokens_follow_target_chi_square(temp):
    """1e6 seeded rounds of the V=512 toy configuration on the GPU.

    The first emitted token must follow softmax(t_root / T), and the token
    after an accepted first node c must follow softmax(t_c / T) (chi-square,
    p > 0.01).  Rounds are independent requests and Philox offsets.
    """
    B = 1024
    calls = 977
    w = make_workload("tiny", seed=9, batch=B, temp=temp)
    # every request gets the same drafter inputs; randomness differs by request
    # index and offset
    w.L[:] = w.L[0]
    w.root[:] = w.root[0]
    x = build_inputs(w)
    # synthetic target, first order: table over (depth, previous token)
    V, Bk = w.V, w.Bk
    tab = np.zeros((Bk + 1, V, V), np.float32)
    for d in range(Bk + 1):
        tab[d] = target_rows(w, 0, np.full(V, d), np.arange(V))
    tab_d = dev(tab)
    tree = dt.Tree.empty(B, w.Nmax, V, stochastic=True)
    ws = dt.workspace(dt.build_workspace_bytes(B, w.Bk, V, w.r, w.k, w.Nmax))
    wsa = dt.workspace(dt.accept_workspace_bytes(B, w.Nmax, V))
    acc = torch.empty(B, Bk, dtype=torch.int32, device="cuda")
    nacc = torch.empty(B, dtype=torch.int32, device="cuda")
    bonus = torch.empty(B, dtype=torch.int32, device="cuda")
    root = int(w.root[0])
    first = torch.zeros(V, dtype=torch.int64, device="cuda")
    second = {}
    ar = torch.arange(w.Nmax, device="cuda")
    for call in range(calls):
        dt.tree_build(x["block_logits"], x["markov_a"], x["markov_b"], x["root_token"],
                      x["n_budget"], x["lam"], k=w.k, Nmax=w.Nmax, temp=temp, out=tree, ws=ws,
                      philox_seed=1234, philox_offset=call)
        n = tree.n_nodes.long()
        valid = ar[None, :] < n[:, None]
        dep = torch.where(valid, tree.depths.long(), 0)
        tok = torch.where(valid, tree.tokens.long(), 0)
        tgt = torch.empty(B, w.Nmax + 1, V, device="cuda")
        tgt[:, 0] = tab_d[0, root]
        tgt[:, 1:] = tab_d[dep, tok]
        dt.tree_accept(tgt, tree, Bk, temp, acc, nacc, bonus, wsa, philox_seed=99,
                       philox_offset=call)
        first_node = acc[:, 0].long()
        tok0 = torch.where(nacc > 0, tree.tokens.gather(1, first_node.clamp(min=0)[:, None])[:, 0],
                           bonus).long()
        first += torch.bincount(tok0, minlength=V)
        # second token given that the first node was accepted
        has2 = nacc > 0
        if has2.any():
            n2 = torch.where(nacc > 1,
                             tree.tokens.gather(1, acc[:, 1].long().clamp(min=0)[:, None])[:, 0],
                             bonus).long()
            pairs = tok0[has2] * V + n2[has2]
            cnt = torch.bincount(pairs, minlength=V * V)
            for key in torch.nonzero(cnt).flatten().tolist():
                second[key] = second.get(key, 0) + int(cnt[key])
    assert dt.read_status(ws) == 0 and dt.read_status(wsa) == 0

    def chi(obs, p):
        obs = np.asarray(obs, np.float64)
        exp_ = obs.sum() * p
        big = exp_ >= 5
        o = np.append(obs[big], obs[~big].sum())
        e = np.append(exp_[big], exp_[~big].sum())
        keep = e > 0
        return scipy.stats.chisquare(o[keep], e[keep] * o[keep].sum() / e[keep].sum()).pvalue

    p0 = accept.softmax(tab[0, root].astype(np.float64) / temp)
    assert chi(first.cpu().numpy(), p0) > 0.01
    # conditional of the second token after the most frequent accepted first token
    by_first = {}
    for key, c in second.items():
        by_first.setdefault(key // V, np.zeros(V))[key % V] += c
    y1 = max(by_first, key=lambda y: by_first[y].sum())
    assert by_first[y1].sum() > 10000
    p1 = accept.softmax(tab[1, y1].astype(np.float64) / temp)
    assert chi(by_first[y1], p1) > 0.01


def test_stochastic_walk_wide_node():
    """A node with 40 children, more rejected siblings than any build emits.

    The walk keeps the whole removed-sibling set (up to Nmax - 1 tokens) and
    its residuals stay those of the oracle: requests 0-2 reject all 40
    children, requests 3-5 reject 30 and accept the 31st.
    """
    B, V, Nmax, nk, Bk, temp = 6, 20000, 48, 40, 2, 1.0
    rng = np.random.default_rng(41)
    tokens = np.stack([rng.choice(V, nk, replace=False) for _ in range(B)]).astype(np.int32)
    t = np.zeros((B, Nmax + 1, V), np.float32)
    q = np.zeros((B, Nmax + 1, V), np.float32)
    for b in range(B):
        t[b, : nk + 1] = rng.standard_normal((nk + 1, V))
        t[b, 0, tokens[b]] = -30.0
        if b >= 3:
            t[b, 0, tokens[b, 30]] = 12.0
        q0 = np.full(V, 0.7 / (V - nk))
        q0[tokens[b]] = 0.3 / nk
        q[b, 0] = (q0 / q0.sum()).astype(np.float32)
    tree = dt.Tree.empty(B, Nmax, V, stochastic=True)
    pad = np.zeros((B, Nmax), np.int32)
    tok = pad.copy()
    tok[:, :nk] = tokens
    par = np.full((B, Nmax), -1, np.int32)
    dep = pad.copy()
    dep[:, :nk] = 1
    rnk = pad.copy()
    rnk[:, :nk] = np.arange(nk)
    tree.tokens.copy_(torch.from_numpy(tok))
    tree.parents.copy_(torch.from_numpy(par))
    tree.depths.copy_(torch.from_numpy(dep))
    tree.ranks.copy_(torch.from_numpy(rnk))
    tree.n_nodes.fill_(nk)
    tree.draft_q.copy_(torch.from_numpy(q))
    acc = torch.empty(B, Bk, dtype=torch.int32, device="cuda")
    nacc = torch.empty(B, dtype=torch.int32, device="cuda")
    bonus = torch.empty(B, dtype=torch.int32, device="cuda")
    ws = dt.workspace(dt.accept_workspace_bytes(B, Nmax, V))
    dt.tree_accept(dev(t), tree, Bk, temp, acc, nacc, bonus, ws, philox_seed=5, philox_offset=2)
    assert dt.read_status(ws) == 0
    acc, nacc, bonus = acc.cpu().numpy(), nacc.cpu().numpy(), bonus.cpu().numpy()
    compared = 0
    for b in range(B):
        o = markov_tree.Tree(
            tokens=tokens[b], parents=np.full(nk, -1, np.int32), depths=np.ones(nk, np.int32),
            ranks=np.arange(nk, dtype=np.int32), keys=np.zeros(nk, np.float32),
            keys64=np.zeros(nk), anc=(np.uint64(1) << np.arange(nk, dtype=np.uint64)),
            expansions={}, margins=[])
        margins = []
        path, bon = accept.stochastic_walk(o, t[b, : nk + 1].astype(np.float64), temp, seed=5,
                                           offset=2, request=b, q_rows={0: q[b, 0]},
                                           margins=margins)
        assert path == ([] if b < 3 else [30]), (b, path)
        if min(m[1] for m in margins) < 1e-4:
            continue  # a coin or race within fp32 rounding of its threshold
        compared += 1
        assert nacc[b] == len(path) and acc[b, : nacc[b]].tolist() == path, b
        assert np.all(acc[b, nacc[b]:] == -1)
        assert bonus[b] == bon, b
    assert compared >= 4
