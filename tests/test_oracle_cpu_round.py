"""The multi-core C++ CPU baseline (oracle/cpu_round.cpp) against the numpy
oracle: the same greedy round (tree, attention rows, accept walk) on small
seeded workloads.  Tree structure and the accept path must be identical,
keys and attention rows equal up to fp64 summation order."""
import math

import numpy as np
import pytest

from gen import attention_inputs, make_workload, target_rows
from oracle import accept, cpu_round, markov_tree, verify_attn


@pytest.mark.parametrize("name,over", [
    ("tiny", {}),
    ("tiny", dict(V=1000, r=32, Bk=5, k=3, N=20, P=100)),
    ("tiny", dict(V=4096, r=64, Bk=6, k=4, N=32, P=300, Hq=8, Hkv=2, d=64)),
])
def test_cpu_round_equals_oracle(name, over):
    w = make_workload(name, seed=3, **over)
    o = markov_tree.build_tree(w.L[0], w.A, w.Bt, int(w.root[0]), w.k, w.Nmax, temp=0.0)
    attn = attention_inputs(w, w.Nmax + 1, 0)
    scale = 1.0 / math.sqrt(w.d)
    d = np.concatenate([[0], o.depths]).astype(np.int64)
    pv = np.concatenate([[w.root[0]], o.tokens]).astype(np.int64)
    tgt = np.zeros((w.Nmax + 1, w.V), np.float32)
    tgt[: o.n + 1] = target_rows(w, 0, d, pv)
    c = cpu_round.round_t0(w.L[0], w.A, w.Bt, w.root[0], w.k, w.Nmax, attn, scale, tgt)
    assert c["n"] == o.n
    assert np.array_equal(c["tokens"], o.tokens)
    assert np.array_equal(c["parents"], o.parents)
    assert np.array_equal(c["depths"], o.depths)
    np.testing.assert_allclose(c["keys"], o.keys64, rtol=1e-12, atol=1e-12)
    ref = verify_attn.tree_attention(*attn, o.anc, o.n, scale)
    np.testing.assert_allclose(c["attn"], ref, rtol=1e-10, atol=1e-10)
    path, bon = accept.greedy_walk(o, tgt[: o.n + 1].astype(np.float64))
    assert c["acc"].tolist() == list(path) and c["bonus"] == bon
