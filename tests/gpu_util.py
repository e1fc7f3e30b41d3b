"""Helpers shared by the GPU parity tests: move seeded workloads to the device
and run the library's calls on them."""
import math

import numpy as np
import torch

from gen import attention_inputs, target_rows

BF16 = torch.bfloat16


def dev(a, dtype=None):
    t = torch.from_numpy(np.ascontiguousarray(a)).cuda()
    return t.to(dtype) if dtype is not None else t


def build_inputs(w):
    import draft_tree_construction_markov_b200 as dt
    ldt = BF16 if w.logit_dtype == "bf16" else torch.float32
    return dict(
        block_logits=dev(w.L, ldt), markov_a=dev(w.A, BF16), markov_b=dev(w.Bt, BF16),
        root_token=dev(w.root), n_budget=dev(w.n_budget), lam=dev(w.lam),
        k_req=dev(w.k_req), calib=None if w.calib is None else dev(np.asarray(w.calib, np.float32)))


def run_build(w, temp=None, seed=None, offset=0, path="auto"):
    """Build the workload's trees; path selects how the waves run ("auto",
    "waves": one launch pair per wave, "persistent": one launch)."""
    import draft_tree_construction_markov_b200 as dt
    temp = w.temp if temp is None else temp
    x = build_inputs(w)
    tree = dt.Tree.empty(w.batch, w.Nmax, w.V, stochastic=temp > 0)
    ws = dt.workspace(dt.build_workspace_bytes(w.batch, w.Bk, w.V, w.r, w.k, w.Nmax))
    dt.set_build_path(path)
    try:
        dt.tree_build(x["block_logits"], x["markov_a"], x["markov_b"], x["root_token"],
                      x["n_budget"], x["lam"], k=w.k, Nmax=w.Nmax, temp=temp, out=tree, ws=ws,
                      calib=x["calib"], k_req=x["k_req"],
                      philox_seed=w.philox_seed if seed is None else seed, philox_offset=offset)
    finally:
        dt.set_build_path("auto")
    status = dt.read_status(ws)
    assert status == 0, f"device status {status}"
    return tree


def tree_to_host(tree, b):
    n = int(tree.n_nodes[b])
    g = lambda t: t[b, :n].cpu().numpy()
    return dict(n=n, tokens=g(tree.tokens), parents=g(tree.parents), depths=g(tree.depths),
                ranks=g(tree.ranks), keys=g(tree.keys),
                anc=g(tree.anc).astype(np.uint64))


def target_for_tree(w, b, depths, tokens, Nmax=None):
    """[Nmax+1, V] rows: root row then one per node (zero padding)."""
    Nmax = Nmax or w.Nmax
    d = np.concatenate([[0], depths]).astype(np.int64)
    p = np.concatenate([[w.root[b]], tokens]).astype(np.int64)
    rows = target_rows(w, b, d, p)
    out = np.zeros((Nmax + 1, w.V), np.float32)
    out[: rows.shape[0]] = rows
    return out


def attn_device_inputs(w, trees_nodes):
    """Per-request attention inputs packed for the C ABI."""
    qs, kps, vps, kts, vts = [], [], [], [], []
    for b in range(w.batch):
        q, kp, vp, kt, vt = attention_inputs(w, w.Nmax + 1, b)
        qs.append(q); kps.append(kp); vps.append(vp); kts.append(kt); vts.append(vt)
    dt_ = BF16 if w.attn_dtype == "bf16" else torch.float32
    starts = np.concatenate([[0], np.cumsum(w.prefix_len)[:-1]]).astype(np.int64)
    return dict(
        q=dev(np.stack(qs), dt_), k_tree=dev(np.stack(kts), dt_), v_tree=dev(np.stack(vts), dt_),
        k_prefix=dev(np.concatenate(kps), dt_), v_prefix=dev(np.concatenate(vps), dt_),
        prefix_start=dev(starts), prefix_len=dev(w.prefix_len.astype(np.int32)),
        host=(qs, kps, vps, kts, vts), scale=1.0 / math.sqrt(w.d))
