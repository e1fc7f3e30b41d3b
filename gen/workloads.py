"""Seeded synthetic workloads for one draft-tree decode round.

The source pages measure on Qwen3 targets with DSpark / DFlash drafters and a
set of public benchmarks (PCTree summary, "setup" paragraph; TreeFlash
explainer, "experiments").  None of those models or datasets is available, so
every input here is synthetic: only the shapes (vocabulary 151936, 32 query /
8 KV heads, head dim 128, hidden 2560) and the structure of a drafter block
(a confident early position whose margin decays with depth) are kept.

Exactness rule.  The Markov factors are drawn on the dyadic grid 2^-7 and
clipped to +-1.5, and bf16 block logits are snapped to the grid 2^-14, so
that the drafter logits z = L + A[prev] . B^T are exact in fp32 whatever the
summation order (products are multiples of 2^-14, partial sums stay below
2^10).  Integer decisions that depend only on z (top-k, greedy argmax of the
target) are therefore identical on any correct implementation.

Nothing in this module applies the method (no softmax, top-k, tree search,
attention or acceptance).  The one matrix product it contains is the
synthetic *target model* of the configurations ("target = draft + noise"),
which stands in for the Qwen3 verifier's LM head.
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import numpy as np

__all__ = [
    "CONFIGS", "Workload", "make_workload", "bf16_round", "to_bf16_bits",
    "target_rows", "attention_inputs", "treeflash_inputs", "rng",
]

# ---------------------------------------------------------------------------
# configuration table (names describe the workload, sizes are the full sizes)
# ---------------------------------------------------------------------------
CONFIGS = {
    # V=512 toy round: fp32 logits, Markov head N(0,0.1), planted token +6,
    # target = draft + N(0,1), 32-token prefix, 2q/2kv heads, d=64.
    "tiny": dict(V=512, Bk=4, k=2, N=8, r=16, sigma_ab=0.1, logit_dtype="f32",
                 L_scale=2.0, plant=("add", 6.0, 6.0), target_sigma=1.0,
                 P=32, Hq=2, Hkv=2, d=64, attn_dtype="f32", batch=1,
                 temp=0.0, lam=0.0),
    # Qwen3-4B-shaped round: B=7, k=4, N=32, r=256, prefix 2048, greedy.
    "qwen3_4b": dict(V=151936, Bk=7, k=4, N=32, r=256, sigma_ab=0.25,
                     logit_dtype="bf16", L_scale=3.0, plant=("margin", 8.0, 2.0),
                     target_sigma=1.0, P=2048, Hq=32, Hkv=8, d=128,
                     attn_dtype="bf16", batch=1, temp=0.0, lam=0.0),
    # Qwen3-8B-shaped round: B=16, k=4, N=64, prefix 4096, T=0.6 stochastic.
    "qwen3_8b": dict(V=151936, Bk=16, k=4, N=64, r=256, sigma_ab=0.25,
                     logit_dtype="bf16", L_scale=3.0, plant=("margin", 8.0, 2.0),
                     target_sigma=1.2, P=4096, Hq=32, Hkv=8, d=128,
                     attn_dtype="bf16", batch=1, temp=0.6, lam=0.0),
    # Acceptance study of the baseline trees: the Qwen3-8B-shaped block
    # (B=16, k=4, N=32, greedy) with a stronger Markov term (sigma 0.35, so
    # the next token depends on the parent more than in the rounds above),
    # 64 requests, 1024-token prefixes.
    "acceptance_study": dict(V=151936, Bk=16, k=4, N=32, r=256, sigma_ab=0.35,
                             logit_dtype="bf16", L_scale=3.0, plant=("margin", 8.0, 2.0),
                             target_sigma=1.0, P=1024, Hq=32, Hkv=8, d=128,
                             attn_dtype="bf16", batch=64, temp=0.0, lam=0.0),
    # Load sweep of the load-adaptive tree size: the acceptance-study block
    # with lognormal prefixes clipped to [512, 8192] (the load-adaptive
    # recipe); every request asks for the full N = 32 tree.
    "load_sweep": dict(V=151936, Bk=16, k=4, N=32, r=256, sigma_ab=0.35,
                       logit_dtype="bf16", L_scale=3.0, plant=("margin", 8.0, 2.0),
                       target_sigma=1.0, P=8192, Hq=32, Hkv=8, d=128,
                       attn_dtype="bf16", batch=64, temp=0.0, lam=0.0, ragged_prefix=True),
    # Load-adaptive batch: 64 requests, lognormal prefixes clipped to
    # [512, 8192], per-request budget from {chain, 8, 16, 32}, lambda 0.01, T=1.
    "load_adaptive": dict(V=151936, Bk=7, k=4, N=32, r=256, sigma_ab=0.25,
                          logit_dtype="bf16", L_scale=3.0,
                          plant=("margin", 8.0, 2.0), target_sigma=1.0,
                          P=8192, Hq=32, Hkv=8, d=128, attn_dtype="bf16",
                          batch=64, temp=1.0, lam=0.01, ragged=True),
}


def rng(*key: int) -> np.random.Generator:
    """Independent PCG64 stream for a tuple of non-negative integers."""
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence(list(key))))


# tags that keep the streams of different arrays apart
_T_MARKOV, _T_BLOCK, _T_Q, _T_KVP, _T_KVT, _T_TGT, _T_META, _T_TF = range(1, 9)


def bf16_round(x: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bf16 (ties to even), kept as float32."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) & 0xFFFF0000
    return u.astype(np.uint32).view(np.float32)


def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """uint16 bit patterns of bf16-exact float32 values."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    if np.any(u & 0xFFFF):
        raise ValueError("values are not bf16-exact")
    return (u >> 16).astype(np.uint16)


def _dyadic(x: np.ndarray, bits: int) -> np.ndarray:
    s = float(2 ** bits)
    return (np.round(x * s) / s).astype(np.float32)


@dataclasses.dataclass
class Workload:
    name: str
    V: int
    Bk: int
    k: int                     # largest children-per-node over the batch
    Nmax: int
    r: int
    batch: int
    temp: float
    L: np.ndarray              # (batch, Bk, V) float32 (bf16-exact if bf16)
    logit_dtype: str           # "f32" | "bf16"
    A: np.ndarray              # (V, r) float32, bf16-exact, dyadic 2^-7
    Bt: np.ndarray             # (V, r) float32, bf16-exact, dyadic 2^-7
    root: np.ndarray           # (batch,) int32
    n_budget: np.ndarray       # (batch,) int32
    k_req: np.ndarray          # (batch,) int32
    lam: np.ndarray            # (batch,) float32
    calib: Optional[np.ndarray]  # (Bk, 2) float32 (alpha, beta) per child depth
    seed: int
    target_sigma: float
    Lt: np.ndarray             # (batch, Bk+1, V) target block rows (float32)
    prefix_len: np.ndarray     # (batch,) int32
    P: int
    Hq: int
    Hkv: int
    d: int
    attn_dtype: str
    philox_seed: int = 0x243F6A8885A308D3
    philox_offset: int = 0


def _block_logits(g, Bk, V, scale, plant, dtype, dyadic=True):
    L = (scale * g.standard_normal((Bk, V))).astype(np.float32)
    planted = g.integers(0, V, size=Bk)
    kind, m0, m1 = plant
    for d in range(Bk):
        if kind == "add":
            L[d, planted[d]] += np.float32(m0)
        else:  # margin over the best other token, decaying linearly with depth
            m = m0 + (m1 - m0) * (d / max(Bk - 1, 1))
            others = np.delete(L[d], planted[d])
            L[d, planted[d]] = np.float32(others.max() + m)
    if dtype == "bf16":
        L = _dyadic(bf16_round(L), 14) if dyadic else bf16_round(L)
    else:
        L = _dyadic(L, 10) if dyadic else L
    return L


def make_workload(name: str, seed: int = 0, dyadic: bool = True, **over) -> Workload:
    """Draw the inputs of one round of configuration ``name`` (sizes overridable).

    ``dyadic=False`` keeps the Markov factors and block logits as plain bf16
    values (no snapping to the dyadic grids): the drafter logits are then no
    longer exact in fp32, and integer decisions must be compared only where
    their margins are well above fp32 rounding.
    """
    c = dict(CONFIGS[name])
    c.update(over)
    V, Bk, r, batch = c["V"], c["Bk"], c["r"], c["batch"]
    g = rng(seed, _T_MARKOV)
    sab = c["sigma_ab"]
    if dyadic:
        A = _dyadic(np.clip(sab * g.standard_normal((V, r)), -1.5, 1.5), 7)
        Bt = _dyadic(np.clip(sab * g.standard_normal((V, r)), -1.5, 1.5), 7)
    else:
        A = bf16_round((sab * g.standard_normal((V, r))).astype(np.float32))
        Bt = bf16_round((sab * g.standard_normal((V, r))).astype(np.float32))
    L = np.empty((batch, Bk, V), np.float32)
    Lt = np.empty((batch, Bk + 1, V), np.float32)
    for b in range(batch):
        gb = rng(seed, _T_BLOCK, b)
        L[b] = _block_logits(gb, Bk, V, c["L_scale"], c["plant"], c["logit_dtype"], dyadic)
        Lt[b, :Bk] = L[b]
        extra = (c["L_scale"] * gb.standard_normal(V)).astype(np.float32)
        Lt[b, Bk] = _dyadic(bf16_round(extra), 14) if c["logit_dtype"] == "bf16" else _dyadic(extra, 10)
    gm = rng(seed, _T_META)
    root = gm.integers(0, V, size=batch).astype(np.int32)
    N, k = c["N"], c["k"]
    if c.get("ragged_prefix"):
        # lognormal prefixes only (same recipe as the load-adaptive batch)
        plen_r = np.clip(np.round(1024.0 * np.exp(0.7 * gm.standard_normal(batch))),
                         512, c["P"]).astype(np.int32)
    if c.get("ragged"):
        # per-request budget drawn from {chain, 8, 16, 32}; chain = k 1, N = Bk
        choice = gm.integers(0, 4, size=batch)
        n_budget = np.array([Bk, 8, 16, 32], np.int32)[choice]
        k_req = np.where(choice == 0, 1, k).astype(np.int32)
        plen = np.clip(np.round(1024.0 * np.exp(0.7 * gm.standard_normal(batch))),
                       512, c["P"]).astype(np.int32)
        Nmax = int(max(n_budget.max(), N))
    else:
        n_budget = np.full(batch, N, np.int32)
        k_req = np.full(batch, k, np.int32)
        plen = plen_r if c.get("ragged_prefix") else np.full(batch, c["P"], np.int32)
        Nmax = N
    lam = np.full(batch, c["lam"], np.float32)
    return Workload(
        name=name, V=V, Bk=Bk, k=k, Nmax=Nmax, r=r, batch=batch,
        temp=float(c["temp"]), L=L, logit_dtype=c["logit_dtype"], A=A, Bt=Bt,
        root=root, n_budget=n_budget, k_req=k_req, lam=lam,
        calib=c.get("calib"), seed=seed, target_sigma=float(c["target_sigma"]),
        Lt=Lt, prefix_len=plen, P=int(plen.max()), Hq=c["Hq"], Hkv=c["Hkv"],
        d=c["d"], attn_dtype=c["attn_dtype"],
    )


def target_rows(w: Workload, b: int, depths: np.ndarray, prevs: np.ndarray,
                out_dtype: str = None) -> np.ndarray:
    """Synthetic verifier logits for request ``b``.

    The stand-in target model is first order: the logits after a node at
    depth ``d`` whose token is ``prev`` are ``Lt[d] + A[prev] . Bt^T`` plus
    Gaussian noise of std ``target_sigma`` seeded by (seed, b, d, prev), i.e.
    "target = draft + N(0, sigma)" of the configuration table.  Being a fixed
    function of (depth, prev) it gives the same row to every round that
    reaches the same node, which the sampling-distribution tests rely on.
    Rows are returned as float32, rounded to bf16 for bf16 workloads.
    """
    depths = np.asarray(depths)
    prevs = np.asarray(prevs)
    out = np.empty((len(depths), w.V), np.float32)
    base = w.A[prevs].astype(np.float32) @ w.Bt.T.astype(np.float32)
    for i, (d, p) in enumerate(zip(depths.tolist(), prevs.tolist())):
        noise = rng(w.seed, _T_TGT, b, d, p).standard_normal(w.V).astype(np.float32)
        out[i] = w.Lt[b, d] + base[i] + np.float32(w.target_sigma) * noise
    dt = out_dtype or w.logit_dtype
    return bf16_round(out) if dt == "bf16" else out


def attention_inputs(w: Workload, n_rows: int, b: int):
    """q (n_rows,Hq,d), k/v prefix (P_b,Hkv,d), k/v tree (n_rows,Hkv,d): N(0,1).

    bf16 workloads get bf16-exact float32 values.  Per-request streams let a
    caller draw one request of a large batch on its own.
    """
    P = int(w.prefix_len[b])
    gq = rng(w.seed, _T_Q, b)
    gp = rng(w.seed, _T_KVP, b)
    gt = rng(w.seed, _T_KVT, b)
    q = gq.standard_normal((n_rows, w.Hq, w.d), dtype=np.float32)
    kp = gp.standard_normal((P, w.Hkv, w.d), dtype=np.float32)
    vp = gp.standard_normal((P, w.Hkv, w.d), dtype=np.float32)
    kt = gt.standard_normal((n_rows, w.Hkv, w.d), dtype=np.float32)
    vt = gt.standard_normal((n_rows, w.Hkv, w.d), dtype=np.float32)
    if w.attn_dtype == "bf16":
        q, kp, vp, kt, vt = (bf16_round(a) for a in (q, kp, vp, kt, vt))
    return q, kp, vp, kt, vt


def treeflash_inputs(seed: int = 0, V: int = 151936, D: int = 2560, Dff: int = 2560,
                     positions: int = 16, batch: int = 16):
    """Drafter hidden states and weights of the SwiGLU AR-approximator workload.

    h ~ N(0,1) per position, embedding E ~ N(0,0.02), gate/up/down and LM head
    ~ N(0, 1/fan_in), RMSNorm weights 1.  All bf16-exact float32 arrays.
    """
    g = rng(seed, _T_TF)
    f = lambda shape, std: bf16_round((std * g.standard_normal(shape)).astype(np.float32))
    return dict(
        h=f((batch, positions, D), 1.0),
        E=f((V, D), 0.02),
        w_norm_h=np.ones(D, np.float32),
        w_norm_e=np.ones(D, np.float32),
        W_gate=f((Dff, 2 * D), (2 * D) ** -0.5),
        W_up=f((Dff, 2 * D), (2 * D) ** -0.5),
        W_down=f((D, Dff), Dff ** -0.5),
        W_lm=f((V, D), D ** -0.5),
        root=g.integers(0, V, size=batch).astype(np.int32),
    )
