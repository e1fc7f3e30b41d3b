"""B200 (sm_100a) draft-tree round: tree_build, tree_verify_attn, tree_accept.

Thin Python surface over libdtree.so (see include/dtree.h for the exact
semantics, layouts and error behaviour of every call).  Tensors must be CUDA
tensors; the library allocates nothing, so each call takes a workspace tensor
(``workspace(...)`` allocates one of the right size).
"""
import ctypes
from dataclasses import dataclass
from typing import Optional

import torch

from . import _lib
from ._lib import DtreeError, check, dtype_code, ptr, stream_ptr

__all__ = ["Tree", "tree_build", "tree_verify_attn", "tree_accept", "markov_logits",
           "read_status", "build_workspace_bytes", "verify_workspace_bytes",
           "accept_workspace_bytes", "workspace", "DtreeError", "num_sms", "tree_load_budget",
           "load_budget_workspace_bytes", "calib_workspace_bytes", "calib_log", "calib_fit",
           "tree_accept_noalloc",
           "shard_range", "shard_cfg", "sharded_workspace_bytes", "sharded_partials_bytes",
           "sharded_build_begin", "sharded_build_gemm", "sharded_build_frontier",
           "tree_build_sharded", "set_build_path", "set_build_wait_test"]


def num_sms() -> int:
    return int(_lib.lib.dt_num_sms())


def workspace(nbytes: int, device="cuda") -> torch.Tensor:
    """Device scratch for one call site; its 256-byte header (the status word
    that read_status returns) starts cleared."""
    ws = torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)
    ws[:256].zero_()
    return ws


@dataclass
class Tree:
    """Device arrays of a batch of draft trees (dt_tree in the C header)."""
    tokens: torch.Tensor      # [batch, Nmax] int32
    parents: torch.Tensor     # [batch, Nmax] int32
    depths: torch.Tensor      # [batch, Nmax] int32
    ranks: torch.Tensor       # [batch, Nmax] int32
    keys: torch.Tensor        # [batch, Nmax] float32
    anc: torch.Tensor         # [batch, Nmax] int64 (uint64 bit patterns)
    n_nodes: torch.Tensor     # [batch] int32
    draft_q: Optional[torch.Tensor] = None   # [batch, Nmax+1, V] float32 (T > 0)

    @staticmethod
    def empty(batch, Nmax, V=None, stochastic=False, device="cuda"):
        i = dict(dtype=torch.int32, device=device)
        return Tree(
            tokens=torch.zeros(batch, Nmax, **i), parents=torch.zeros(batch, Nmax, **i),
            depths=torch.zeros(batch, Nmax, **i), ranks=torch.zeros(batch, Nmax, **i),
            keys=torch.zeros(batch, Nmax, dtype=torch.float32, device=device),
            anc=torch.zeros(batch, Nmax, dtype=torch.int64, device=device),
            n_nodes=torch.zeros(batch, **i),
            draft_q=(torch.zeros(batch, Nmax + 1, V, dtype=torch.float32, device=device)
                     if stochastic else None))

    def c_struct(self):
        return _lib.DtTree(*(ctypes.c_void_p(t.data_ptr()) if t is not None else None for t in
                             (self.tokens, self.parents, self.depths, self.ranks, self.keys,
                              self.anc, self.n_nodes, self.draft_q)))


def build_workspace_bytes(batch, Bk, V, r, k, Nmax) -> int:
    return int(_lib.lib.dt_tree_build_workspace_bytes(batch, Bk, V, r, k, Nmax))


def verify_workspace_bytes(batch, Nmax, Hq, Hkv, d, max_prefix) -> int:
    return int(_lib.lib.dt_tree_verify_attn_workspace_bytes(batch, Nmax, Hq, Hkv, d, max_prefix))


def accept_workspace_bytes(batch, Nmax, V) -> int:
    return int(_lib.lib.dt_tree_accept_workspace_bytes(batch, Nmax, V))


def tree_build(block_logits, markov_a, markov_b, root_token, n_budget, lam, *, k, Nmax, temp,
               out: Tree, ws, calib=None, k_req=None, philox_seed=0, philox_offset=0,
               stream=None, variant="pctree"):
    """dt_tree_build (variant "pctree") or dt_tree_build_ex with a baseline
    variant ("chain", "marginal", "shared_markov").  block_logits
    [batch,Bk,V] fp32|bf16; markov_a/markov_b [V,r] bf16."""
    batch, Bk, V = block_logits.shape
    r = markov_a.shape[1]
    st = out.c_struct()
    args = (ptr(block_logits), dtype_code(block_logits), ptr(markov_a), ptr(markov_b), r,
            ptr(calib), ptr(root_token), ptr(n_budget), ptr(k_req), ptr(lam), batch, Bk, V, k,
            Nmax, float(temp), philox_seed, philox_offset)
    tail = (ctypes.byref(st), ptr(ws), ws.numel(), stream_ptr(stream))
    if variant == "pctree":
        check(_lib.lib.dt_tree_build(*args, *tail), "dt_tree_build")
    else:
        check(_lib.lib.dt_tree_build_ex(*args, _lib.TREE_VARIANTS[variant], *tail),
              "dt_tree_build_ex")
    return out


def markov_logits(block_logits, markov_a, markov_b, req, depth, token, out, ws, stream=None):
    """dt_markov_logits: z rows [n_rows, V] fp32 for (request, depth, token) triples."""
    batch, Bk, V = block_logits.shape
    check(_lib.lib.dt_markov_logits(
        ptr(block_logits), dtype_code(block_logits), ptr(markov_a), ptr(markov_b),
        markov_a.shape[1], batch, Bk, V, ptr(req), ptr(depth), ptr(token), req.numel(), ptr(out),
        ptr(ws), ws.numel(), stream_ptr(stream)), "dt_markov_logits")
    return out


def tree_verify_attn(q, k_prefix, v_prefix, prefix_start, prefix_len, max_prefix, k_tree, v_tree,
                     anc, n_nodes, scale, out, ws, stream=None):
    """dt_tree_verify_attn.  q/out [batch,Nmax+1,Hq,d]; k/v_prefix [rows,Hkv,d]."""
    batch, n1, Hq, d = q.shape
    Hkv = k_prefix.shape[1]
    check(_lib.lib.dt_tree_verify_attn(
        ptr(q), ptr(k_prefix), ptr(v_prefix), ptr(prefix_start), ptr(prefix_len), int(max_prefix),
        ptr(k_tree), ptr(v_tree), ptr(anc), ptr(n_nodes), batch, n1 - 1, Hq, Hkv, d, float(scale),
        dtype_code(q), ptr(out), ptr(ws), ws.numel(), stream_ptr(stream)), "dt_tree_verify_attn")
    return out


def tree_accept(target_logits, tree: Tree, Bk, temp, acc_nodes, n_acc, bonus, ws,
                philox_seed=0, philox_offset=0, stream=None):
    """dt_tree_accept.  target_logits [batch,Nmax+1,V] fp32|bf16."""
    batch, n1, V = target_logits.shape
    st = tree.c_struct()
    check(_lib.lib.dt_tree_accept(
        ptr(target_logits), dtype_code(target_logits), ctypes.byref(st), batch, Bk, V, n1 - 1,
        float(temp), philox_seed, philox_offset, ptr(acc_nodes), ptr(n_acc), ptr(bonus), ptr(ws),
        ws.numel(), stream_ptr(stream)), "dt_tree_accept")
    return acc_nodes, n_acc, bonus


def tree_accept_noalloc(target_logits, tree: Tree, Bk, temp, acc_nodes, n_acc, bonus,
                        philox_seed=0, philox_offset=0, stream=None):
    """dt_tree_accept_noalloc: dt_tree_accept with the library's fixed scratch
    (no workspace; batch 1 at V = 151936 fits, larger sizes raise
    DT_EUNSUPPORTED)."""
    batch, n1, V = target_logits.shape
    st = tree.c_struct()
    check(_lib.lib.dt_tree_accept_noalloc(
        ptr(target_logits), dtype_code(target_logits), ctypes.byref(st), batch, Bk, V, n1 - 1,
        float(temp), philox_seed, philox_offset, ptr(acc_nodes), ptr(n_acc), ptr(bonus),
        stream_ptr(stream)), "dt_tree_accept_noalloc")
    return acc_nodes, n_acc, bonus


def treeflash_workspace_bytes(batch, gamma, D, Dff, V, M, budget) -> int:
    return int(_lib.lib.dt_treeflash_workspace_bytes(batch, gamma, D, Dff, V, M, budget))


def treeflash_build(h, embed, w_norm_h, w_norm_e, w_gate, w_up, w_down, w_lm, root, *, M,
                    budget, out: Tree, ws, stream=None):
    """dt_treeflash_build.  h [batch,gamma,D] bf16; embed/w_lm [V,D] bf16; w_gate/w_up
    [Dff,2D] bf16; w_down [D,Dff] bf16; w_norm_h/w_norm_e [D] fp32; root [batch] int32."""
    batch, gamma, D = h.shape
    V = w_lm.shape[0]
    Dff = w_gate.shape[0]
    st = out.c_struct()
    check(_lib.lib.dt_treeflash_build(
        ptr(h), ptr(embed), ptr(w_norm_h), ptr(w_norm_e), ptr(w_gate), ptr(w_up), ptr(w_down),
        ptr(w_lm), ptr(root), batch, gamma, D, Dff, V, M, budget, ctypes.byref(st), ptr(ws),
        ws.numel(), stream_ptr(stream)), "dt_treeflash_build")
    return out


def tree_load_budget(tree: Tree, capacity, ws, *, prefix_len=None, prefix_unit=0, n_keep=None,
                     stream=None):
    """dt_tree_load_budget: cut the batch's trees (in place) to a round's
    verification capacity by survival; returns ``tree``."""
    batch, Nmax = tree.keys.shape
    st = tree.c_struct()
    check(_lib.lib.dt_tree_load_budget(
        ctypes.byref(st), batch, Nmax, ptr(prefix_len), int(capacity), int(prefix_unit),
        ptr(n_keep), ptr(ws), ws.numel(), stream_ptr(stream)), "dt_tree_load_budget")
    return tree


def load_budget_workspace_bytes() -> int:
    return int(_lib.lib.dt_tree_load_budget_workspace_bytes())


def calib_workspace_bytes(Bk=1, n_alpha=1, n_beta=1) -> int:
    return int(_lib.lib.dt_calib_workspace_bytes(Bk, n_alpha, n_beta))


def calib_log(tree: Tree, acc_nodes, n_acc, Bk, depth, ell, y, ws, stream=None):
    """dt_calib_log: (depth, l, y) [batch, Nmax] of every child of a reached node."""
    batch, Nmax = tree.keys.shape
    st = tree.c_struct()
    check(_lib.lib.dt_calib_log(
        ctypes.byref(st), ptr(acc_nodes), ptr(n_acc), batch, Bk, Nmax, ptr(depth), ptr(ell), ptr(y),
        ptr(ws), ws.numel(), stream_ptr(stream)), "dt_calib_log")
    return depth, ell, y


def calib_fit(depth, ell, y, Bk, grid, calib, ws, loglik=None, min_samples=1, stream=None):
    """dt_calib_fit over the flattened samples; grid = (alpha0, dalpha, n_alpha,
    beta0, dbeta, n_beta); writes calib [Bk, 2] fp32 (and loglik [Bk] fp64)."""
    a0, da, na, b0, db, nb = grid
    check(_lib.lib.dt_calib_fit(
        ptr(depth), ptr(ell), ptr(y), depth.numel(), Bk, float(a0), float(da), int(na), float(b0),
        float(db), int(nb), int(min_samples), ptr(calib), ptr(loglik), ptr(ws), ws.numel(),
        stream_ptr(stream)), "dt_calib_fit")
    return calib


# ------------------------------------------------ vocabulary-sharded build --
def shard_range(V, world, rank):
    """(v_base, v_len): the Markov-factor rows Bm[v_base : v_base + v_len] rank holds."""
    a, b = ctypes.c_int(0), ctypes.c_int(0)
    _lib.lib.dt_shard_range(V, world, rank, ctypes.byref(a), ctypes.byref(b))
    return a.value, b.value


def shard_cfg(batch, Bk, V, r, k, Nmax, world, ncta=None):
    ncta = int(_lib.lib.dt_shard_ncta(V, world)) if ncta is None else ncta
    return _lib.ShardCfg(batch, Bk, V, r, k, Nmax, world, ncta)


def sharded_workspace_bytes(cfg) -> int:
    return int(_lib.lib.dt_sharded_workspace_bytes(ctypes.byref(cfg)))


def sharded_partials_bytes(cfg) -> int:
    return int(_lib.lib.dt_sharded_partials_bytes(ctypes.byref(cfg)))


def sharded_build_begin(cfg, root_token, n_budget, lam, out: Tree, ws, k_req=None, stream=None):
    st = out.c_struct()
    check(_lib.lib.dt_sharded_build_begin(
        ctypes.byref(cfg), ptr(root_token), ptr(n_budget), ptr(k_req), ptr(lam), ctypes.byref(st),
        ptr(ws), ws.numel(), stream_ptr(stream)), "dt_sharded_build_begin")


def sharded_build_gemm(cfg, wave, rank, block_logits, markov_a, markov_b_shard, ws, partials,
                       stream=None):
    check(_lib.lib.dt_sharded_build_gemm(
        ctypes.byref(cfg), wave, rank, ptr(block_logits), dtype_code(block_logits), ptr(markov_a),
        ptr(markov_b_shard), ptr(ws), ws.numel(), ptr(partials), stream_ptr(stream)),
        "dt_sharded_build_gemm")


def sharded_build_frontier(cfg, wave, gathered, n_budget, lam, out: Tree, ws, calib=None,
                           k_req=None, stream=None):
    st = out.c_struct()
    check(_lib.lib.dt_sharded_build_frontier(
        ctypes.byref(cfg), wave, ptr(gathered), ptr(calib), ptr(n_budget), ptr(k_req), ptr(lam),
        ctypes.byref(st), ptr(ws), ws.numel(), stream_ptr(stream)), "dt_sharded_build_frontier")


def tree_build_sharded(cfg, rank, block_logits, markov_a, markov_b_shard, root_token, n_budget,
                       lam, out: Tree, ws, partials, gathered, all_gather, calib=None, k_req=None,
                       stream=None):
    """The sharded build's wave loop on one rank.  ``partials`` holds this
    rank's block (sharded_partials_bytes), ``gathered`` world blocks;
    ``all_gather(gathered, partials)`` must fill ``gathered`` with every
    rank's block in rank order (torch.distributed.all_gather_into_tensor over
    the ranks sharing the vocabulary)."""
    sharded_build_begin(cfg, root_token, n_budget, lam, out, ws, k_req=k_req, stream=stream)
    for wave in range(cfg.Bk):
        sharded_build_gemm(cfg, wave, rank, block_logits, markov_a, markov_b_shard, ws, partials,
                           stream=stream)
        all_gather(gathered, partials)
        sharded_build_frontier(cfg, wave, gathered, n_budget, lam, out, ws, calib=calib,
                               k_req=k_req, stream=stream)
    return out


def set_build_path(path: str) -> None:
    """How tree_build runs its waves on this host thread: "auto", "waves" or
    "persistent" (dt_set_build_path)."""
    _lib.lib.dt_set_build_path(_lib.BUILD_PATHS[path])


def set_build_wait_test(stall_cta: int, wait_ns: int) -> None:
    """Test hook: the next persistent build on this thread stalls one CTA at its
    first grid barrier and bounds every wait by wait_ns (dt_set_build_wait_test)."""
    _lib.lib.dt_set_build_wait_test(int(stall_cta), int(wait_ns))


def read_status(ws, stream=None) -> int:
    """Synchronise and return (then clear) the device status word of a workspace."""
    v = ctypes.c_int32(0)
    check(_lib.lib.dt_read_status(ptr(ws), stream_ptr(stream), ctypes.byref(v)), "dt_read_status")
    return int(v.value)
