"""dt_tree_accept_noalloc: the acceptance walk for callers that cannot
allocate device memory (a plugin whose host framework owns the device memory,
or a serving loop that must not call cudaMalloc).  Its scratch is a fixed
array inside the library, so this test checks, through the C ABI, that two
calls in a row give exactly the outputs of dt_tree_accept with a caller
workspace: the second call must not be disturbed by what the first one left
in the shared array.  It runs alone or after every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

from gen import make_workload

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import draft_tree_construction_markov_b200 as dt
    from draft_tree_construction_markov_b200 import _lib
    from tests.gpu_util import BF16, dev, run_build, target_for_tree, tree_to_host

    # the C entry point with the signature the binding declares for it (checked
    # here, not reassigned, so the binding's own declaration is what runs)
    _fn = _lib.lib.dt_tree_accept_noalloc
    assert _fn.restype is ctypes.c_int
    assert list(_fn.argtypes) == [
        ctypes.c_void_p, ctypes.c_int, ctypes.POINTER(_lib.DtTree), ctypes.c_int, ctypes.c_int,
        ctypes.c_int, ctypes.c_int, ctypes.c_float, ctypes.c_uint64, ctypes.c_uint64,
        ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]


def _outputs(w):
    return (torch.full((w.batch, w.Bk), -7, dtype=torch.int32, device="cuda"),
            torch.full((w.batch,), -7, dtype=torch.int32, device="cuda"),
            torch.full((w.batch,), -7, dtype=torch.int32, device="cuda"))


def _noalloc(w, tgt, tree, temp, seed, offset):
    acc, nacc, bonus = _outputs(w)
    st = tree.c_struct()
    code = _fn(ctypes.c_void_p(tgt.data_ptr()), _lib.dtype_code(tgt), ctypes.byref(st), w.batch,
               w.Bk, w.V, w.Nmax, temp, seed, offset, ctypes.c_void_p(acc.data_ptr()),
               ctypes.c_void_p(nacc.data_ptr()), ctypes.c_void_p(bonus.data_ptr()),
               _lib.stream_ptr())
    assert code == _lib.DT_OK
    torch.cuda.synchronize()
    return acc.cpu().numpy(), nacc.cpu().numpy(), bonus.cpu().numpy()


def _with_workspace(w, tgt, tree, temp, seed, offset):
    acc, nacc, bonus = _outputs(w)
    ws = dt.workspace(dt.accept_workspace_bytes(w.batch, w.Nmax, w.V))
    dt.tree_accept(tgt, tree, w.Bk, temp, acc, nacc, bonus, ws, philox_seed=seed,
                   philox_offset=offset)
    assert dt.read_status(ws) == 0
    return acc.cpu().numpy(), nacc.cpu().numpy(), bonus.cpu().numpy()


@pytest.mark.parametrize("name,temp", [("tiny", 1.0), ("qwen3_4b", 0.0), ("qwen3_4b", 0.8)])
def test_noalloc_accept_matches_workspace_accept_twice(name, temp):
    w = make_workload(name, seed=3, temp=temp)
    tree = run_build(w, temp=temp)
    h = tree_to_host(tree, 0)
    tdt = BF16 if w.logit_dtype == "bf16" else torch.float32
    tgt = dev(target_for_tree(w, 0, h["depths"], h["tokens"])[None], tdt)
    # two calls in a row with different random streams, each against the
    # workspace entry point on the same arguments
    for seed, offset in ((11, 0), (12, 5)):
        got = _noalloc(w, tgt, tree, temp, seed, offset)
        want = _with_workspace(w, tgt, tree, temp, seed, offset)
        for g, x in zip(got, want):
            assert np.array_equal(g, x)


def test_noalloc_rejects_sizes_beyond_its_scratch():
    w = make_workload("qwen3_4b", seed=0, batch=4)
    tree = dt.Tree.empty(4, w.Nmax, w.V, stochastic=True)
    tgt = torch.zeros(4, w.Nmax + 1, w.V, dtype=BF16, device="cuda")
    acc, nacc, bonus = _outputs(w)
    st = tree.c_struct()
    code = _fn(ctypes.c_void_p(tgt.data_ptr()), _lib.DT_BF16, ctypes.byref(st), 4, w.Bk, w.V,
               w.Nmax, 1.0, 1, 0, ctypes.c_void_p(acc.data_ptr()),
               ctypes.c_void_p(nacc.data_ptr()), ctypes.c_void_p(bonus.data_ptr()),
               _lib.stream_ptr())
    assert code == _lib.DT_EUNSUPPORTED
