"""The C-ABI library loads and exports every symbol its header declares, and
rejects bad arguments before touching a device (runs without a GPU)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    src = open(os.path.join(ROOT, "include", "dtree.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(dt_[a-z_0-9]+)\s*\(", src)))


def test_library_exports_every_declared_symbol():
    import draft_tree_construction_markov_b200._lib as L
    names = _declared_functions()
    assert {"dt_tree_build", "dt_tree_verify_attn", "dt_tree_accept"} <= set(names)
    for n in names:
        assert hasattr(L.lib, n), n


def test_workspace_queries_are_positive_and_grow():
    import draft_tree_construction_markov_b200 as dt
    a = dt.build_workspace_bytes(1, 7, 151936, 256, 4, 32)
    b = dt.build_workspace_bytes(64, 7, 151936, 256, 4, 32)
    assert 0 < a < b
    assert dt.verify_workspace_bytes(1, 32, 32, 8, 128, 2048) > 0
    assert dt.accept_workspace_bytes(1, 32, 151936) > 0
    assert dt.build_workspace_bytes(0, 7, 10, 16, 1, 1) == 0


def _call_build(L, **kw):
    p = ctypes.c_void_p(0x1000)  # never dereferenced: validation fails first
    args = dict(logits=p, ldt=1, a=p, b=p, r=16, calib=None, root=p, nb=p, kreq=None, lam=p,
                batch=1, Bk=4, V=512, k=2, Nmax=8, temp=0.0, seed=0, off=0)
    args.update(kw)
    tree = L.DtTree(p, p, p, p, p, p, p, p)
    return L.lib.dt_tree_build(args["logits"], args["ldt"], args["a"], args["b"], args["r"],
                               args["calib"], args["root"], args["nb"], args["kreq"], args["lam"],
                               args["batch"], args["Bk"], args["V"], args["k"], args["Nmax"],
                               args["temp"], args["seed"], args["off"], ctypes.byref(tree),
                               None, 0, None)


@pytest.mark.parametrize("kw,code", [
    (dict(logits=None), 1),            # null pointer
    (dict(ldt=7), 1),                  # unknown dtype
    (dict(Nmax=65), 2),                # beyond the 64-bit ancestor mask
    (dict(k=17), 2),                   # k > 16
    (dict(r=24), 2),                   # r not a multiple of 16
    (dict(Bk=17), 2),
    (dict(k=600, V=512), 2),           # k > 16 reported first
    (dict(temp=-1.0), 1),
    (dict(off=1 << 32), 1),            # Philox offset must fit 32 bits
    (dict(), 5),                       # no workspace
])
def test_build_rejects_bad_arguments(kw, code):
    import draft_tree_construction_markov_b200._lib as L
    assert _call_build(L, **kw) == code


def test_accept_and_attention_reject_bad_arguments():
    import draft_tree_construction_markov_b200._lib as L
    p = ctypes.c_void_p(0x1000)
    tree = L.DtTree(p, p, p, p, p, p, p, None)
    # T > 0 needs the draft distributions
    assert L.lib.dt_tree_accept(p, 1, ctypes.byref(tree), 1, 4, 512, 8, 1.0, 0, 0, p, p, p,
                                None, 0, None) == L.DT_EINVAL
    assert L.lib.dt_tree_accept(p, 1, ctypes.byref(tree), 1, 4, 512, 8, 0.0, 0, 0, p, p, p,
                                None, 0, None) == L.DT_EWORKSPACE
    # head_dim 96 unsupported; Hq not a multiple of Hkv
    assert L.lib.dt_tree_verify_attn(p, p, p, p, p, 32, p, p, p, p, 1, 8, 4, 2, 96, 0.1, 1, p,
                                     None, 0, None) == L.DT_EUNSUPPORTED
    assert L.lib.dt_tree_verify_attn(p, p, p, p, p, 32, p, p, p, p, 1, 8, 6, 4, 64, 0.1, 1, p,
                                     None, 0, None) == L.DT_EINVAL


def test_new_entry_points_reject_bad_arguments_without_a_device():
    import draft_tree_construction_markov_b200._lib as L
    p = ctypes.c_void_p(0x1000)  # never dereferenced: validation fails first
    tree = L.DtTree(p, p, p, p, p, p, p, p)
    t = ctypes.byref(tree)
    # baseline variants: an unknown variant
    assert L.lib.dt_tree_build_ex(p, 1, p, p, 16, None, p, p, None, p, 1, 4, 512, 2, 8, 0.0, 0, 0,
                                  7, t, p, 1 << 20, None) == L.DT_EINVAL
    # load budget: negative capacity, too large a batch, no workspace
    assert L.lib.dt_tree_load_budget(t, 2, 8, None, -1, 0, None, p, 256, None) == L.DT_EINVAL
    assert L.lib.dt_tree_load_budget(t, 1025, 8, None, 5, 0, None, p, 256, None) == \
        L.DT_EUNSUPPORTED
    assert L.lib.dt_tree_load_budget(t, 2, 8, None, 5, 0, None, None, 0, None) == L.DT_EWORKSPACE
    # calibration: negative alpha start, too large a grid, too small a workspace
    assert L.lib.dt_calib_fit(p, p, p, 10, 4, -1.0, 0.1, 4, 0.0, 0.1, 4, 1, p, None, p, 4096,
                              None) == L.DT_EINVAL
    assert L.lib.dt_calib_fit(p, p, p, 10, 4, 0.0, 0.1, 2048, 0.0, 0.1, 1024, 1, p, None, p,
                              1 << 30, None) == L.DT_EUNSUPPORTED
    need = L.lib.dt_calib_workspace_bytes(4, 64, 64)
    assert need > 256
    assert L.lib.dt_calib_fit(p, p, p, 10, 4, 0.0, 0.1, 64, 0.0, 0.1, 64, 1, p, None, p, need - 1,
                              None) == L.DT_EWORKSPACE
    assert L.lib.dt_calib_log(t, p, p, 1025, 4, 8, p, p, p, p, 256, None) == L.DT_EUNSUPPORTED
    # sharded build: more partials per rank than the smallest shard has tiles
    bad = L.ShardCfg(1, 4, 512, 16, 2, 8, 2, 3)
    assert L.lib.dt_sharded_workspace_bytes(ctypes.byref(bad)) == 0
    assert L.lib.dt_sharded_build_begin(ctypes.byref(bad), p, p, None, p, t, p, 1 << 20,
                                        None) == L.DT_EUNSUPPORTED
    good = L.ShardCfg(1, 4, 512, 16, 2, 8, 2, 2)
    assert L.lib.dt_sharded_workspace_bytes(ctypes.byref(good)) > 0
    assert L.lib.dt_sharded_build_gemm(ctypes.byref(good), 0, 2, p, 1, p, p, p, 1 << 20, p,
                                       None) == L.DT_EINVAL      # rank outside the world
    assert L.lib.dt_sharded_build_frontier(ctypes.byref(good), 4, p, None, p, None, p, t, p,
                                           1 << 20, None) == L.DT_EINVAL   # wave >= Bk


def _prototypes():
    """name -> [C parameter types] for every function declared in the header."""
    src = open(os.path.join(ROOT, "include", "dtree.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    out = {}
    for m in re.finditer(r"\b(dt_[a-z_0-9]+)\s*\(([^)]*)\)\s*;", src):
        params = [p.strip() for p in m.group(2).split(",") if p.strip() and p.strip() != "void"]
        types = []
        for p in params:
            p = re.sub(r"\s+", " ", p)
            name = re.search(r"(\w+)\s*$", p).group(1)
            types.append(p[: p.rfind(name)].strip())
        out[m.group(1)] = types
    return out


def _ctype_for(c):
    import ctypes as C
    if "*" in c:
        return "ptr"
    base = c.replace("const ", "").strip()
    return {"int": C.c_int, "float": C.c_float, "uint64_t": C.c_uint64, "int64_t": C.c_int64,
            "size_t": C.c_size_t, "dt_dtype": C.c_int, "dt_tree_variant": C.c_int,
            "dt_stream": "ptr"}[base]


def test_binding_signatures_match_the_header():
    """Every function the binding gives argtypes to has the header's parameter
    count, and each parameter the same kind (pointer, or the same scalar)."""
    import ctypes as C
    import draft_tree_construction_markov_b200._lib as L
    protos = _prototypes()
    checked = 0
    for name, types in protos.items():
        fn = getattr(L.lib, name)
        if fn.argtypes is None:
            continue
        assert len(fn.argtypes) == len(types), name
        for i, (ct, at) in enumerate(zip(types, fn.argtypes)):
            want = _ctype_for(ct)
            if want == "ptr":
                assert at is C.c_void_p or issubclass(at, C._Pointer), (name, i, ct, at)
            else:
                assert at is want, (name, i, ct, at)
        checked += 1
    assert checked >= 20
