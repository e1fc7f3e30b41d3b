"""ctypes binding of libdtree.so: argument marshalling only.

Every computation happens inside the library's CUDA kernels; this module turns
torch tensors into device pointers and sizes, and status codes into
exceptions.  Importing it fails loudly if the compiled library is missing.
"""
import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libdtree.so")

DT_OK, DT_EINVAL, DT_EUNSUPPORTED, DT_ECUDA, DT_ETIMEOUT, DT_EWORKSPACE, DT_EDEVICE = range(7)
STATUS_NAMES = {0: "DT_OK", 1: "DT_EINVAL", 2: "DT_EUNSUPPORTED", 3: "DT_ECUDA",
                4: "DT_ETIMEOUT", 5: "DT_EWORKSPACE", 6: "DT_EDEVICE"}
DT_F32, DT_BF16 = 0, 1
TREE_VARIANTS = {"pctree": 0, "chain": 1, "marginal": 2, "shared_markov": 3}

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with "
        "`python draft_tree_construction_markov_b200/build.py` (nvcc, sm_100a)")

lib = ctypes.CDLL(LIB_PATH)

_vp, _sz, _i32, _u64, _f32 = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int, ctypes.c_uint64, ctypes.c_float


class DtTree(ctypes.Structure):
    _fields_ = [("d_tokens", _vp), ("d_parents", _vp), ("d_depths", _vp), ("d_ranks", _vp),
                ("d_keys", _vp), ("d_anc", _vp), ("d_n_nodes", _vp), ("d_draft_q", _vp)]


class ShardCfg(ctypes.Structure):
    _fields_ = [(nm, ctypes.c_int) for nm in ("batch", "Bk", "V", "r", "k", "Nmax", "world",
                                               "ncta")]


def _sig(name, restype, *args):
    f = getattr(lib, name)
    f.restype = restype
    f.argtypes = list(args)
    return f


_sig("dt_num_sms", _i32)
_sig("dt_tree_build_workspace_bytes", _sz, _i32, _i32, _i32, _i32, _i32, _i32)
_sig("dt_tree_build", _i32, _vp, _i32, _vp, _vp, _i32, _vp, _vp, _vp, _vp, _vp,
     _i32, _i32, _i32, _i32, _i32, _f32, _u64, _u64, ctypes.POINTER(DtTree), _vp, _sz, _vp)
_sig("dt_tree_build_ex", _i32, _vp, _i32, _vp, _vp, _i32, _vp, _vp, _vp, _vp, _vp,
     _i32, _i32, _i32, _i32, _i32, _f32, _u64, _u64, _i32, ctypes.POINTER(DtTree), _vp, _sz, _vp)
_sig("dt_markov_logits_workspace_bytes", _sz, _i32, _i32, _i32)
_sig("dt_markov_logits", _i32, _vp, _i32, _vp, _vp, _i32, _i32, _i32, _i32, _vp, _vp, _vp,
     _i32, _vp, _vp, _sz, _vp)
_sig("dt_tree_verify_attn_workspace_bytes", _sz, _i32, _i32, _i32, _i32, _i32, _i32)
_sig("dt_tree_verify_attn", _i32, _vp, _vp, _vp, _vp, _vp, _i32, _vp, _vp, _vp, _vp,
     _i32, _i32, _i32, _i32, _i32, _f32, _i32, _vp, _vp, _sz, _vp)
_sig("dt_tree_accept_workspace_bytes", _sz, _i32, _i32, _i32)
_sig("dt_tree_accept", _i32, _vp, _i32, ctypes.POINTER(DtTree), _i32, _i32, _i32, _i32, _f32,
     _u64, _u64, _vp, _vp, _vp, _vp, _sz, _vp)
_sig("dt_tree_accept_noalloc", _i32, _vp, _i32, ctypes.POINTER(DtTree), _i32, _i32, _i32, _i32,
     _f32, _u64, _u64, _vp, _vp, _vp, _vp)
_sig("dt_treeflash_workspace_bytes", _sz, _i32, _i32, _i32, _i32, _i32, _i32, _i32)
_sig("dt_treeflash_build", _i32, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i32, _i32, _i32,
     _i32, _i32, _i32, _i32, ctypes.POINTER(DtTree), _vp, _sz, _vp)
_sig("dt_tree_load_budget_workspace_bytes", _sz)
_sig("dt_tree_load_budget", _i32, ctypes.POINTER(DtTree), _i32, _i32, _vp, ctypes.c_int64, _i32,
     _vp, _vp, _sz, _vp)
_sig("dt_calib_workspace_bytes", _sz, _i32, _i32, _i32)
_sig("dt_calib_log", _i32, ctypes.POINTER(DtTree), _vp, _vp, _i32, _i32, _i32, _vp, _vp, _vp, _vp,
     _sz, _vp)
_sig("dt_calib_fit", _i32, _vp, _vp, _vp, _i32, _i32, _f32, _f32, _i32, _f32, _f32, _i32, _i32,
     _vp, _vp, _vp, _sz, _vp)
_PC = ctypes.POINTER(ShardCfg)
_sig("dt_shard_range", None, _i32, _i32, _i32, ctypes.POINTER(_i32), ctypes.POINTER(_i32))
_sig("dt_shard_ncta", _i32, _i32, _i32)
_sig("dt_sharded_workspace_bytes", _sz, _PC)
_sig("dt_sharded_partials_bytes", _sz, _PC)
_sig("dt_sharded_build_begin", _i32, _PC, _vp, _vp, _vp, _vp, ctypes.POINTER(DtTree), _vp, _sz, _vp)
_sig("dt_sharded_build_gemm", _i32, _PC, _i32, _i32, _vp, _i32, _vp, _vp, _vp, _sz, _vp, _vp)
_sig("dt_sharded_build_frontier", _i32, _PC, _i32, _vp, _vp, _vp, _vp, _vp, ctypes.POINTER(DtTree),
     _vp, _sz, _vp)
_sig("dt_read_status", _i32, _vp, _vp, ctypes.POINTER(ctypes.c_int32))
_sig("dt_set_profile_events", None, ctypes.POINTER(ctypes.c_void_p), ctypes.POINTER(ctypes.c_int32),
     _i32, ctypes.POINTER(ctypes.c_int32))

_sig("dt_set_build_path", None, _i32)
_sig("dt_set_build_wait_test", None, _i32, _u64)

KERNEL_KINDS = ["build_init", "markov_gemm", "frontier", "draft_q", "accept_prepass",
                "accept_walk", "attn", "attn_combine", "other", "tf_lmhead", "tf_mlp", "pbuild"]
BUILD_PATHS = {"auto": 0, "waves": 1, "persistent": 2}


class DtreeError(RuntimeError):
    def __init__(self, code, where):
        super().__init__(f"{where}: {STATUS_NAMES.get(code, code)}")
        self.code = code


def check(code, where):
    if code != DT_OK:
        raise DtreeError(code, where)


def ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def dtype_code(t):
    if t.dtype == torch.float32:
        return DT_F32
    if t.dtype == torch.bfloat16:
        return DT_BF16
    raise TypeError(f"unsupported dtype {t.dtype}")


def stream_ptr(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)
