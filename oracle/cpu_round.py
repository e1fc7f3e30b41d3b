"""Loader of the multi-core C++ restatement of the oracle's greedy round
(cpu_round.cpp).  Test and measurement infrastructure only: bench.py times it
as the multi-core CPU baseline, and tests/test_oracle_cpu_round.py checks it
against the numpy oracle.

The shared object is compiled on first use with -O3 -march=native -fopenmp
for the host it runs on, into the temporary directory (keyed by the source
and the host CPU), so that a build made on one machine never runs on another.
"""
import ctypes
import hashlib
import os
import platform
import subprocess
import tempfile

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "cpu_round.cpp")
_lib = None


def _cpu_id():
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name") or line.startswith("flags"):
                    return line
    except OSError:
        pass
    return platform.processor()


def load():
    global _lib
    if _lib is not None:
        return _lib
    key = hashlib.sha256(open(_SRC, "rb").read() + _cpu_id().encode()).hexdigest()[:16]
    so = os.path.join(tempfile.gettempdir(), f"dtree_cpu_round_{key}.so")
    if not os.path.exists(so):
        tmp = so + f".{os.getpid()}.tmp"
        subprocess.run(["g++", "-O3", "-march=native", "-fopenmp", "-shared", "-fPIC",
                        "-std=c++17", "-o", tmp, _SRC], check=True)
        os.replace(tmp, so)
    lib = ctypes.CDLL(so)
    f = lib.cpu_round_t0
    P = ctypes.c_void_p
    i, dbl = ctypes.c_int, ctypes.c_double
    f.restype = i
    f.argtypes = [P, P, P, i, i, i, i, i, i, P, P, P, P, P, i, i, i, i, dbl, P, P, P, P, P, P,
                  P, P, P, P]
    _lib = lib
    return lib


def threads():
    """Threads the OpenMP runtime will use (all host cores unless limited)."""
    return int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))


def round_t0(L, A, Bt, root, k, N, attn, scale, target):
    """One greedy round: L (Bk, V), A and Bt (V, r) float32; attn = (q, kp, vp,
    kt, vt) float32 of one request; target (N+1, V) float32.  Returns a dict
    with the tree, attention rows (fp64) and the accept result."""
    lib = load()
    L, A, Bt = (np.ascontiguousarray(x, np.float32) for x in (L, A, Bt))
    q, kp, vp, kt, vt = (np.ascontiguousarray(x, np.float32) for x in attn)
    target = np.ascontiguousarray(target, np.float32)
    Bk, V = L.shape
    r = A.shape[1]
    P, Hkv, d = kp.shape
    Hq = q.shape[1]
    tok = np.zeros(max(N, 1), np.int32)
    par = np.zeros_like(tok)
    dep = np.zeros_like(tok)
    keys = np.zeros(max(N, 1), np.float64)
    n = np.zeros(1, np.int32)
    out = np.zeros((N + 1, Hq, d), np.float64)
    acc = np.full(Bk, -1, np.int32)
    nacc = np.zeros(1, np.int32)
    bonus = np.zeros(1, np.int32)
    p = lambda x: x.ctypes.data_as(ctypes.c_void_p)
    rc = lib.cpu_round_t0(p(L), p(A), p(Bt), V, r, Bk, k, N, int(root), p(q), p(kp), p(vp),
                          p(kt), p(vt), P, Hq, Hkv, d, float(scale), p(target), p(tok), p(par),
                          p(dep), p(keys), p(n), p(out), p(acc), p(nacc), p(bonus))
    if rc != 0:
        raise ValueError("cpu_round_t0 rejected its arguments")
    m = int(n[0])
    return dict(n=m, tokens=tok[:m], parents=par[:m], depths=dep[:m], keys=keys[:m],
                attn=out[: m + 1], acc=acc[: int(nacc[0])], bonus=int(bonus[0]))
