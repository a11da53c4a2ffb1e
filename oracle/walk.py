"""ctypes wrapper around the fp64 C oracle (``stree_oracle.c``) -- test infrastructure.

Every function takes numpy arrays in the layouts of the scan
(x [b,T,H,P], dt [b,T,H], A [H], B/C [b,T,G,N], D [H], h0 [b,H,P,N],
parent int32 [b,T]) and converts them to contiguous fp64 / int32 before the call.
The inputs given here must be the values the device sees (already rounded to
the stored dtype); the oracle computes in fp64 from them.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "stree_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lib = None


def build_oracle(force: bool = False) -> str:
    """Compile the C oracle into ``oracle/liboracle.so`` (gcc, -O2, OpenMP)."""
    stale = (not os.path.exists(_LIB_PATH)
             or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC))
    if force or stale:
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.run(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp",
                        "-o", tmp, _SRC, "-lm"], check=True)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build_oracle())
        i32, dp, ip, up = (ctypes.c_int, ctypes.POINTER(ctypes.c_double),
                           ctypes.POINTER(ctypes.c_int32), ctypes.POINTER(ctypes.c_uint32))
        lib.oracle_build_tree.argtypes = [ip, i32, i32, up, ip, ip]
        lib.oracle_tree_scan.argtypes = [dp, dp, dp, dp, dp, dp, dp, ip,
                                         i32, i32, i32, i32, i32, i32, dp, i32]
        lib.oracle_commit.argtypes = [dp, dp, dp, dp, dp, ip, ip, ip, i32,
                                      i32, i32, i32, i32, i32, i32, dp, ip, ip, i32]
        for f in (lib.oracle_build_tree, lib.oracle_tree_scan, lib.oracle_commit,
                  lib.oracle_max_threads):
            f.restype = ctypes.c_int
        _lib = lib
    return _lib


def _f64(a):
    return np.ascontiguousarray(a, dtype=np.float64)


def _i32(a):
    return np.ascontiguousarray(a, dtype=np.int32)


def _ptr(a, ct):
    return a.ctypes.data_as(ctypes.POINTER(ct))


def oracle_max_threads() -> int:
    return int(_load().oracle_max_threads())


def oracle_build_tree(parent):
    """parent int32 [b,T] -> (anc uint32 [b,T,W], depth int32 [b,T], ok int32 [b])."""
    parent = _i32(parent)
    batch, T = parent.shape
    W = (T + 31) // 32
    anc = np.zeros((batch, T, W), np.uint32)
    depth = np.zeros((batch, T), np.int32)
    ok = np.zeros((batch,), np.int32)
    _load().oracle_build_tree(_ptr(parent, ctypes.c_int32), T, batch,
                              _ptr(anc, ctypes.c_uint32), _ptr(depth, ctypes.c_int32),
                              _ptr(ok, ctypes.c_int32))
    return anc, depth, ok


def _shapes(x, B, h0):
    batch, T, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    assert h0.shape == (batch, H, P, N) and B.shape[:2] == (batch, T)
    assert H % G == 0
    return batch, T, H, P, N, G


def oracle_tree_scan(x, dt, A, B, C, D, h0, parent, nthreads: int = 1):
    """fp64 y [b,T,H,P]: every node's output from a walk of its root path."""
    x, dt, A, B, C, D, h0 = map(_f64, (x, dt, A, B, C, D, h0))
    parent = _i32(parent)
    batch, T, H, P, N, G = _shapes(x, B, h0)
    y = np.full((batch, T, H, P), np.nan)
    bad = _load().oracle_tree_scan(
        _ptr(x, ctypes.c_double), _ptr(dt, ctypes.c_double), _ptr(A, ctypes.c_double),
        _ptr(B, ctypes.c_double), _ptr(C, ctypes.c_double), _ptr(D, ctypes.c_double),
        _ptr(h0, ctypes.c_double), _ptr(parent, ctypes.c_int32),
        T, batch, H, P, N, G, _ptr(y, ctypes.c_double), int(nthreads))
    if bad:
        raise ValueError(f"{bad} sequence(s) with an invalid packed tree")
    return y


def oracle_commit(x, dt, A, B, h0, parent, path, path_len, nthreads: int = 1,
                  allow_invalid: bool = False):
    """fp64 h_new [b,H,P,N] by replaying the accepted path from h0.

    Returns (h_new, ok int32 [b], leaf int32 [b]).  Rejected sequences keep NaN
    unless ``allow_invalid`` is False, in which case a ValueError is raised.
    """
    x, dt, A, B, h0 = map(_f64, (x, dt, A, B, h0))
    parent, path, path_len = _i32(parent), _i32(path), _i32(path_len)
    batch, T, H, P, N, G = _shapes(x, B, h0)
    if path.ndim == 1:
        path = path.reshape(batch, -1)
    maxlen = path.shape[1]
    h_new = np.full((batch, H, P, N), np.nan)
    ok = np.zeros((batch,), np.int32)
    leaf = np.zeros((batch,), np.int32)
    bad = _load().oracle_commit(
        _ptr(x, ctypes.c_double), _ptr(dt, ctypes.c_double), _ptr(A, ctypes.c_double),
        _ptr(B, ctypes.c_double), _ptr(h0, ctypes.c_double), _ptr(parent, ctypes.c_int32),
        _ptr(path, ctypes.c_int32), _ptr(path_len, ctypes.c_int32), maxlen,
        T, batch, H, P, N, G, _ptr(h_new, ctypes.c_double),
        _ptr(ok, ctypes.c_int32), _ptr(leaf, ctypes.c_int32), int(nthreads))
    if bad and not allow_invalid:
        raise ValueError(f"{bad} sequence(s) with an invalid tree or accepted path")
    return h_new, ok, leaf


def default_threads() -> int:
    try:
        return max(1, len(os.sched_getaffinity(0)))
    except AttributeError:  # pragma: no cover
        return max(1, os.cpu_count() or 1)
