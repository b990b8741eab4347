"""fp64 CPU oracle for greedy RVQ encode / gather-sum decode.

TEST INFRASTRUCTURE ONLY: the test suite, the smoke check and the bench's CPU
baseline leg use it; the product path (the CUDA library and its binding) never
imports it.  The arithmetic lives in `rvq_oracle.c` (plain C, fp64, one OpenMP
loop over rows); this module compiles it with gcc and marshals numpy arrays.

Functions (all inputs are float32 arrays whose values are the stored fp32/bf16
values; the C side widens each element to double):
  encode(x, C, rows=None, threads=0)        -> ids [M,L] int32, residual [M,D], recon [M,D], dist [M,L]
  decode(ids, C, threads=0)                 -> recon [M,D] fp64 (raises on an id outside [0,K))
  check_path(x, C, rows, ids, threads=0)    -> per-level best, argmin, second, chosen for given ids
  distances(r, C_l)                         -> fp64 distance vector of one level
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "rvq_oracle.c")
_LIB = os.path.join(_HERE, "librvq_oracle.so")
_lock = threading.Lock()
_lib = None

CFLAGS = ["-O2", "-fopenmp", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared", "-std=c11"]


def build(src: str = _SRC, out: str = _LIB, force: bool = False) -> str:
    """Compile the oracle with gcc (idempotent unless the source is newer)."""
    if not force and os.path.exists(out) and os.path.getmtime(out) >= os.path.getmtime(src):
        return out
    tmp = out + f".tmp{os.getpid()}"
    subprocess.check_call(["gcc", *CFLAGS, src, "-o", tmp, "-lm"])
    os.replace(tmp, out)
    return out


def load(path: str | None = None):
    """Load (building if needed) the oracle library; `path` selects another build of it."""
    global _lib
    if path is not None:
        return _declare(ctypes.CDLL(path))
    with _lock:
        if _lib is None:
            _lib = _declare(ctypes.CDLL(build()))
    return _lib


def _declare(lib):
    f32p = ctypes.POINTER(ctypes.c_float)
    f64p = ctypes.POINTER(ctypes.c_double)
    i32p = ctypes.POINTER(ctypes.c_int32)
    i64p = ctypes.POINTER(ctypes.c_int64)
    I, I64 = ctypes.c_int, ctypes.c_int64
    lib.rvq_oracle_encode.argtypes = [f32p, I64, I, f32p, I, I, i64p, I64, i32p, f64p, f64p, f64p, I]
    lib.rvq_oracle_decode.argtypes = [i32p, I64, I, f32p, I, I, f64p, I]
    lib.rvq_oracle_check_path.argtypes = [f32p, I64, I, f32p, I, I, i64p, I64, i32p,
                                          f64p, i32p, f64p, f64p, I]
    lib.rvq_oracle_distances.argtypes = [f64p, f32p, I, I, f64p]
    lib.rvq_oracle_max_threads.argtypes = [I]
    lib.rvq_oracle_embed_backward.argtypes = [i32p, I64, I, I, I, f32p, f64p, i64p, f64p, I]
    lib.rvq_oracle_codebook_update.argtypes = [f32p, i32p, I64, I, I, f32p, f64p, i64p, f64p]
    lib.rvq_oracle_balance.argtypes = [i64p, I64, I, i32p, i64p]
    for fn in ("rvq_oracle_encode", "rvq_oracle_decode", "rvq_oracle_check_path",
               "rvq_oracle_distances", "rvq_oracle_max_threads"):
        getattr(lib, fn).restype = ctypes.c_int
    return lib


def _p(a, ct):
    return a.ctypes.data_as(ctypes.POINTER(ct)) if a is not None else None


def _f32(a):
    return np.ascontiguousarray(a, dtype=np.float32)


class OracleError(RuntimeError):
    def __init__(self, code):
        super().__init__(f"oracle returned {code}")
        self.code = code


def threads(n: int = 0, lib=None) -> int:
    return (lib or load()).rvq_oracle_max_threads(int(n))


def encode(x, C, rows=None, threads: int = 0, lib=None):
    lib = lib or load()
    x, C = _f32(x), _f32(C)
    N, D = x.shape
    L, K, D2 = C.shape
    assert D == D2
    r = None if rows is None else np.ascontiguousarray(rows, dtype=np.int64)
    M = N if r is None else len(r)
    ids = np.empty((M, L), np.int32)
    res = np.empty((M, D), np.float64)
    rec = np.empty((M, D), np.float64)
    dist = np.empty((M, L), np.float64)
    rc = lib.rvq_oracle_encode(_p(x, ctypes.c_float), N, D, _p(C, ctypes.c_float), L, K,
                               _p(r, ctypes.c_int64), M, _p(ids, ctypes.c_int32),
                               _p(res, ctypes.c_double), _p(rec, ctypes.c_double),
                               _p(dist, ctypes.c_double), int(threads))
    if rc != 0:
        raise OracleError(rc)
    return ids, res, rec, dist


def decode(ids, C, threads: int = 0, lib=None):
    lib = lib or load()
    ids = np.ascontiguousarray(ids, dtype=np.int32)
    C = _f32(C)
    M, L = ids.shape
    L2, K, D = C.shape
    assert L == L2
    out = np.empty((M, D), np.float64)
    rc = lib.rvq_oracle_decode(_p(ids, ctypes.c_int32), M, L, _p(C, ctypes.c_float), K, D,
                               _p(out, ctypes.c_double), int(threads))
    if rc != 0:
        raise OracleError(rc)
    return out


def check_path(x, C, rows, ids, threads: int = 0, lib=None):
    lib = lib or load()
    x, C = _f32(x), _f32(C)
    N, D = x.shape
    L, K, _ = C.shape
    rows = np.ascontiguousarray(rows, dtype=np.int64)
    ids = np.ascontiguousarray(ids, dtype=np.int32)
    M = len(rows)
    assert ids.shape == (M, L)
    best = np.empty((M, L)); second = np.empty((M, L)); chosen = np.empty((M, L))
    argmin = np.empty((M, L), np.int32)
    rc = lib.rvq_oracle_check_path(_p(x, ctypes.c_float), N, D, _p(C, ctypes.c_float), L, K,
                                   _p(rows, ctypes.c_int64), M, _p(ids, ctypes.c_int32),
                                   _p(best, ctypes.c_double), _p(argmin, ctypes.c_int32),
                                   _p(second, ctypes.c_double), _p(chosen, ctypes.c_double),
                                   int(threads))
    if rc != 0:
        raise OracleError(rc)
    return {"best": best, "argmin": argmin, "second": second, "chosen": chosen}


def distances(r, C_l, lib=None):
    lib = lib or load()
    r = np.ascontiguousarray(r, dtype=np.float64)
    C_l = _f32(C_l)
    K, D = C_l.shape
    out = np.empty(K, np.float64)
    rc = lib.rvq_oracle_distances(_p(r, ctypes.c_double), _p(C_l, ctypes.c_float), K, D,
                                  _p(out, ctypes.c_double))
    if rc != 0:
        raise OracleError(rc)
    return out


def embed_backward(ids, g, K, bounds: bool = False, threads: int = 0, lib=None):
    """grad [L,K,H] fp64 of e[n] = sum_l E_l[ids[n,l]] given g = dLoss/de [N,H] (rows summed in
    ascending n); with bounds=True also count [L,K] and absum [L,K,H] (sum of |g| per row)."""
    lib = lib or load()
    ids = np.ascontiguousarray(ids, dtype=np.int32)
    g = _f32(g)
    N, L = ids.shape
    N2, H = g.shape
    assert N == N2
    grad = np.zeros((L, K, H), np.float64)
    count = np.zeros((L, K), np.int64) if bounds else None
    absum = np.zeros((L, K, H), np.float64) if bounds else None
    rc = lib.rvq_oracle_embed_backward(_p(ids, ctypes.c_int32), N, L, K, H, _p(g, ctypes.c_float),
                                       _p(grad, ctypes.c_double),
                                       _p(count, ctypes.c_int64) if bounds else None,
                                       _p(absum, ctypes.c_double) if bounds else None, int(threads))
    if rc != 0:
        raise OracleError(rc)
    return (grad, count, absum) if bounds else grad


def codebook_update(points, ids, old_codebook, bounds: bool = False, lib=None):
    """One k-means update of one level: new [K,D] fp64 (cluster means in ascending row order; an
    empty cluster keeps its old codeword) and count [K]; with bounds=True also absum [K,D]."""
    lib = lib or load()
    points = _f32(points)
    ids = np.ascontiguousarray(ids, dtype=np.int32).reshape(-1)
    old = _f32(old_codebook)
    N, D = points.shape
    K, D2 = old.shape
    assert D == D2 and ids.shape[0] == N
    new = np.empty((K, D), np.float64)
    count = np.empty(K, np.int64)
    absum = np.empty((K, D), np.float64) if bounds else None
    rc = lib.rvq_oracle_codebook_update(_p(points, ctypes.c_float), _p(ids, ctypes.c_int32), N, D, K,
                                        _p(old, ctypes.c_float), _p(new, ctypes.c_double),
                                        _p(count, ctypes.c_int64),
                                        _p(absum, ctypes.c_double) if bounds else None)
    if rc != 0:
        raise OracleError(rc)
    return (new, count, absum) if bounds else (new, count)


def balance(lengths, world: int, lib=None):
    """Longest-processing-time-first assignment of sequences to ranks: (owner [S], load [world])."""
    lib = lib or load()
    lengths = np.ascontiguousarray(lengths, dtype=np.int64)
    S = lengths.shape[0]
    owner = np.empty(S, np.int32)
    ld = np.empty(world, np.int64)
    rc = lib.rvq_oracle_balance(_p(lengths, ctypes.c_int64), S, int(world), _p(owner, ctypes.c_int32),
                                _p(ld, ctypes.c_int64))
    if rc != 0:
        raise OracleError(rc)
    return owner, ld
