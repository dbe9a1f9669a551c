"""fp64 CPU oracle of the DashAttention forward pass -- TEST INFRASTRUCTURE.

Only the test-suite, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product library never does, and
the two share no code: this package wraps ``dash_oracle.c`` (plain C, double
precision, OpenMP) with ctypes and numpy, and ``backward.py`` differentiates that
forward (numpy, double precision).

Every function follows "DashAttention: Differentiable and Adaptive Sparse
Hierarchical Attention" (arXiv 2605.18753); the C file cites the section and
equation of each step.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from pathlib import Path

import numpy as np

_HERE = Path(__file__).resolve().parent
_SRC = _HERE / "dash_oracle.c"
_LIB = _HERE / "libdash_oracle.so"
_lib = None


def build(force: bool = False) -> Path:
    """Compile dash_oracle.c into libdash_oracle.so next to it (gcc, -O2, OpenMP)."""
    if force or not _LIB.exists() or _LIB.stat().st_mtime < _SRC.stat().st_mtime:
        tmp = _LIB.with_suffix(".so.tmp%d" % os.getpid())
        cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", "-fvisibility=hidden",
               str(_SRC), "-o", str(tmp), "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        # tests/test_oracle_mutations.py points this at a deliberately broken copy
        override = os.environ.get("DASH_ORACLE_LIB")
        if override:
            lib = ctypes.CDLL(override)
        else:
            build()
            lib = ctypes.CDLL(str(_LIB))
        P = ctypes.c_void_p
        i64, i32, f64 = ctypes.c_int64, ctypes.c_int, ctypes.c_double
        lib.dash_oracle_entmax_sort.argtypes = [P, i32, f64, P, P, P]
        lib.dash_oracle_entmax_bisect.argtypes = [P, i32, f64, i32, P, P]
        lib.dash_oracle_pool.argtypes = [P, i64, i32, i32, i32, i32, P]
        lib.dash_oracle_pool_q.argtypes = [P, P, i64, i32, i32, i32, i32, P]
        lib.dash_oracle_pool.restype = None
        lib.dash_oracle_fwd_rows.argtypes = [P, P, i64, i64, P, P, i64, i32, i32, i32, i32, f64, f64, f64,
                                             i32, i32, P, P, P, P, P, P, P, P]
        lib.dash_oracle_fwd_rows_q.argtypes = [P, P, i64, i64, P, P, i64, i32, i32, i32, i32, f64, f64, f64, i32,
                                               i32, P, P, P, i32, P, P, P, P, P, P]
        lib.dash_oracle_dense_attention.argtypes = [P, i64, P, P, i64, i32, i32, i32, i32, P]
        lib.dash_oracle_set_threads.argtypes = [i32]
        lib.dash_oracle_set_threads.restype = None
        lib.dash_oracle_max_threads.restype = i32
        _lib = lib
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _f64(a):
    return np.ascontiguousarray(a, dtype=np.float64)


def _f32(a):
    return np.ascontiguousarray(a, dtype=np.float32)


def set_threads(n: int) -> None:
    _load().dash_oracle_set_threads(int(n))


def max_threads() -> int:
    return int(_load().dash_oracle_max_threads())


def entmax_sort(s, alpha: float):
    """alpha-entmax of a 1-D score vector by the sort-based exact threshold.

    Returns (p, tau, support_size); tau is in the (alpha-1)*s domain."""
    s = _f64(s)
    p = np.empty_like(s)
    tau = ctypes.c_double()
    ks = ctypes.c_int()
    rc = _load().dash_oracle_entmax_sort(_ptr(s), s.size, float(alpha), _ptr(p), ctypes.byref(tau),
                                         ctypes.byref(ks))
    if rc:
        raise ValueError("entmax_sort rejected its input (rc=%d)" % rc)
    return p, tau.value, ks.value


def entmax_bisect(s, alpha: float, iters: int = 200):
    """alpha-entmax by plain bisection on [max-1, max-n^(1-alpha)]; returns (p, tau)."""
    s = _f64(s)
    p = np.empty_like(s)
    tau = ctypes.c_double()
    rc = _load().dash_oracle_entmax_bisect(_ptr(s), s.size, float(alpha), int(iters), _ptr(p),
                                           ctypes.byref(tau))
    if rc:
        raise ValueError("entmax_bisect rejected its input (rc=%d)" % rc)
    return p, tau.value


def pool(K, block_size: int, n_chunks: int | None = None):
    """Chunk means of K [nk, hkv, d] -> [n_chunks, hkv, d] (float64)."""
    K = _f32(K)
    nk, hkv, d = K.shape
    if n_chunks is None:
        n_chunks = nk // block_size
    out = np.empty((n_chunks, hkv, d), dtype=np.float64)
    _load().dash_oracle_pool(_ptr(K), nk, hkv, d, int(block_size), int(n_chunks), _ptr(out))
    return out


def pool_q(K, Qbar, block_size: int, n_chunks: int | None = None):
    """Learned-query chunk summaries: K [nk, hkv, d], Qbar [n_chunks, hkv, d] ->
    [n_chunks, hkv, d] (float64), softmax(<q̄_c, k_t>/sqrt(d)) weights over each chunk."""
    K = _f32(K)
    nk, hkv, d = K.shape
    if n_chunks is None:
        n_chunks = nk // block_size
    Qbar = _f32(np.broadcast_to(np.asarray(Qbar, dtype=np.float32), (n_chunks, hkv, d)))
    out = np.empty((n_chunks, hkv, d), dtype=np.float64)
    _load().dash_oracle_pool_q(_ptr(K), _ptr(Qbar), nk, hkv, d, int(block_size), int(n_chunks), _ptr(out))
    return out


def n_chunks_for(nk: int, block_size: int, causal: bool) -> int:
    return nk // block_size if causal else -(-nk // block_size)


def fwd_rows(Q_rows, rows, nq: int, K, V, block_size: int, alpha: float, *, gamma: float = 1.0,
             sigma: float = 1e8, causal: bool = True, route: int = 0, w_in=None, r_in=None,
             want=("out", "tau", "w", "routed"), qbar=None, local: int = 1):
    """Oracle forward for selected query rows of ONE batch element.

    Q_rows [nrows, hq, d] are the rows' query vectors, rows [nrows] their
    indices in [0, nq); K, V are [nk, hkv, d].  qbar [n_chunks, hkv, d] (or a
    shape that broadcasts to it): learned Stage-0 summary queries (None: q̄ = 0,
    mean pooling).  local: chunks of the local window (1: the query's own chunk; 2: it
    and the one before, App. B.1.1).  Returns a dict with the
    requested outputs among out, tau, w, routed, xmt, lambda (see the C file).
    """
    lib = _load()
    Q_rows = _f32(Q_rows)
    K = _f32(K)
    V = _f32(V)
    rows = np.ascontiguousarray(rows, dtype=np.int64)
    nrows, hq, d = Q_rows.shape
    nk, hkv, d2 = K.shape
    assert d2 == d and V.shape == K.shape and rows.shape == (nrows,)
    nch = n_chunks_for(nk, block_size, causal)
    res = {}
    res["out"] = np.empty((nrows, hq, d)) if "out" in want else None
    res["tau"] = np.empty((nrows, hq)) if "tau" in want else None
    res["w"] = np.empty((nrows, hkv, nch)) if "w" in want else None
    res["routed"] = np.empty((nrows, hkv, nch), dtype=np.uint8) if "routed" in want else None
    res["xmt"] = np.empty((nrows, hq, nch)) if "xmt" in want else None
    res["lambda"] = np.empty((nrows, hq)) if "lambda" in want else None
    if w_in is not None:
        w_in = _f64(w_in).reshape(nrows, hkv, nch)
        r_in = np.ascontiguousarray(r_in, dtype=np.uint8).reshape(nrows, hkv, nch)
    if qbar is not None or local != 1:
        qb = None if qbar is None else _f32(np.broadcast_to(np.asarray(qbar, dtype=np.float32), (nch, hkv, d)))
        rc = lib.dash_oracle_fwd_rows_q(_ptr(Q_rows), _ptr(rows), nrows, int(nq), _ptr(K), _ptr(V), nk, hq, hkv,
                                        d, int(block_size), float(alpha), float(gamma), float(sigma),
                                        int(bool(causal)), int(route), _ptr(w_in), _ptr(r_in), _ptr(qb), int(local),
                                        _ptr(res["out"]), _ptr(res["tau"]), _ptr(res["w"]), _ptr(res["routed"]),
                                        _ptr(res["xmt"]), _ptr(res["lambda"]))
        if rc:
            raise ValueError("oracle fwd_rows_q rejected its input (rc=%d)" % rc)
        return {k: v for k, v in res.items() if v is not None}
    rc = lib.dash_oracle_fwd_rows(_ptr(Q_rows), _ptr(rows), nrows, int(nq), _ptr(K), _ptr(V), nk, hq, hkv, d,
                                  int(block_size), float(alpha), float(gamma), float(sigma), int(bool(causal)),
                                  int(route), _ptr(w_in), _ptr(r_in), _ptr(res["out"]), _ptr(res["tau"]),
                                  _ptr(res["w"]), _ptr(res["routed"]), _ptr(res["xmt"]), _ptr(res["lambda"]))
    if rc:
        raise ValueError("oracle fwd_rows rejected its input (rc=%d)" % rc)
    return {k: v for k, v in res.items() if v is not None}


def fwd(Q, K, V, block_size: int, alpha: float, **kw):
    """Oracle forward of every row of one batch element: Q [nq, hq, d]."""
    Q = _f32(Q)
    rows = np.arange(Q.shape[0], dtype=np.int64)
    return fwd_rows(Q, rows, Q.shape[0], K, V, block_size, alpha, **kw)


def dense_attention(Q, K, V, causal: bool = True):
    """Dense (causal, bottom-right aligned) softmax attention in fp64 for one batch element."""
    Q = _f32(Q)
    K = _f32(K)
    V = _f32(V)
    nq, hq, d = Q.shape
    nk, hkv, _ = K.shape
    out = np.empty((nq, hq, d))
    rc = _load().dash_oracle_dense_attention(_ptr(Q), nq, _ptr(K), _ptr(V), nk, hq, hkv, d,
                                             int(bool(causal)), _ptr(out))
    if rc:
        raise ValueError("dense_attention rejected its input")
    return out
