"""fp64 CPU oracle for prefix-aware decode attention.

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` are the only
callers.  The product path never imports this package, and this package never
imports the product package.

The arithmetic lives in ``oracle.c`` (plain C, double precision): the attention
formula of the PAT review (section 三, 核心公式) applied to each request and head
over its full paged KV, plus the log-sum-exp merge of partial results (the
review's Merge stage).  Parity status of each function, and what pins it:

  oracle_attend_dense   pinned: torch fp64 scaled_dot_product_attention,
                        closed forms (two keys, identical keys, single key),
                        hand-derived golden cases, invariants.
  oracle_merge          pinned: merge of any split equals the unsplit result,
                        closed form of two one-key parts.
  oracle_attend_paged   pinned: dense gather done independently in numpy, then
                        torch fp64 SDPA; GQA head mapping by explicit repeat.
  attend_rows           (a later workload: a chunk of new tokens appended to a
                        session's persistent KV, each attending causally)
                        pinned: torch fp64 SDPA with an explicit causal mask
                        over the gathered context + chunk, the decode special
                        case, invariance to the order of context tokens.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so (gcc -O2; no fast-math, no FMA contraction)."""
    src = os.path.join(_HERE, "oracle.c")
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(src):
        tmp = "%s.%d.tmp" % (_LIB, os.getpid())  # ranks started together may both build
        subprocess.check_call(["gcc", "-O2", "-std=c99", "-ffp-contract=off", "-fPIC", "-shared",
                               "-pthread", src, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _l():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        vp, i32, i64, dbl = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_double
        lib.oracle_attend_dense.argtypes = [i32, dbl, vp, vp, vp, i64, vp, vp]
        lib.oracle_attend_dense.restype = None
        lib.oracle_merge.argtypes = [i32, i32, vp, vp, vp, vp]
        lib.oracle_merge.restype = None
        lib.oracle_attend_paged.argtypes = [i32, i32, i32, i32, i32, dbl, vp, vp, vp, i64, vp, i32, vp,
                                            vp, i32, vp, vp, i32]
        lib.oracle_attend_paged.restype = ctypes.c_int
        _lib = lib
    return _lib


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def attend_dense(q, K, V, scale=None):
    """One query row over dense keys, all float64.  Returns (out[D], lse)."""
    q = _c(q, np.float64)
    K = _c(K, np.float64)
    V = _c(V, np.float64)
    D = q.shape[0]
    n = K.shape[0]
    if scale is None:
        scale = 1.0 / np.sqrt(D)
    out = np.empty(D, dtype=np.float64)
    lse = np.empty(1, dtype=np.float64)
    _l().oracle_attend_dense(D, float(scale), q.ctypes.data, K.ctypes.data, V.ctypes.data, n,
                             out.ctypes.data, lse.ctypes.data)
    return out, float(lse[0])


def merge(o, lse):
    """Merge partial results o[n][D], lse[n] of one row.  Returns (out[D], lse)."""
    o = _c(o, np.float64)
    lse = _c(lse, np.float64)
    n, D = o.shape
    out = np.empty(D, dtype=np.float64)
    L = np.empty(1, dtype=np.float64)
    _l().oracle_merge(D, n, o.ctypes.data, lse.ctypes.data, out.ctypes.data, L.ctypes.data)
    return out, float(L[0])


def attend_paged(q, k_pool, v_pool, block_table, kv_lens, scale=None, queries=None, nthreads=None):
    """Paged decode attention in fp64.

    q uint16[B][Hq][D]; pools uint16[num_pages][Hkv][P][D]; block_table int32[B][max_pages];
    kv_lens int32[B].  Returns (out float64[n][Hq][D], lse float64[n][Hq]) for the requested
    queries (all by default).
    """
    q = _c(q, np.uint16)
    k_pool = _c(k_pool, np.uint16)
    v_pool = _c(v_pool, np.uint16)
    bt = _c(block_table, np.int32)
    kl = _c(kv_lens, np.int32)
    B, Hq, D = q.shape
    num_pages, Hkv, P, _ = k_pool.shape
    if queries is None:
        qs = np.arange(B, dtype=np.int32)
    else:
        qs = _c(queries, np.int32)
    n = len(qs)
    out = np.empty((n, Hq, D), dtype=np.float64)
    lse = np.empty((n, Hq), dtype=np.float64)
    if nthreads is None:
        nthreads = os.cpu_count() or 1
    rc = _l().oracle_attend_paged(B, Hq, Hkv, D, P, float(scale or 0.0), q.ctypes.data, k_pool.ctypes.data,
                                  v_pool.ctypes.data, num_pages, bt.ctypes.data, bt.shape[1], kl.ctypes.data,
                                  qs.ctypes.data, n, out.ctypes.data, lse.ctypes.data, int(nthreads))
    if rc != 0:
        raise ValueError("oracle_attend_paged: invalid arguments")
    return out, lse


def attend_rows(q_rows, row_req, row_pos, k_pool, v_pool, block_table, scale=None, nthreads=None):
    """Attention of query rows over a prefix of their request's paged KV, fp64.

    Row r belongs to request row_req[r] and sits at token position row_pos[r]
    of it; it attends over that request's tokens 0 .. row_pos[r] (its own
    included), all already in the paged cache.  A chunk of C new tokens
    appended to a session of L tokens is C rows at positions L .. L + C - 1
    (causal inside the chunk; the persistent context before it); a decode
    token is the row at position kv_len - 1.  This is the stateful-session
    workload of "Attention Once Is All You Need" (new data advances the
    session's KV; a query consumes it), with the PAT review's formula per row.

    q_rows uint16[N][Hq][D]; row_req, row_pos int[N]; pools and block_table as
    for attend_paged.  Returns (out float64[N][Hq][D], lse float64[N][Hq]).
    Each row is the paged decode attention of a one-row batch whose block
    table row is its request's and whose length is row_pos + 1.
    """
    bt = _c(block_table, np.int32)
    req = np.asarray(row_req, dtype=np.int64)
    pos = np.asarray(row_pos, dtype=np.int64)
    if len(req) != len(pos) or len(req) != len(q_rows):
        raise ValueError("attend_rows: q_rows, row_req and row_pos differ in length")
    if (pos < 0).any() or (pos >= bt.shape[1] * k_pool.shape[2]).any():
        raise ValueError("attend_rows: row position outside the block table")
    rows_bt = np.ascontiguousarray(bt[req])
    rows_len = (pos + 1).astype(np.int32)
    return attend_paged(q_rows, k_pool, v_pool, rows_bt, rows_len, scale=scale, nthreads=nthreads)
