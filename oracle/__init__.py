"""ctypes front of the CPU oracle (oracle.c).

TEST INFRASTRUCTURE ONLY: the plain, slow double-precision restatement of
the lightning indexer + top-k (dense, PIVOT Reuse/Refine/block pre-filter,
decode) and of the token-sparse attention over the selected positions that
the CUDA library is checked against.  ``oracle.adaptive`` restates the
adaptive top-k budget from the cutoff margin in numpy.  Only the tests, ``__graft_entry__.smoke``
and the benchmark's CPU-baseline leg may import this package.  It imports
nothing from the product package and the product imports nothing from it.

Array conventions: bf16 tensors are numpy ``uint16`` bit patterns, fp32
tensors are ``float32``; indices are int32; -1 pads a short top-k.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from . import build as _build

BF16, F32 = 0, 1
DENSE, REUSE, REFINE, BLOCK, QUEST = 0, 1, 2, 3, 4

_libs = {}
_active = [None]


def load(path: str) -> ctypes.CDLL:
    """Load an oracle shared library (the default one, or a test-built variant)."""
    if path not in _libs:
        L = ctypes.CDLL(path)
        vp, fp, ip, dp, llp = (ctypes.c_void_p, ctypes.POINTER(ctypes.c_float),
                               ctypes.POINTER(ctypes.c_int), ctypes.POINTER(ctypes.c_double),
                               ctypes.POINTER(ctypes.c_longlong))
        i, ll = ctypes.c_int, ctypes.c_longlong
        L.ora_score_row.argtypes = [vp, vp, fp, i, i, i, ll, ll, i, dp]
        L.ora_select.argtypes = [dp, ip, i, i, ip]
        L.ora_group_proxy.argtypes = [vp, fp, i, i, i, ll, i, vp, fp]
        L.ora_dense_topk.argtypes = [vp, vp, fp, i, ip, i, i, i, i, llp, i, ip, i]
        L.ora_block_mean.argtypes = [vp, i, i, ll, i, vp]
        L.ora_pivot_topk.argtypes = [vp, vp, fp, i, ip, i, i, i, i, i, i, i, i, i, llp, i, ip, i]
        L.ora_decode_topk.argtypes = [vp, vp, fp, i, ip, i, i, i, i, i, i, i, i, i, llp, i, ip, i]
        L.ora_sparse_attn.argtypes = [vp, vp, i, ip, ip, ip, i, i, i, i, i, ctypes.c_double, llp, i, dp, dp, i]
        for f in (L.ora_score_row, L.ora_select, L.ora_group_proxy, L.ora_block_mean, L.ora_dense_topk,
                  L.ora_pivot_topk, L.ora_decode_topk, L.ora_sparse_attn):
            f.restype = ctypes.c_int
        _libs[path] = L
    return _libs[path]


def lib() -> ctypes.CDLL:
    """The library every function below calls (liboracle.so unless switched)."""
    if _active[0] is None:
        _active[0] = load(_build.build())
    return _active[0]


class use:
    """Context manager: route this module's functions to another oracle build."""

    def __init__(self, path: str):
        self.L = load(path)

    def __enter__(self):
        self.prev = _active[0]
        _active[0] = self.L
        return self

    def __exit__(self, *exc):
        _active[0] = self.prev


def _threads(n):
    return int(n) if n else (os.cpu_count() or 1)


def _dtype_code(a: np.ndarray) -> int:
    if a.dtype == np.uint16:
        return BF16
    if a.dtype == np.float32:
        return F32
    raise TypeError(f"oracle takes bf16 bit patterns (uint16) or float32, got {a.dtype}")


def _c(a, dt):
    a = np.ascontiguousarray(a, dtype=dt)
    return a


def _ptr(a, ct=None):
    return a.ctypes.data_as(ctypes.POINTER(ct)) if ct else a.ctypes.data_as(ctypes.c_void_p)


def _check(rc, what):
    if rc != 0:
        raise ValueError(f"oracle {what} rejected its arguments (rc={rc})")


def score_row(q, k, w, q_row: int, key0: int, n: int) -> np.ndarray:
    """I[q_row, key0+s] for s < n, in double.  q [R,H,d], k [*,d], w [R,H]."""
    q = np.ascontiguousarray(q); k = np.ascontiguousarray(k); w = _c(w, np.float32)
    dt = _dtype_code(q)
    assert _dtype_code(k) == dt
    R, H, d = q.shape
    out = np.empty(n, np.float64)
    _check(lib().ora_score_row(_ptr(q), _ptr(k), _ptr(w, ctypes.c_float), dt, H, d, q_row, key0, n,
                               _ptr(out, ctypes.c_double)), "score_row")
    return out


def select(scores, k: int, pos=None) -> np.ndarray:
    """Top-k by (score desc, position asc), listed in ascending position, -1 padded."""
    s = _c(scores, np.float64)
    out = np.empty(k, np.int32)
    p = _c(pos, np.int32) if pos is not None else None
    _check(lib().ora_select(_ptr(s, ctypes.c_double), _ptr(p, ctypes.c_int) if p is not None else None,
                            len(s), k, _ptr(out, ctypes.c_int)), "select")
    return out


def group_proxy(q, w, m0: int, cnt: int):
    """(qbar [H,d] in q's dtype, wbar [H] fp32) of members m0..m0+cnt-1."""
    q = np.ascontiguousarray(q); w = _c(w, np.float32)
    dt = _dtype_code(q)
    R, H, d = q.shape
    qbar = np.empty((H, d), q.dtype)
    wbar = np.empty(H, np.float32)
    _check(lib().ora_group_proxy(_ptr(q), _ptr(w, ctypes.c_float), dt, H, d, m0, cnt, _ptr(qbar),
                                 _ptr(wbar, ctypes.c_float)), "group_proxy")
    return qbar, wbar


def block_mean(k, r0: int, bn: int):
    """Mean key [d] (in k's dtype) of key rows r0 .. r0+bn-1 of k [*, d]."""
    k = np.ascontiguousarray(k)
    dt = _dtype_code(k)
    d = k.shape[1]
    out = np.empty(d, k.dtype)
    _check(lib().ora_block_mean(_ptr(k), dt, d, r0, bn, _ptr(out)), "block_mean")
    return out


def _rows(rows, total):
    if rows is None:
        rows = np.arange(total, dtype=np.int64)
    return _c(rows, np.int64)


def dense_topk(q, k, w, cu_seqlens, topk: int, rows=None, threads=None) -> np.ndarray:
    """Dense top-k of the given global rows (all rows by default): [nrows, topk]."""
    q = np.ascontiguousarray(q); k = np.ascontiguousarray(k); w = _c(w, np.float32)
    cu = _c(cu_seqlens, np.int32)
    dt = _dtype_code(q)
    T, H, d = q.shape
    r = _rows(rows, T)
    out = np.empty((len(r), topk), np.int32)
    _check(lib().ora_dense_topk(_ptr(q), _ptr(k), _ptr(w, ctypes.c_float), dt, _ptr(cu, ctypes.c_int),
                                len(cu) - 1, H, d, topk, _ptr(r, ctypes.c_longlong), len(r),
                                _ptr(out, ctypes.c_int), _threads(threads)), "dense_topk")
    return out


def pivot_topk(q, k, w, cu_seqlens, topk: int, g: int, c: int, mode: int, rows=None,
               threads=None, bn: int = 64, dense_below: int = 0) -> np.ndarray:
    """PIVOT Reuse (mode=REUSE), Refine (mode=REFINE) or Refine over block
    pre-filter candidates (block size bn; blocks ranked by their mean key,
    mode=BLOCK, or by the Quest min/max bound, mode=QUEST) top-k of member rows.
    Groups whose last member's prefix holds at most dense_below keys take the
    dense top-k (the guardrail; 0 = off)."""
    q = np.ascontiguousarray(q); k = np.ascontiguousarray(k); w = _c(w, np.float32)
    cu = _c(cu_seqlens, np.int32)
    dt = _dtype_code(q)
    T, H, d = q.shape
    r = _rows(rows, T)
    out = np.empty((len(r), topk), np.int32)
    _check(lib().ora_pivot_topk(_ptr(q), _ptr(k), _ptr(w, ctypes.c_float), dt, _ptr(cu, ctypes.c_int),
                                len(cu) - 1, H, d, topk, g, c, mode, bn, int(dense_below),
                                _ptr(r, ctypes.c_longlong),
                                len(r), _ptr(out, ctypes.c_int), _threads(threads)), "pivot_topk")
    return out


def decode_topk(q, kcache, w, kv_len, topk: int, c: int = 0, mode: int = DENSE, reqs=None,
                threads=None, bn: int = 64) -> np.ndarray:
    """Decode top-k: q [B,G,H,d], kcache [B,n_max,d], w [B,G,H] -> [nreqs,G,topk]."""
    q = np.ascontiguousarray(q); kc = np.ascontiguousarray(kcache); w = _c(w, np.float32)
    kv = _c(kv_len, np.int32)
    dt = _dtype_code(q)
    B, G, H, d = q.shape
    n_max = kc.shape[1]
    r = _rows(reqs, B)
    out = np.empty((len(r), G, topk), np.int32)
    _check(lib().ora_decode_topk(_ptr(q), _ptr(kc), _ptr(w, ctypes.c_float), dt, _ptr(kv, ctypes.c_int),
                                 B, G, n_max, H, d, topk, c, mode, bn, _ptr(r, ctypes.c_longlong), len(r),
                                 _ptr(out, ctypes.c_int), _threads(threads)), "decode_topk")
    return out


def sparse_attn(q, kv, idx, cu_q, cu_kv, Dv: int, scale: float, rows=None, threads=None):
    """Token-sparse attention of query rows over their listed kv positions:
    q [R, Ha, Dqk], kv [Nkv, Dqk], idx [R, topk] (-1 = none), cu_q / cu_kv the
    request boundaries over query rows and kv rows.  Returns (o [n, Ha, Dv],
    lse [n, Ha]) in float64."""
    q = np.ascontiguousarray(q); kv = np.ascontiguousarray(kv)
    ix = _c(idx, np.int32)
    cq, ck = _c(cu_q, np.int32), _c(cu_kv, np.int32)
    dt = _dtype_code(q)
    R, Ha, Dqk = q.shape
    topk = ix.shape[1]
    r = _rows(rows, R)
    o = np.empty((len(r), Ha, Dv), np.float64)
    lse = np.empty((len(r), Ha), np.float64)
    _check(lib().ora_sparse_attn(_ptr(q), _ptr(kv), dt, _ptr(ix, ctypes.c_int), _ptr(cq, ctypes.c_int),
                                 _ptr(ck, ctypes.c_int), len(cq) - 1, Ha, Dqk, Dv, topk, float(scale),
                                 _ptr(r, ctypes.c_longlong), len(r), _ptr(o, ctypes.c_double),
                                 _ptr(lse, ctypes.c_double), _threads(threads)), "sparse_attn")
    return o, lse
