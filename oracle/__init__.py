"""Plain fp64 CPU oracle for factorized sparse causal self-attention (ctypes front end).

TEST INFRASTRUCTURE ONLY: the test suite, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` are the only callers.  It shares no code with the CUDA library and never imports it.

The arithmetic lives in ``st_oracle.c`` (the plain definition: per-row scan of the page
predicates, scores, two-pass softmax, output, and plain-calculus gradients).  This module only
marshals numpy arrays.  Set kinds and head-mode numbers are documented in ``st_oracle.c``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "st_oracle.c")
LIB = os.path.join(HERE, "liboracle.so")

SA1, SA2, SU, FA1, FA2, FU = 1, 2, 3, 4, 5, 6
KIND_NAMES = {SA1: "sA1", SA2: "sA2", SU: "sU", FA1: "fA1", FA2: "fA2", FU: "fU"}
STRIDED, FIXED = 1, 2
ALTERNATING, MERGED, SINGLE_A1, SINGLE_A2 = 1, 2, 3, 4


def build(force: bool = False) -> str:
    """Compile st_oracle.c into liboracle.so next to it (gcc, -O2, OpenMP)."""
    if force or not os.path.exists(LIB) or os.path.getmtime(LIB) < os.path.getmtime(SRC):
        tmp = LIB + ".tmp%d" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c99", SRC,
                               "-o", tmp, "-lm"])
        os.replace(tmp, LIB)
    return LIB


_lib = None


def _L():
    global _lib
    if _lib is None:
        # ORACLE_LIB lets the mutation tests load a deliberately broken build of st_oracle.c.
        path = os.environ.get("ORACLE_LIB") or build()
        lib = ctypes.CDLL(path)
        i64, i32, p = ctypes.c_int64, ctypes.c_int, ctypes.c_void_p
        lib.oracle_allowed.argtypes = [i32, i64, i64, i64, i64, i64]
        lib.oracle_allowed.restype = i32
        lib.oracle_row_set.argtypes = [i32, i64, i64, i64, i64, p]
        lib.oracle_row_set.restype = i64
        lib.oracle_set_counts.argtypes = [i32, i64, i64, i64, i64, p]
        lib.oracle_head_kinds.argtypes = [i32, i32, i32, i64, i64, i64, p, p]
        lib.oracle_head_kinds.restype = i32
        common = [p, p, p, i64, i64, i64, i64, i64, p, p, i64, i64]
        lib.oracle_fwd.argtypes = common + [p, p]
        lib.oracle_fwd_rows.argtypes = common + [i64, p, p, p]
        lib.oracle_decode.argtypes = common + [i64, p, p]
        bcommon = [p, p, p, p, i64, i64, i64, i64, i64, p, p, i64, i64]
        lib.oracle_bwd.argtypes = bcommon + [p, p, p]
        lib.oracle_bwd_rows.argtypes = bcommon + [i64, p, p, p, p]
        lib.oracle_bwd_keys.argtypes = bcommon + [i64, p, p, p]
        lib.oracle_num_threads.restype = i32
        _lib = lib
    return _lib


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _f64(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def allowed(kind: int, i: int, j: int, l: int, c: int = 0, o: int = 0) -> bool:
    return bool(_L().oracle_allowed(kind, i, j, l, c, o))


def row_set(kind: int, i: int, l: int, c: int = 0, o: int = 0) -> np.ndarray:
    out = np.empty(i + 1, dtype=np.int64)
    cnt = _L().oracle_row_set(kind, i, l, c, o, _ptr(out))
    return out[:cnt].copy()


def set_counts(kind: int, n: int, l: int, c: int = 0, o: int = 0) -> np.ndarray:
    out = np.empty(n, dtype=np.int64)
    _L().oracle_set_counts(kind, n, l, c, o, _ptr(out))
    return out


def head_kinds(family: int, head_mode: int, num_heads: int, l: int, c: int = 0, step: int = 0):
    kind = np.empty(num_heads, dtype=np.int32)
    off = np.empty(num_heads, dtype=np.int64)
    rc = _L().oracle_head_kinds(family, head_mode, num_heads, l, c, step, _ptr(kind), _ptr(off))
    if rc != 0:
        raise ValueError("bad head-mode arguments")
    return kind, off


def _dims(q, k, v, do=None):
    """(B, H, n, d, e): q and k are [B, H, n, d], v (and do) [B, H, n, e]."""
    B, H, n, d = q.shape
    e = v.shape[-1]
    if k.shape != (B, H, n, d) or v.shape != (B, H, n, e) or (do is not None and do.shape != v.shape):
        raise ValueError("q, k must be [B, H, n, d] and v, dO [B, H, n, e]")
    return B, H, n, d, e


class Problem:
    """Per-head set kinds and offsets for one pattern.  Q and K are [B, H, n, d]; V, O and dO are
    [B, H, n, e] (e = d unless the query-key width is reduced)."""

    def __init__(self, family: int, head_mode: int, num_heads: int, l: int, c: int = 0,
                 step: int = 0):
        self.l, self.c = int(l), int(c)
        self.kind, self.off = head_kinds(family, head_mode, num_heads, l, c, step)

    @classmethod
    def from_kinds(cls, kinds, offs, l: int, c: int = 0) -> "Problem":
        p = cls.__new__(cls)
        p.l, p.c = int(l), int(c)
        p.kind = np.ascontiguousarray(np.asarray(kinds, dtype=np.int32))
        p.off = np.ascontiguousarray(np.asarray(offs, dtype=np.int64))
        return p

    def fwd(self, q, k, v):
        q, k, v = _f64(q), _f64(k), _f64(v)
        B, H, n, d, e = _dims(q, k, v)
        o = np.empty_like(v)
        lse = np.empty((B, H, n), dtype=np.float64)
        _L().oracle_fwd(_ptr(q), _ptr(k), _ptr(v), B, H, n, d, e, _ptr(self.kind), _ptr(self.off),
                        self.l, self.c, _ptr(o), _ptr(lse))
        return o, lse

    def fwd_rows(self, q, k, v, rows):
        """rows: flat indices (b*H + h)*n + i."""
        q, k, v = _f64(q), _f64(k), _f64(v)
        B, H, n, d, e = _dims(q, k, v)
        rows = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
        o = np.empty((len(rows), e), dtype=np.float64)
        lse = np.empty(len(rows), dtype=np.float64)
        _L().oracle_fwd_rows(_ptr(q), _ptr(k), _ptr(v), B, H, n, d, e, _ptr(self.kind),
                             _ptr(self.off), self.l, self.c, len(rows), _ptr(rows), _ptr(o),
                             _ptr(lse))
        return o, lse

    def decode(self, q, k, v, pos):
        """One query row per (batch, head) at position pos against the cache rows 0..pos.
        q: [B, H, d]; k: [B, H, n, d]; v: [B, H, n, e].  Returns o [B, H, e], lse [B, H]."""
        q, k, v = _f64(q), _f64(k), _f64(v)
        B, H, n, d = k.shape
        e = v.shape[-1]
        if q.shape != (B, H, d) or v.shape != (B, H, n, e) or not 0 <= pos < n:
            raise ValueError("q must be [B, H, d], v [B, H, n, e] and 0 <= pos < n")
        o = np.empty((B, H, e), dtype=np.float64)
        lse = np.empty((B, H), dtype=np.float64)
        _L().oracle_decode(_ptr(q), _ptr(k), _ptr(v), B, H, n, d, e, _ptr(self.kind), _ptr(self.off),
                           self.l, self.c, int(pos), _ptr(o), _ptr(lse))
        return o, lse

    def bwd(self, q, k, v, do):
        q, k, v, do = _f64(q), _f64(k), _f64(v), _f64(do)
        B, H, n, d, e = _dims(q, k, v, do)
        dq, dk, dv = np.empty_like(q), np.empty_like(k), np.empty_like(v)
        _L().oracle_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(do), B, H, n, d, e, _ptr(self.kind),
                        _ptr(self.off), self.l, self.c, _ptr(dq), _ptr(dk), _ptr(dv))
        return dq, dk, dv

    def bwd_rows(self, q, k, v, do, rows):
        """dQ (and lse, D) for flat query rows."""
        q, k, v, do = _f64(q), _f64(k), _f64(v), _f64(do)
        B, H, n, d, e = _dims(q, k, v, do)
        rows = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
        dq = np.empty((len(rows), d), dtype=np.float64)
        lse = np.empty(len(rows), dtype=np.float64)
        D = np.empty(len(rows), dtype=np.float64)
        _L().oracle_bwd_rows(_ptr(q), _ptr(k), _ptr(v), _ptr(do), B, H, n, d, e, _ptr(self.kind),
                             _ptr(self.off), self.l, self.c, len(rows), _ptr(rows), _ptr(dq),
                             _ptr(lse), _ptr(D))
        return dq, lse, D

    def bwd_keys(self, q, k, v, do, keys):
        """dK and dV for flat key rows."""
        q, k, v, do = _f64(q), _f64(k), _f64(v), _f64(do)
        B, H, n, d, e = _dims(q, k, v, do)
        keys = np.ascontiguousarray(np.asarray(keys, dtype=np.int64))
        dk = np.empty((len(keys), d), dtype=np.float64)
        dv = np.empty((len(keys), e), dtype=np.float64)
        _L().oracle_bwd_keys(_ptr(q), _ptr(k), _ptr(v), _ptr(do), B, H, n, d, e, _ptr(self.kind),
                             _ptr(self.off), self.l, self.c, len(keys), _ptr(keys), _ptr(dk),
                             _ptr(dv))
        return dk, dv


def num_threads() -> int:
    return int(_L().oracle_num_threads())
