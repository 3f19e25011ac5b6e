"""ctypes front end of the fp64 top-k indexer oracle (``smla_indexer_oracle.c``).

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and
the CPU legs of ``bench.py`` may import this module; the product path never
imports, links or calls it, and it imports nothing from the product package.

bf16 tensors travel as raw ``uint16`` bit patterns, ``w`` as float32, page
tables and lengths as int32.  The definition, its sources and the tie rule
are in the header of ``smla_indexer_oracle.c``; the pins that check it are in
``tests/test_indexer_oracle.py``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(_HERE, "smla_indexer_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libsmla_indexer_oracle.so")
_lib = None

PAGE_SIZE = 64


def build(force: bool = False, src: str = SRC, out: str = _LIB_PATH) -> str:
    """Compile the indexer oracle with gcc (fp64, IEEE semantics, OpenMP)."""
    if force or not os.path.exists(out) or os.path.getmtime(out) < os.path.getmtime(src):
        tmp = out + f".tmp{os.getpid()}"
        subprocess.run(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", src, "-o", tmp,
                        "-lm"], check=True)
        os.replace(tmp, out)
    return out


def load_library(path: str):
    """Load an indexer-oracle build from ``path`` (the tests also load
    planted-mistake builds this way)."""
    lib = ctypes.CDLL(path)
    P, i32, i64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64
    lib.smla_ix_oracle_scores.argtypes = [P, P, P, P, i32, i64, P, i32, i32, i32, i32, i32, i32,
                                          P]
    lib.smla_ix_oracle_scores.restype = ctypes.c_long
    lib.smla_ix_oracle_topk.argtypes = [P, P, P, P, i32, i64, P, i32, i32, i32, i32, i32, i32, P]
    lib.smla_ix_oracle_topk.restype = ctypes.c_long
    lib.smla_ix_oracle_select.argtypes = [P, P, i32, i32, i32, P]
    lib.smla_ix_oracle_select.restype = None
    return lib


def _load(lib=None):
    global _lib
    if lib is not None:
        return lib
    if _lib is None:
        _lib = load_library(build())
    return _lib


def _args(q_bits, w, k_bits, page_table, n_vis, page_size):
    q = np.ascontiguousarray(q_bits, np.uint16)
    w = np.ascontiguousarray(w, np.float32)
    k = np.ascontiguousarray(k_bits, np.uint16)
    pt = np.ascontiguousarray(page_table, np.int32)
    n = np.ascontiguousarray(n_vis, np.int32)
    if q.ndim != 4:
        raise ValueError("qI must be [B, T, HI, DI] bf16 bits")
    B, T, HI, DI = q.shape
    if w.shape != (B, T, HI):
        raise ValueError("w must be [B, T, HI]")
    if n.shape != (B, T):
        raise ValueError("n_vis must be [B, T]")
    if pt.ndim != 2 or pt.shape[0] != B:
        raise ValueError("page_table must be [B, pt_stride]")
    rows = k.reshape(-1, DI).shape[0]
    if rows % page_size:
        raise ValueError("index-key rows must be a whole number of pages")
    return q, w, k, pt, n, (B, T, HI, DI, pt.shape[1], rows // page_size)


def _p(a):
    return a.ctypes.data_as(ctypes.c_void_p)


def scores(q_bits, w, k_bits, page_table, n_vis, *, page_size=PAGE_SIZE, lib=None):
    """Index scores I [B, T, max n] (fp64; -inf past each token's visible
    length and at positions that are not candidates) and the count of visible
    positions that are not candidates."""
    lib = _load(lib)
    q, w, k, pt, n, (B, T, HI, DI, pt_stride, num_pages) = _args(q_bits, w, k_bits, page_table,
                                                                 n_vis, page_size)
    n_max = int(n.max()) if n.size else 0
    out = np.zeros((B, T, max(n_max, 1)), np.float64)
    bad = lib.smla_ix_oracle_scores(_p(q), _p(w), _p(k), _p(pt), pt_stride, num_pages, _p(n), B,
                                    T, HI, DI, page_size, max(n_max, 1), _p(out))
    return out[:, :, :n_max], int(bad)


def topk(q_bits, w, k_bits, page_table, n_vis, K, *, page_size=PAGE_SIZE, lib=None):
    """The selected positions [B, T, K] int32 (ascending, then -1) and the
    count of visible positions that are not candidates."""
    lib = _load(lib)
    q, w, k, pt, n, (B, T, HI, DI, pt_stride, num_pages) = _args(q_bits, w, k_bits, page_table,
                                                                 n_vis, page_size)
    out = np.zeros((B, T, K), np.int32)
    bad = lib.smla_ix_oracle_topk(_p(q), _p(w), _p(k), _p(pt), pt_stride, num_pages, _p(n), B, T,
                                  HI, DI, page_size, int(K), _p(out))
    return out, int(bad)


def select(scores, n_vis, K, *, lib=None):
    """The selection rule applied to given scores [B, T, n_max] (any float
    dtype, widened exactly to fp64; NaN marks a position that is not a
    candidate): [B, T, K] int32, ascending positions then -1."""
    lib = _load(lib)
    sc = np.ascontiguousarray(scores, np.float64)
    n = np.ascontiguousarray(n_vis, np.int32)
    if sc.ndim != 3 or n.shape != sc.shape[:2]:
        raise ValueError("scores must be [B, T, n_max] and n_vis [B, T]")
    B, T, n_max = sc.shape
    out = np.zeros((B, T, K), np.int32)
    lib.smla_ix_oracle_select(_p(sc), _p(n), B * T, n_max, int(K), _p(out))
    return out
