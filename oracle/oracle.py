"""ctypes front end of the fp64 CPU oracle (``smla_oracle.c``).

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this module.  The product path
(the CUDA library and its binding) never imports, links or calls it, and this
module imports nothing from the product package.

Inputs are numpy arrays: bf16 tensors travel as their raw ``uint16`` bit
patterns, indices and page tables as ``int32``.  Outputs are float64.

The definition the oracle follows, with its sources, is in the header of
``smla_oracle.c``; the pins that check it are in ``tests/test_oracle_pins.py``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "smla_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libsmla_oracle.so")
_lib = None

DC = 512
DR = 64
PAGE_SIZE = 64


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (fp64, IEEE semantics, OpenMP)."""
    if force or not os.path.exists(_LIB_PATH) or (
        os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC)
    ):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11",
               _SRC, "-o", tmp, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _bind(lib):
    P = ctypes.c_void_p
    i32, i64, dbl = ctypes.c_int, ctypes.c_int64, ctypes.c_double
    lib.smla_oracle_decode.argtypes = [P, P, P, i32, i64, P, i32, i32, i32, i32,
                                       i32, i32, i32, dbl, P, P]
    lib.smla_oracle_decode.restype = ctypes.c_long
    lib.smla_oracle_partial.argtypes = [P, P, P, i32, i64, P, i32, i32, i32, i32,
                                        i32, i32, i32, dbl, i32, P, P, P]
    lib.smla_oracle_partial.restype = ctypes.c_long
    lib.smla_oracle_combine.argtypes = [P, P, P, ctypes.c_long, i32, i32, P, P]
    lib.smla_oracle_combine.restype = None
    lib.smla_oracle_max_threads.argtypes = []
    lib.smla_oracle_max_threads.restype = i32
    lib.smla_oracle_set_threads.argtypes = [i32]
    lib.smla_oracle_set_threads.restype = None
    return lib


def load_library(path: str):
    """Load an oracle build from ``path`` (the tests also load planted-mistake
    builds this way, to show that the pins catch them)."""
    return _bind(ctypes.CDLL(path))


def _load(lib=None):
    global _lib
    if lib is not None:
        return lib
    if _lib is None:
        _lib = load_library(build())
    return _lib


def max_threads() -> int:
    return int(_load().smla_oracle_max_threads())


def set_threads(n: int) -> None:
    _load().smla_oracle_set_threads(int(n))


def _c(a, dtype):
    a = np.ascontiguousarray(a, dtype=dtype)
    return a, a.ctypes.data_as(ctypes.c_void_p)


def _check_inputs(q, cache, page_table, idx, dc, dr, page_size):
    q = np.asarray(q)
    cache = np.asarray(cache)
    idx = np.asarray(idx)
    page_table = np.asarray(page_table)
    D = dc + dr
    if q.ndim != 4 or q.shape[-1] != D:
        raise ValueError(f"q must be [B,T,H,{D}] bf16 bits, got {q.shape}")
    B, T, H, _ = q.shape
    if idx.shape[:2] != (B, T) or idx.ndim != 3:
        raise ValueError(f"idx must be [B,T,K], got {idx.shape}")
    if page_table.ndim != 2 or page_table.shape[0] != B:
        raise ValueError(f"page_table must be [B, pt_stride], got {page_table.shape}")
    rows = cache.reshape(-1, D).shape[0]
    if rows % page_size:
        raise ValueError("cache rows must be a whole number of pages")
    return B, T, H, idx.shape[2], page_table.shape[1], rows // page_size


def decode(q, cache, page_table, idx, scale, *, dc=DC, dr=DR, page_size=PAGE_SIZE,
           lib=None):
    """Unsplit decode. Returns (o [B,T,H,dc] f64, lse [B,T,H] f64, n_bad)."""
    lib = _load(lib)
    B, T, H, K, pt_stride, num_pages = _check_inputs(q, cache, page_table, idx,
                                                     dc, dr, page_size)
    q, qp = _c(q, np.uint16)
    cache, cp = _c(cache, np.uint16)
    page_table, ptp = _c(page_table, np.int32)
    idx, ip = _c(idx, np.int32)
    o = np.zeros((B, T, H, dc), np.float64)
    lse = np.zeros((B, T, H), np.float64)
    n_bad = lib.smla_oracle_decode(qp, cp, ptp, pt_stride, num_pages, ip, B, T, H,
                                   K, dc, dr, page_size, float(scale),
                                   o.ctypes.data_as(ctypes.c_void_p),
                                   lse.ctypes.data_as(ctypes.c_void_p))
    return o, lse, int(n_bad)


def partial(q, cache, page_table, idx, scale, nsplit, *, dc=DC, dr=DR,
            page_size=PAGE_SIZE, lib=None):
    """Split-K partials: (part_o [B,T,H,S,dc], part_m [B,T,H,S], part_lse, n_bad)."""
    if nsplit < 1:
        raise ValueError("nsplit must be >= 1")
    lib = _load(lib)
    B, T, H, K, pt_stride, num_pages = _check_inputs(q, cache, page_table, idx,
                                                     dc, dr, page_size)
    q, qp = _c(q, np.uint16)
    cache, cp = _c(cache, np.uint16)
    page_table, ptp = _c(page_table, np.int32)
    idx, ip = _c(idx, np.int32)
    po = np.zeros((B, T, H, nsplit, dc), np.float64)
    pm = np.zeros((B, T, H, nsplit), np.float64)
    pl = np.zeros((B, T, H, nsplit), np.float64)
    n_bad = lib.smla_oracle_partial(qp, cp, ptp, pt_stride, num_pages, ip, B, T, H,
                                    K, dc, dr, page_size, float(scale), int(nsplit),
                                    po.ctypes.data_as(ctypes.c_void_p),
                                    pm.ctypes.data_as(ctypes.c_void_p),
                                    pl.ctypes.data_as(ctypes.c_void_p))
    return po, pm, pl, int(n_bad)


def combine(part_o, part_m, part_lse, *, lib=None):
    """LSE combine over the split axis: (o [..., dc], lse [...])."""
    lib = _load(lib)
    part_o = np.ascontiguousarray(part_o, np.float64)
    part_m = np.ascontiguousarray(part_m, np.float64)
    part_lse = np.ascontiguousarray(part_lse, np.float64)
    lead = part_m.shape[:-1]
    nsplit = part_m.shape[-1]
    dc = part_o.shape[-1]
    if part_o.shape != lead + (nsplit, dc) or part_lse.shape != part_m.shape:
        raise ValueError("partial shapes disagree")
    n_units = int(np.prod(lead)) if lead else 1
    o = np.zeros(lead + (dc,), np.float64)
    lse = np.zeros(lead, np.float64)
    lib.smla_oracle_combine(part_o.ctypes.data_as(ctypes.c_void_p),
                            part_m.ctypes.data_as(ctypes.c_void_p),
                            part_lse.ctypes.data_as(ctypes.c_void_p),
                            n_units, nsplit, dc,
                            o.ctypes.data_as(ctypes.c_void_p),
                            lse.ctypes.data_as(ctypes.c_void_p))
    return o, lse


def dense_positions(seq_lens, K):
    """Index lists of the dense-context (KV-split verify) variant: query token
    (b, t) attends to every position 0 .. seq_lens[b, t] - 1 of its sequence,
    so its list is those positions followed by -1 up to width K.

    "The Occupancy Hypothesis: How One Kernel Parameter Unlocked 1.8x Decode
    Speedup on Blackwell", sections "The Occupancy Insight" and "The Broader
    Context": the verify kernel divides each query token's whole KV sequence
    into NSPLIT splits (2875 tokens per split at 46K and NSPLIT 16), with a
    partial pass and a reduce.  The visible prefix length is an input.
    """
    seq_lens = np.asarray(seq_lens, np.int64)
    if seq_lens.ndim != 2:
        raise ValueError("seq_lens must be [B, T]")
    if seq_lens.size and (seq_lens.min() < 0 or seq_lens.max() > K):
        raise ValueError("seq_lens must lie in [0, K]")
    j = np.arange(K, dtype=np.int64)
    return np.where(j[None, None, :] < seq_lens[..., None], j, -1).astype(np.int32)


def decode_dense(q, cache, page_table, seq_lens, scale, *, K=None, dc=DC, dr=DR,
                 page_size=PAGE_SIZE, lib=None):
    """Dense-context decode: the sparse definition over each query token's
    full visible prefix (``dense_positions``).  Returns (o, lse, n_bad)."""
    seq_lens = np.asarray(seq_lens, np.int64)
    if K is None:
        K = int(seq_lens.max()) if seq_lens.size else 0
    return decode(q, cache, page_table, dense_positions(seq_lens, K), scale, dc=dc, dr=dr,
                  page_size=page_size, lib=lib)

