"""ctypes binding of libsmla.so (the C ABI in include/smla.h).

Argument marshalling only: every step of the decode runs in the library's
CUDA kernels.  torch tensors supply device memory and the current stream.
If the library is missing, calls raise -- there is no fallback path.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libsmla.so")

DC, DR, D, PAGE_SIZE = 512, 64, 576, 64
MAX_HEADS, MAX_NSPLIT = 64, 1024
NOALLOC_SCRATCH_BYTES = 16 << 20
# Largest K (index-list width, dense longest visible length, indexer selection
# width): the library's split arithmetic (ceil(K / nsplit) rounded up to whole
# pages, then K + that split length) and its fill loops are 32-bit.  The
# library does not check this bound itself.
MAX_K = 2**30 - 64

STATUS = {
    0: "SMLA_OK", 1: "SMLA_ERR_INVALID_ARG", 2: "SMLA_ERR_UNSUPPORTED", 3: "SMLA_ERR_MISALIGNED",
    4: "SMLA_ERR_WORKSPACE_TOO_SMALL", 5: "SMLA_ERR_INDEX_RANGE", 6: "SMLA_ERR_CUDA",
    7: "SMLA_ERR_TIMEOUT",
}

# exported symbol -> (restype, argtypes)
_P, _I, _I64, _F, _SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_float, ctypes.c_size_t
SIGNATURES = {
    "smla_choose_nsplit": (_I, [_I, _I, _I, _I, _I]),
    "smla_workspace_bytes": (_SZ, [_I, _I, _I, _I]),
    "smla_decode_partial": (_I, [_P, _P, _I64, _P, _I, _P, _I, _I, _I, _I, _I, _F, _I, _P, _P, _P,
                                 _P]),
    "smla_lse_combine": (_I, [_P, _P, _P, _I, _I, _I, _I, _P, _P, _P]),
    "smla_decode": (_I, [_P, _P, _I64, _P, _I, _P, _I, _I, _I, _I, _I, _F, _I, _P, _SZ, _P, _P,
                         _P]),
    "smla_decode_partial_ws": (_I, [_P, _P, _I64, _P, _I, _P, _I, _I, _I, _I, _I, _F, _I, _P, _SZ,
                                    _P]),
    "smla_decode_noalloc": (_I, [_P, _P, _I64, _P, _I, _P, _I, _I, _I, _I, _I, _F, _I, _P, _P,
                                 _P]),
    "smla_workspace_host_bytes": (_SZ, [_I, _I, _I, _I, _I, _I]),
    "smla_decode_host": (_I, [_P, _P, _I64, _P, _I, _P, _I, _I, _I, _I, _I, _F, _I, _P, _SZ, _P, _P,
                              _P]),
    "smla_dense_nsplit": (_I, [_I, _I, _I, _I]),
    "smla_dense_workspace_bytes": (_SZ, [_I, _I, _I, _I, _I]),
    "smla_decode_dense": (_I, [_P, _P, _I64, _P, _I, _P, _I, _I, _I, _I, _I, _F, _I, _P, _SZ, _P,
                               _P, _P]),
    "smla_decode_dense_partial": (_I, [_P, _P, _I64, _P, _I, _P, _I, _I, _I, _I, _I, _F, _I, _P,
                                       _P, _P, _P]),
    "smla_indexer_workspace_bytes": (_SZ, [_I, _I, _I]),
    "smla_indexer_topk": (_I, [_P, _P, _P, _I64, _P, _I, _P, _I, _I, _I, _I, _I, _I, _P, _SZ, _P,
                               _P]),
    "smla_indexer_scores": (_I, [_P, _P, _P, _I64, _P, _I, _P, _I, _I, _I, _I, _I, _P, _SZ, _P,
                                 _P]),
    "smla_indexer_select": (_I, [_P, _P, _I, _I, _I, _I, _P, _SZ, _P, _P]),
    "smla_indexer_select_workspace_bytes": (_SZ, [_I, _I, _I]),
    "smla_selftest_wait_timeout": (_I, [ctypes.c_ulonglong, _P]),
    "smla_check_device": (_I, [_I, ctypes.POINTER(ctypes.c_ulonglong), _P]),
    "smla_status_string": (ctypes.c_char_p, [_I]),
    "smla_last_error": (ctypes.c_char_p, []),
    "smla_version": (_I, []),
}


class SmlaError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = f"{where}: {STATUS.get(status, status)}"
        if status == 6:
            msg += f" ({lib().smla_last_error().decode()})"
        super().__init__(msg)


_lib = None


def lib():
    """Load libsmla.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m sparse_mla_decode_partial_b200.build`")
        handle = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(handle, name)
            fn.restype = res
            fn.argtypes = args
        _lib = handle
    return _lib


def _k_in_range(K: int) -> int:
    if K > MAX_K:
        raise ValueError(f"K = {K} is above the library's limit {MAX_K}")
    return K


def _check(status: int, where: str):
    if status != 0:
        raise SmlaError(status, where)


def _stream(stream) -> Optional[int]:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else t.data_ptr()


def _need(t, dtype, name, device=None, shape=None):
    """Type, dtype, contiguity, shape (when given: the library reads or writes
    exactly that many elements through the pointer) and device of a tensor."""
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {list(shape)}, got {list(t.shape)}")
    _on_device(t, name, device)


def _on_device(t, name, device):
    if not t.is_cuda or (device is not None and t.device != device):
        raise ValueError(f"{name} must be a CUDA tensor on {device}")


def choose_nsplit(B: int, T: int, H: int, K: int, sm_count: int = 0) -> int:
    return int(lib().smla_choose_nsplit(B, T, H, _k_in_range(K), sm_count))


def workspace_bytes(B: int, T: int, H: int, nsplit: int) -> int:
    return int(lib().smla_workspace_bytes(B, T, H, nsplit))


def _decode_args(q, cache, page_table, idx):
    _need(q, torch.bfloat16, "q")
    dev = q.device
    _need(cache, torch.bfloat16, "cache", dev)
    _need(page_table, torch.int32, "page_table", dev)
    _need(idx, torch.int32, "idx", dev)
    if q.dim() != 4 or q.shape[-1] != D:
        raise ValueError(f"q must be [B,T,H,{D}]")
    B, T, H, _ = q.shape
    if idx.dim() != 3 or tuple(idx.shape[:2]) != (B, T):
        raise ValueError("idx must be [B,T,K]")
    if page_table.dim() != 2 or page_table.shape[0] != B:
        raise ValueError("page_table must be [B, pt_stride]")
    if cache.numel() % (PAGE_SIZE * D):
        raise ValueError("cache must be [num_pages, 64, 576]")
    num_pages = cache.numel() // (PAGE_SIZE * D)
    return B, T, H, _k_in_range(idx.shape[2]), page_table.shape[1], num_pages


def decode_partial(q, cache, page_table, idx, scale: float, nsplit: int, *, part_o=None,
                   part_m=None, part_lse=None, stream=None):
    """Partial pass; returns (part_o [B,T,H,S,512], part_m [B,T,H,S], part_lse [B,T,H,S])."""
    B, T, H, K, pt_stride, num_pages = _decode_args(q, cache, page_table, idx)
    dev = q.device
    if part_o is None:
        part_o = torch.empty((B, T, H, nsplit, DC), dtype=torch.float32, device=dev)
    if part_m is None:
        part_m = torch.empty((B, T, H, nsplit), dtype=torch.float32, device=dev)
    if part_lse is None:
        part_lse = torch.empty((B, T, H, nsplit), dtype=torch.float32, device=dev)
    _need(part_o, torch.float32, "part_o", dev, (B, T, H, nsplit, DC))
    _need(part_m, torch.float32, "part_m", dev, (B, T, H, nsplit))
    _need(part_lse, torch.float32, "part_lse", dev, (B, T, H, nsplit))
    _check(lib().smla_decode_partial(_ptr(q), _ptr(cache), num_pages, _ptr(page_table), pt_stride,
                                     _ptr(idx), B, T, H, K, PAGE_SIZE, float(scale), int(nsplit),
                                     _ptr(part_o), _ptr(part_m), _ptr(part_lse),
                                     _stream(stream)), "smla_decode_partial")
    return part_o, part_m, part_lse


def lse_combine(part_o, part_m, part_lse, *, o=None, lse=None, stream=None):
    """LSE combine; returns (o bf16 [B,T,H,512], lse fp32 [B,T,H])."""
    _need(part_m, torch.float32, "part_m")
    dev = part_m.device
    _need(part_o, torch.float32, "part_o", dev)
    _need(part_lse, torch.float32, "part_lse", dev)
    if part_m.dim() != 4:
        raise ValueError("part_m must be [B,T,H,S]")
    B, T, H, S = part_m.shape
    if tuple(part_o.shape) != (B, T, H, S, DC) or part_lse.shape != part_m.shape:
        raise ValueError("partial shapes disagree")
    if o is None:
        o = torch.empty((B, T, H, DC), dtype=torch.bfloat16, device=dev)
    if lse is None:
        lse = torch.empty((B, T, H), dtype=torch.float32, device=dev)
    _need(o, torch.bfloat16, "o", dev, (B, T, H, DC))
    _need(lse, torch.float32, "lse", dev, (B, T, H))
    _check(lib().smla_lse_combine(_ptr(part_o), _ptr(part_m), _ptr(part_lse), B, T, H, S, _ptr(o),
                                  _ptr(lse), _stream(stream)), "smla_lse_combine")
    return o, lse


def decode(q, cache, page_table, idx, scale: float, nsplit: int = 0, *, workspace=None,
           o=None, lse=None, stream=None):
    """Whole decode (partial + combine); returns (o bf16 [B,T,H,512], lse fp32 [B,T,H]).

    nsplit = 0 uses the library's heuristic.  A workspace (uint8 CUDA tensor)
    is allocated here when not given.
    """
    B, T, H, K, pt_stride, num_pages = _decode_args(q, cache, page_table, idx)
    dev = q.device
    if nsplit == 0:
        nsplit = choose_nsplit(B, T, H, K, 0)
    need = workspace_bytes(B, T, H, nsplit) if nsplit > 1 else 0
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)
    _need(workspace, torch.uint8, "workspace", dev)
    if o is None:
        o = torch.empty((B, T, H, DC), dtype=torch.bfloat16, device=dev)
    if lse is None:
        lse = torch.empty((B, T, H), dtype=torch.float32, device=dev)
    _need(o, torch.bfloat16, "o", dev, (B, T, H, DC))
    _need(lse, torch.float32, "lse", dev, (B, T, H))
    _check(lib().smla_decode(_ptr(q), _ptr(cache), num_pages, _ptr(page_table), pt_stride,
                             _ptr(idx), B, T, H, K, PAGE_SIZE, float(scale), int(nsplit),
                             _ptr(workspace), workspace.numel(), _ptr(o), _ptr(lse),
                             _stream(stream)), "smla_decode")
    return o, lse


def decode_noalloc(q, cache, page_table, idx, scale: float, nsplit: int = 0, *, o, lse,
                   stream=None):
    """Whole decode through smla_decode_noalloc: no workspace argument and no
    allocation anywhere (the split-K partials use the library's own device
    scratch array).  For callers that cannot allocate device memory while they
    decode, so o and lse must be given.  Calls that overlap on the GPU race on
    the shared scratch."""
    B, T, H, K, pt_stride, num_pages = _decode_args(q, cache, page_table, idx)
    _need(o, torch.bfloat16, "o", q.device, (B, T, H, DC))
    _need(lse, torch.float32, "lse", q.device, (B, T, H))
    _check(lib().smla_decode_noalloc(_ptr(q), _ptr(cache), num_pages, _ptr(page_table),
                                     pt_stride, _ptr(idx), B, T, H, K, PAGE_SIZE, float(scale),
                                     int(nsplit), _ptr(o), _ptr(lse), _stream(stream)),
           "smla_decode_noalloc")
    return o, lse


def dense_nsplit(B: int, T: int, H: int, K: int) -> int:
    return int(lib().smla_dense_nsplit(B, T, H, _k_in_range(K)))


def dense_workspace_bytes(B: int, T: int, H: int, K: int, nsplit: int) -> int:
    return int(lib().smla_dense_workspace_bytes(B, T, H, K, nsplit))


def _dense_args(q, cache, page_table, seq_lens, K):
    _need(q, torch.bfloat16, "q")
    dev = q.device
    _need(cache, torch.bfloat16, "cache", dev)
    _need(page_table, torch.int32, "page_table", dev)
    _need(seq_lens, torch.int32, "seq_lens", dev)
    if q.dim() != 4 or q.shape[-1] != D:
        raise ValueError(f"q must be [B,T,H,{D}]")
    B, T, H, _ = q.shape
    if tuple(seq_lens.shape) != (B, T):
        raise ValueError("seq_lens must be [B,T]")
    if page_table.dim() != 2 or page_table.shape[0] != B:
        raise ValueError("page_table must be [B, pt_stride]")
    if cache.numel() % (PAGE_SIZE * D):
        raise ValueError("cache must be [num_pages, 64, 576]")
    if K is None:
        K = int(seq_lens.max().item()) if seq_lens.numel() else 0
    return B, T, H, _k_in_range(int(K)), page_table.shape[1], cache.numel() // (PAGE_SIZE * D)


def decode_dense(q, cache, page_table, seq_lens, scale: float, nsplit: int = 0, *, K=None,
                 workspace=None, o=None, lse=None, stream=None):
    """Dense-context decode (KV-split verify): query token (b, t) attends to
    positions 0 .. seq_lens[b, t] - 1 of sequence b.  K defaults to the longest
    length (read from seq_lens, which synchronises); pass it to stay
    asynchronous.  Returns (o bf16 [B,T,H,512], lse fp32 [B,T,H])."""
    B, T, H, K, pt_stride, num_pages = _dense_args(q, cache, page_table, seq_lens, K)
    dev = q.device
    if nsplit == 0:
        nsplit = dense_nsplit(B, T, H, K)
    need = dense_workspace_bytes(B, T, H, K, nsplit)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)
    _need(workspace, torch.uint8, "workspace", dev)
    if o is None:
        o = torch.empty((B, T, H, DC), dtype=torch.bfloat16, device=dev)
    if lse is None:
        lse = torch.empty((B, T, H), dtype=torch.float32, device=dev)
    _need(o, torch.bfloat16, "o", dev, (B, T, H, DC))
    _need(lse, torch.float32, "lse", dev, (B, T, H))
    _check(lib().smla_decode_dense(_ptr(q), _ptr(cache), num_pages, _ptr(page_table), pt_stride,
                                   _ptr(seq_lens), B, T, H, K, PAGE_SIZE, float(scale),
                                   int(nsplit), _ptr(workspace), workspace.numel(), _ptr(o),
                                   _ptr(lse), _stream(stream)), "smla_decode_dense")
    return o, lse


def decode_dense_partial(q, cache, page_table, seq_lens, scale: float, nsplit: int, *, K=None,
                         part_o=None, part_m=None, part_lse=None, stream=None):
    """Partial pass of the dense variant; returns (part_o [B,T,H,S,512],
    part_m [B,T,H,S], part_lse [B,T,H,S])."""
    B, T, H, K, pt_stride, num_pages = _dense_args(q, cache, page_table, seq_lens, K)
    dev = q.device
    if part_o is None:
        part_o = torch.empty((B, T, H, nsplit, DC), dtype=torch.float32, device=dev)
    if part_m is None:
        part_m = torch.empty((B, T, H, nsplit), dtype=torch.float32, device=dev)
    if part_lse is None:
        part_lse = torch.empty((B, T, H, nsplit), dtype=torch.float32, device=dev)
    _need(part_o, torch.float32, "part_o", dev, (B, T, H, nsplit, DC))
    _need(part_m, torch.float32, "part_m", dev, (B, T, H, nsplit))
    _need(part_lse, torch.float32, "part_lse", dev, (B, T, H, nsplit))
    _check(lib().smla_decode_dense_partial(_ptr(q), _ptr(cache), num_pages, _ptr(page_table),
                                           pt_stride, _ptr(seq_lens), B, T, H, K, PAGE_SIZE,
                                           float(scale), int(nsplit), _ptr(part_o), _ptr(part_m),
                                           _ptr(part_lse), _stream(stream)),
           "smla_decode_dense_partial")
    return part_o, part_m, part_lse


def workspace_host_bytes(B: int, T: int, H: int, K: int, pt_stride: int, nsplit: int) -> int:
    return int(lib().smla_workspace_host_bytes(B, T, H, K, pt_stride, nsplit))


def decode_host(q, cache, page_table, idx, scale: float, nsplit: int = 0, *, o, lse,
                workspace=None, stream=None):
    """Whole decode through smla_decode_host: q, page_table, idx, o and lse are
    pinned CPU tensors (the per-step data of a host-driven decode loop), cache
    and workspace live on the GPU.  The inputs are pulled over the host link
    by a copy kernel and o, lse are written straight back into host memory;
    both are asynchronous on the stream (synchronise before reading o)."""
    for t, n, dt in ((q, "q", torch.bfloat16), (page_table, "page_table", torch.int32),
                     (idx, "idx", torch.int32), (o, "o", torch.bfloat16), (lse, "lse", torch.float32)):
        if not isinstance(t, torch.Tensor) or t.dtype != dt or not t.is_contiguous():
            raise TypeError(f"{n} must be a contiguous {dt} tensor")
        if t.is_cuda or not t.is_pinned():
            raise ValueError(f"{n} must be a pinned CPU tensor")
    _need(cache, torch.bfloat16, "cache")
    dev = cache.device
    if q.dim() != 4 or q.shape[-1] != D:
        raise ValueError(f"q must be [B,T,H,{D}]")
    B, T, H, _ = q.shape
    if idx.dim() != 3 or tuple(idx.shape[:2]) != (B, T):
        raise ValueError("idx must be [B,T,K]")
    if page_table.dim() != 2 or page_table.shape[0] != B:
        raise ValueError("page_table must be [B, pt_stride]")
    K, pt_stride = _k_in_range(idx.shape[2]), page_table.shape[1]
    if tuple(o.shape) != (B, T, H, DC) or tuple(lse.shape) != (B, T, H):
        raise ValueError(f"o must be [{B}, {T}, {H}, {DC}] and lse [{B}, {T}, {H}]")
    if cache.numel() % (PAGE_SIZE * D):
        raise ValueError("cache must be [num_pages, 64, 576]")
    num_pages = cache.numel() // (PAGE_SIZE * D)
    if nsplit == 0:
        nsplit = choose_nsplit(B, T, H, K, 0)
    need = workspace_host_bytes(B, T, H, K, pt_stride, nsplit)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)
    _need(workspace, torch.uint8, "workspace", dev)
    _check(lib().smla_decode_host(_ptr(q), _ptr(cache), num_pages, _ptr(page_table), pt_stride,
                                  _ptr(idx), B, T, H, K, PAGE_SIZE, float(scale), int(nsplit),
                                  _ptr(workspace), workspace.numel(), _ptr(o), _ptr(lse),
                                  _stream(stream)), "smla_decode_host")
    return o, lse


INDEXER_DIM, INDEXER_MAX_HEADS, INDEXER_MAX_N = 128, 64, 524288


def indexer_workspace_bytes(B: int, T: int, max_n: int) -> int:
    return int(lib().smla_indexer_workspace_bytes(B, T, max_n))


def indexer_select_workspace_bytes(B: int, T: int, max_n: int) -> int:
    return int(lib().smla_indexer_select_workspace_bytes(B, T, max_n))


def _indexer_args(q_index, w, k_index, page_table, n_vis):
    _need(q_index, torch.bfloat16, "q_index")
    dev = q_index.device
    _need(w, torch.float32, "w", dev)
    _need(k_index, torch.bfloat16, "k_index", dev)
    _need(page_table, torch.int32, "page_table", dev)
    _need(n_vis, torch.int32, "n_vis", dev)
    if q_index.dim() != 4 or q_index.shape[-1] != INDEXER_DIM:
        raise ValueError(f"q_index must be [B,T,HI,{INDEXER_DIM}]")
    B, T, HI, _ = q_index.shape
    if tuple(w.shape) != (B, T, HI) or tuple(n_vis.shape) != (B, T):
        raise ValueError("w must be [B,T,HI] and n_vis [B,T]")
    if page_table.dim() != 2 or page_table.shape[0] != B:
        raise ValueError("page_table must be [B, pt_stride]")
    if k_index.numel() % (PAGE_SIZE * INDEXER_DIM):
        raise ValueError("k_index must be [num_pages, 64, 128]")
    return B, T, HI, page_table.shape[1], k_index.numel() // (PAGE_SIZE * INDEXER_DIM)


def indexer_topk(q_index, w, k_index, page_table, n_vis, K: int, max_n: int, *, out=None,
                 workspace=None, stream=None):
    """Top-k indexer: the min(K, n) positions with the largest index score
    per query token, ascending then -1 (int32 [B, T, K]).  max_n bounds
    n_vis (it sizes the work and the score buffer)."""
    B, T, HI, pt_stride, num_pages = _indexer_args(q_index, w, k_index, page_table, n_vis)
    dev = q_index.device
    K = _k_in_range(int(K))
    if out is None:
        out = torch.empty((B, T, K), dtype=torch.int32, device=dev)
    _need(out, torch.int32, "out", dev, (B, T, K))
    if workspace is None:
        workspace = torch.empty(max(16, indexer_workspace_bytes(B, T, max_n)), dtype=torch.uint8,
                                device=dev)
    _need(workspace, torch.uint8, "workspace", dev)
    _check(lib().smla_indexer_topk(_ptr(q_index), _ptr(w), _ptr(k_index), num_pages,
                                   _ptr(page_table), pt_stride, _ptr(n_vis), B, T, HI, int(max_n),
                                   int(K), PAGE_SIZE, _ptr(workspace), workspace.numel(),
                                   _ptr(out), _stream(stream)), "smla_indexer_topk")
    return out


def indexer_scores(q_index, w, k_index, page_table, n_vis, max_n: int, *, scores=None,
                   workspace=None, stream=None):
    """Index scores fp32 [B, T, max_n] for every visible position (NaN where
    a position is not a candidate; entries past n_vis are not written)."""
    B, T, HI, pt_stride, num_pages = _indexer_args(q_index, w, k_index, page_table, n_vis)
    dev = q_index.device
    if scores is None:
        scores = torch.full((B, T, max(max_n, 1)), float("nan"), dtype=torch.float32, device=dev)
    # rows of max_n scores, one per query token (nothing is written when max_n is 0)
    _need(scores, torch.float32, "scores", dev, (B, T, max_n) if max_n > 0 else None)
    if workspace is None:
        workspace = torch.empty(max(16, indexer_workspace_bytes(B, T, 0)), dtype=torch.uint8,
                                device=dev)
    _need(workspace, torch.uint8, "workspace", dev)
    _check(lib().smla_indexer_scores(_ptr(q_index), _ptr(w), _ptr(k_index), num_pages,
                                     _ptr(page_table), pt_stride, _ptr(n_vis), B, T, HI,
                                     int(max_n), PAGE_SIZE, _ptr(workspace), workspace.numel(),
                                     _ptr(scores), _stream(stream)), "smla_indexer_scores")
    return scores


def indexer_select(scores, n_vis, K: int, *, out=None, workspace=None, stream=None):
    """The indexer's selection rule on given scores fp32 [B, T, max_n]."""
    _need(scores, torch.float32, "scores")
    dev = scores.device
    if scores.dim() != 3:
        raise ValueError("scores must be [B, T, max_n]")
    B, T, max_n = scores.shape
    _need(n_vis, torch.int32, "n_vis", dev, (B, T))
    K = _k_in_range(int(K))
    if out is None:
        out = torch.empty((B, T, K), dtype=torch.int32, device=dev)
    _need(out, torch.int32, "out", dev, (B, T, K))
    if workspace is None:
        workspace = torch.empty(max(16, indexer_select_workspace_bytes(B, T, max_n)),
                                dtype=torch.uint8, device=dev)
    _need(workspace, torch.uint8, "workspace", dev)
    _check(lib().smla_indexer_select(_ptr(scores), _ptr(n_vis), B, T, max_n, int(K),
                                     _ptr(workspace), workspace.numel(), _ptr(out),
                                     _stream(stream)), "smla_indexer_select")
    return out


def check_device(clear: bool = True, stream=None):
    """Synchronise and read the sticky device status: (status, n_bad_index)."""
    n = ctypes.c_ulonglong(0)
    st = lib().smla_check_device(1 if clear else 0, ctypes.byref(n), _stream(stream))
    return int(st), int(n.value)


def selftest_wait_timeout(limit_ns: int, stream=None) -> None:
    """Launch the bounded-wait self-test: one warp waits on a barrier that
    nothing arrives at and gives up after limit_ns, raising the timeout flag
    that check_device() then reports."""
    _check(lib().smla_selftest_wait_timeout(int(limit_ns), _stream(stream)),
           "smla_selftest_wait_timeout")


def status_string(status: int) -> str:
    return lib().smla_status_string(status).decode()
