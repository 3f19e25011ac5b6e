"""fp64 CPU oracles for split-K sparse MLA decode and its top-k indexer --
test infrastructure only.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The CUDA library never uses it.
"""
from . import indexer
from .oracle import (DC, DR, PAGE_SIZE, build, combine, decode, decode_dense, dense_positions,
                     max_threads, partial, set_threads)

__all__ = ["indexer", "DC", "DR", "PAGE_SIZE", "build", "combine", "decode", "decode_dense",
           "dense_positions", "max_threads", "partial", "set_threads"]
