"""Split-K sparse MLA decode for NVIDIA B200 (sm_100a).

The compute path is the C-ABI library ``libsmla.so`` built from ``csrc/``;
``binding`` marshals torch tensors into it.  ``workloads`` draws the seeded
synthetic inputs.  Importing this package loads nothing; the library is
loaded on first use and its absence is an error, never a fallback.
"""
__all__ = ["binding", "workloads"]
