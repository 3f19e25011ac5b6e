"""Seeded synthetic inputs for split-K sparse MLA decode.

This module only draws random numbers and lays them out; it holds none of
the method's arithmetic.  Both the CUDA path and the fp64 oracle are fed from
it, so it imports neither.

Every workload is a paged latent KV cache plus the per-token top-k index
lists that select rows from it:

* ``q``          bf16 ``[B, T, H, 576]``: per head ``[q_nope (512) | q_pe (64)]``
* ``cache``      bf16 ``[num_pages, 64, 576]``: per token ``[c (512) | k_pe (64)]``
* ``page_table`` int32 ``[B, pt_stride]``: physical page of each logical page
                 (``-1`` where a sequence owns no page)
* ``idx``        int32 ``[B, T, K]``: logical token positions, ``-1`` = padding

Values are N(0, 1) * 0.5 rounded to bf16.  Index lists are distinct positions
in random order.  The five named workloads follow the problem statement's
configurations (tiny / single-request / speculative verify / batched /
mixed-length); the pages themselves give only their shapes in prose: the
grid arithmetic of "The Occupancy Hypothesis" (section "The Occupancy
Insight", q_len 9 and 8 heads per rank at 46K context) and the C=1 / C=64
concurrency sweep of "The Moment of Truth" (section "The Split-K Imperative").
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional, Sequence

import torch

DC = 512
DR = 64
D = DC + DR
PAGE_SIZE = 64


@dataclasses.dataclass
class Workload:
    name: str
    q: torch.Tensor            # bf16 [B,T,H,D]
    cache: torch.Tensor        # bf16 [P,PAGE_SIZE,D]
    page_table: torch.Tensor   # int32 [B,pt_stride]
    idx: torch.Tensor          # int32 [B,T,K]
    scale: float
    ctx_lens: list             # tokens owned by each sequence
    nsplit: Optional[int]      # the configuration's fixed NSPLIT, None = heuristic
    nsplit_sweep: tuple        # NSPLIT values the configuration sweeps
    seq_lens: Optional[torch.Tensor] = None  # int32 [B,T]: dense variant's visible lengths

    @property
    def dense(self) -> bool:
        return self.seq_lens is not None

    @property
    def B(self):
        return self.q.shape[0]

    @property
    def T(self):
        return self.q.shape[1]

    @property
    def H(self):
        return self.q.shape[2]

    @property
    def K(self):
        if self.dense:
            return int(self.seq_lens.max()) if self.seq_lens.numel() else 0
        return self.idx.shape[2]

    @property
    def num_pages(self):
        return self.cache.shape[0]

    @property
    def pt_stride(self):
        return self.page_table.shape[1]

    def n_valid(self) -> int:
        """Number of attended rows (non-padding index entries, or visible
        positions of the dense variant) over the whole batch."""
        if self.dense:
            return int(self.seq_lens.to(torch.int64).sum())
        return int((self.idx >= 0).sum())

    def to(self, device) -> "Workload":
        return dataclasses.replace(
            self, q=self.q.to(device), cache=self.cache.to(device),
            page_table=self.page_table.to(device), idx=self.idx.to(device),
            seq_lens=None if self.seq_lens is None else self.seq_lens.to(device))


def _normal_bf16(shape, gen, chunk_rows=1 << 14) -> torch.Tensor:
    """N(0,1)*0.5 rounded to bf16, drawn in row chunks to bound host memory."""
    out = torch.empty(shape, dtype=torch.bfloat16)
    flat = out.view(-1, shape[-1])
    for r0 in range(0, flat.shape[0], chunk_rows):
        r1 = min(flat.shape[0], r0 + chunk_rows)
        flat[r0:r1] = (torch.randn((r1 - r0, shape[-1]), generator=gen) * 0.5).to(torch.bfloat16)
    return out


def make_workload(name: str, *, B: int, T: int, H: int, K: int,
                  ctx_lens: Sequence[int], seed: int, paged: bool = True,
                  shuffle_pages: bool = True, causal: bool = False,
                  scale: Optional[float] = None, nsplit: Optional[int] = None,
                  nsplit_sweep: Sequence[int] = ()) -> Workload:
    """Draw one workload.

    ``ctx_lens[b]`` tokens of sequence ``b`` live in the cache.  With
    ``causal``, query token ``t`` of sequence ``b`` draws its indices from
    ``[0, ctx_lens[b] - T + t)`` (the sequence holds ``T`` draft tokens at its
    end, and token ``t`` sees the context plus the ``t`` drafts before it);
    otherwise from ``[0, ctx_lens[b])``.  Where fewer than ``K``
    positions are available, the list is padded with ``-1`` at its tail.
    """
    gen = torch.Generator().manual_seed(seed)
    ctx_lens = [int(c) for c in ctx_lens]
    assert len(ctx_lens) == B
    pages_per_seq = [(c + PAGE_SIZE - 1) // PAGE_SIZE for c in ctx_lens]
    total_pages = sum(pages_per_seq)
    pt_stride = max(pages_per_seq)

    q = _normal_bf16((B, T, H, D), gen)
    cache = _normal_bf16((total_pages, PAGE_SIZE, D), gen)

    if paged and shuffle_pages:
        perm = torch.randperm(total_pages, generator=gen).to(torch.int32)
    else:
        perm = torch.arange(total_pages, dtype=torch.int32)
    page_table = torch.full((B, pt_stride), -1, dtype=torch.int32)
    off = 0
    for b, n in enumerate(pages_per_seq):
        page_table[b, :n] = perm[off:off + n]
        off += n

    idx = torch.full((B, T, K), -1, dtype=torch.int32)
    for b in range(B):
        for t in range(T):
            avail = ctx_lens[b] - T + t if causal else ctx_lens[b]
            n = min(K, avail)
            idx[b, t, :n] = torch.randperm(avail, generator=gen)[:n].to(torch.int32)

    if scale is None:
        scale = 1.0 / math.sqrt(D)
    return Workload(name=name, q=q, cache=cache, page_table=page_table, idx=idx,
                    scale=float(scale), ctx_lens=ctx_lens, nsplit=nsplit,
                    nsplit_sweep=tuple(nsplit_sweep))


def mixed_ctx_lens(B: int, seed: int, lo: int = 1024, hi: int = 131072) -> list:
    """Context lengths floor(exp(U(ln lo, ln hi))): log-uniform in [lo, hi]."""
    gen = torch.Generator().manual_seed(seed + 7919)
    u = torch.rand(B, generator=gen, dtype=torch.float64)
    lens = torch.exp(math.log(lo) + u * (math.log(hi) - math.log(lo))).floor()
    return [int(min(max(v, lo), hi)) for v in lens.tolist()]


def make_dense_workload(name: str, *, B: int, T: int, H: int, ctx_lens: Sequence[int],
                        seed: int, paged: bool = True, scale: Optional[float] = None,
                        nsplit: Optional[int] = None, nsplit_sweep: Sequence[int] = ()) -> Workload:
    """Draw a dense-context (verify) workload: the cache and query as
    ``make_workload`` draws them, no index lists, and ``seq_lens[b, t] =
    ctx_lens[b] - T + t + 1``: the sequence ends with its ``T`` draft tokens
    and token ``t`` sees every position up to and including its own."""
    w = make_workload(name, B=B, T=T, H=H, K=0, ctx_lens=ctx_lens, seed=seed, paged=paged,
                      scale=scale, nsplit=nsplit, nsplit_sweep=nsplit_sweep)
    lens = torch.tensor([[c - T + t + 1 for t in range(T)] for c in w.ctx_lens], dtype=torch.int32)
    if int(lens.min()) < 0:
        raise ValueError("every context must hold its T draft tokens")
    return dataclasses.replace(w, seq_lens=lens)


# name -> (description, builder)
def tiny(seed: int = 0) -> Workload:
    """B1 T1 H8 K256, contiguous 4096-token cache, NSPLIT 4."""
    return make_workload("tiny", B=1, T=1, H=8, K=256, ctx_lens=[4096], seed=seed,
                         paged=False, nsplit=4, nsplit_sweep=(4,))


def single_request(seed: int = 1) -> Workload:
    """B1 T1 H16 K2048, 65536-token paged cache (shuffled page table)."""
    return make_workload("single_request", B=1, T=1, H=16, K=2048,
                         ctx_lens=[65536], seed=seed,
                         nsplit_sweep=(1, 4, 16, 32, 64))


def spec_verify(seed: int = 2) -> Workload:
    """B1 T9 H8 K2048 per token, context 46080 + 9 draft tokens, causal draws."""
    return make_workload("spec_verify", B=1, T=9, H=8, K=2048, ctx_lens=[46080 + 9],
                         seed=seed, causal=True, nsplit_sweep=(16, 64))


def batched(seed: int = 3, B: int = 64) -> Workload:
    """B64 T1 H16 K2048, 16384 tokens per sequence, pages interleaved globally."""
    return make_workload("batched", B=B, T=1, H=16, K=2048, ctx_lens=[16384] * B,
                         seed=seed)


def mixed(seed: int = 4, B: int = 60) -> Workload:
    """B60 T1 H64 K2048, log-uniform context in [1024, 131072], -1 tail padding."""
    return make_workload("mixed", B=B, T=1, H=64, K=2048,
                         ctx_lens=mixed_ctx_lens(B, seed), seed=seed)


def dense_verify(seed: int = 5) -> Workload:
    """B1 T9 H8, 46080-token context + 9 draft tokens, dense causal verify
    (every visible position), NSPLIT swept over {16, 64} as on the pages."""
    return make_dense_workload("dense_verify", B=1, T=9, H=8, ctx_lens=[46080 + 9], seed=seed,
                               nsplit_sweep=(16, 64))


# ---------------------------------------------------------------- top-k indexer inputs
INDEX_DIM = 128


@dataclasses.dataclass
class IndexerWorkload:
    """Inputs of the top-k indexer: per-token index queries and head weights,
    a paged index-key cache (the latent cache's page numbering), and the
    visible length of every query token."""
    name: str
    q_index: torch.Tensor      # bf16 [B, T, HI, 128]
    w: torch.Tensor            # fp32 [B, T, HI]
    k_index: torch.Tensor      # bf16 [P, PAGE_SIZE, 128]
    page_table: torch.Tensor   # int32 [B, pt_stride]
    n_vis: torch.Tensor        # int32 [B, T]
    K: int
    ctx_lens: list

    @property
    def B(self):
        return self.q_index.shape[0]

    @property
    def T(self):
        return self.q_index.shape[1]

    @property
    def HI(self):
        return self.q_index.shape[2]

    @property
    def num_pages(self):
        return self.k_index.shape[0]

    @property
    def pt_stride(self):
        return self.page_table.shape[1]

    @property
    def max_n(self):
        return int(self.n_vis.max()) if self.n_vis.numel() else 0

    def to(self, device) -> "IndexerWorkload":
        return dataclasses.replace(self, q_index=self.q_index.to(device), w=self.w.to(device),
                                   k_index=self.k_index.to(device),
                                   page_table=self.page_table.to(device),
                                   n_vis=self.n_vis.to(device))


def make_indexer_workload(name: str, *, B: int, T: int, HI: int, K: int, ctx_lens: Sequence[int],
                          seed: int, causal: bool = False, integer: bool = False,
                          shuffle_pages: bool = True) -> IndexerWorkload:
    """Draw indexer inputs.  Values are N(0,1)*0.5 rounded to bf16 (query and
    keys) and N(0,1)*0.5 fp32 weights; with ``integer`` they are small
    integers instead (queries and keys in [-2, 2], weights in [-2, 2]), so
    that every score is an exact integer in fp32 whatever the summation
    order.  n_vis[b, t] = ctx_lens[b], or with ``causal`` ctx_lens[b] - T + t
    + 1 (draft token t sees the context and the drafts up to itself)."""
    gen = torch.Generator().manual_seed(seed)
    ctx_lens = [int(c) for c in ctx_lens]
    assert len(ctx_lens) == B
    pages_per_seq = [max(1, (c + PAGE_SIZE - 1) // PAGE_SIZE) for c in ctx_lens]
    total_pages = sum(pages_per_seq)
    pt_stride = max(pages_per_seq)
    if integer:
        q = torch.randint(-2, 3, (B, T, HI, INDEX_DIM), generator=gen).to(torch.bfloat16)
        k = torch.randint(-2, 3, (total_pages, PAGE_SIZE, INDEX_DIM), generator=gen).to(torch.bfloat16)
        w = torch.randint(-2, 3, (B, T, HI), generator=gen).to(torch.float32)
    else:
        q = _normal_bf16((B, T, HI, INDEX_DIM), gen)
        k = _normal_bf16((total_pages, PAGE_SIZE, INDEX_DIM), gen)
        w = torch.randn((B, T, HI), generator=gen) * 0.5
    perm = (torch.randperm(total_pages, generator=gen) if shuffle_pages
            else torch.arange(total_pages)).to(torch.int32)
    page_table = torch.full((B, pt_stride), -1, dtype=torch.int32)
    off = 0
    for b, n in enumerate(pages_per_seq):
        page_table[b, :n] = perm[off:off + n]
        off += n
    n_vis = torch.tensor([[(c - T + t + 1) if causal else c for t in range(T)] for c in ctx_lens],
                         dtype=torch.int32)
    return IndexerWorkload(name=name, q_index=q, w=w.to(torch.float32), k_index=k,
                           page_table=page_table, n_vis=n_vis, K=K, ctx_lens=ctx_lens)


def indexer_mixed(seed: int = 6, B: int = 60) -> IndexerWorkload:
    """The indexer ahead of the mixed-length decode: B60 T1, contexts
    log-uniform in [1024, 131072], 64 index heads of 128 values, top-2048."""
    return make_indexer_workload("indexer_mixed", B=B, T=1, HI=64, K=2048,
                                 ctx_lens=mixed_ctx_lens(B, seed), seed=seed)


WORKLOADS = {
    "tiny": tiny,
    "single_request": single_request,
    "spec_verify": spec_verify,
    "batched": batched,
    "mixed": mixed,
    "dense_verify": dense_verify,
}
