"""The benchmark's accounting on CPU: the algorithmic bytes every roofline
figure divides, counted here query token by query token from the definition
of what a decode must move, and the roofline record's arithmetic.

Per query token of the sparse path: each selected row once (576 bf16 =
1152 B) with the page-table entry that maps it (4 B), the K index entries
(4 B each), q (H x 1152 B); the combine adds o (H x 512 bf16) and lse
(H x 4 B).  The dense verify variant's tokens attend to nested prefixes of
one sequence, so a row of the longest prefix counts once.  The indexer reads
every visible key once (128 bf16), one page-table entry per page of keys,
the queries and weights, the length, and writes K positions.
"""
import os
import sys

import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from sparse_mla_decode_partial_b200 import workloads  # noqa: E402


def sparse_bytes_by_token(w):
    partial = 0
    for b in range(w.B):
        for t in range(w.T):
            valid = sum(1 for j in range(w.K) if int(w.idx[b, t, j]) != -1)
            partial += valid * (1152 + 4) + w.K * 4 + w.H * 1152
    return partial, partial + w.B * w.T * w.H * (1024 + 4)


def dense_bytes_by_token(w):
    partial = 0
    for b in range(w.B):
        partial += max(int(w.seq_lens[b, t]) for t in range(w.T)) * (1152 + 4)
        for t in range(w.T):
            partial += 4 + w.H * 1152
    return partial, partial + w.B * w.T * w.H * (1024 + 4)


def indexer_bytes_by_token(w):
    total = 0
    for b in range(w.B):
        for t in range(w.T):
            n = max(int(w.n_vis[b, t]), 0)
            total += n * 256 + -(-n // 64) * 4 + w.HI * (256 + 4) + 4 + w.K * 4
    return total


def index_lists_only(name, B, T, H, K, valid_per_token):
    """A workload with only what the byte count reads: shapes and index
    lists with `valid` entries then -1 (the cache is not drawn)."""
    idx = torch.full((B, T, K), -1, dtype=torch.int32)
    for (b, t), v in valid_per_token.items():
        idx[b, t, :v] = torch.arange(v, dtype=torch.int32)
    return workloads.Workload(name=name, q=torch.empty((B, T, H, 0), dtype=torch.bfloat16),
                              cache=torch.empty((1, 64, 0), dtype=torch.bfloat16),
                              page_table=torch.zeros((B, 1), dtype=torch.int32), idx=idx,
                              scale=0.1, ctx_lens=[0] * B, nsplit=None, nsplit_sweep=())


def test_sparse_bytes_match_the_token_by_token_count():
    w = workloads.make_workload("acct", B=3, T=2, H=5, K=40, ctx_lens=[25, 40, 100], seed=9,
                                causal=True)
    assert (w.idx == -1).any() and (w.idx != -1).any()     # ragged: some padding
    assert bench.workload_bytes(w) == sparse_bytes_by_token(w)
    t = workloads.tiny()
    assert bench.workload_bytes(t) == sparse_bytes_by_token(t)


def test_dense_bytes_count_each_row_of_the_longest_prefix_once():
    w = workloads.make_dense_workload("acct_dense", B=2, T=3, H=4, ctx_lens=[70, 200], seed=8)
    assert bench.workload_bytes(w) == dense_bytes_by_token(w)
    # one query token: its prefix, i.e. the sparse count of the full list
    one = workloads.make_dense_workload("acct_one", B=1, T=1, H=4, ctx_lens=[130], seed=8)
    assert bench.workload_bytes(one)[0] == 130 * 1156 + 4 + 4 * 1152


def test_indexer_bytes_match_the_token_by_token_count():
    w = workloads.make_indexer_workload("acct_ix", B=3, T=2, HI=8, K=50, ctx_lens=[65, 1, 300],
                                        seed=7, causal=True)
    assert bench.indexer_bytes(w) == indexer_bytes_by_token(w)


def test_headline_per_launch_bytes():
    """The partial pass's algorithmic bytes per launch quoted with every
    bench line: single_request exactly, the others from their index lists."""
    sr = workloads.single_request()
    assert bench.workload_bytes(sr)[0] == 2_394_112 == sparse_bytes_by_token(sr)[0]
    batched = index_lists_only("batched", 64, 1, 16, 2048, {(b, 0): 2048 for b in range(64)})
    assert bench.workload_bytes(batched)[0] == 64 * 2_394_112 == 153_223_168
    lens = workloads.mixed_ctx_lens(60, 4)
    mixed = index_lists_only("mixed", 60, 1, 64, 2048, {(b, 0): min(2048, c) for b, c in enumerate(lens)})
    want = sum(min(2048, c) for c in lens) * 1156 + 60 * (2048 * 4 + 64 * 1152)
    assert bench.workload_bytes(mixed)[0] == want == 142_034_140
    spec = index_lists_only("spec_verify", 1, 9, 8, 2048, {(0, t): 2048 for t in range(9)})
    assert bench.workload_bytes(spec)[0] == 9 * (2048 * 1156 + 2048 * 4 + 8 * 1152) == 21_464_064
    dv_lens = torch.tensor([[46089 - 9 + t + 1 for t in range(9)]], dtype=torch.int32)
    dv = index_lists_only("dense_verify", 1, 9, 8, 0, {})
    dv.seq_lens = dv_lens
    assert bench.workload_bytes(dv)[0] == 46089 * 1156 + 9 * (4 + 8 * 1152) == 53_361_864


def test_indexer_key_bytes_of_the_mixed_contexts():
    lens = workloads.mixed_ctx_lens(60, 6)
    w = workloads.IndexerWorkload(name="ix", q_index=torch.empty((60, 1, 64, 0)),
                                  w=torch.empty((60, 1, 64)), k_index=torch.empty((1, 64, 0)),
                                  page_table=torch.zeros((60, 1), dtype=torch.int32),
                                  n_vis=torch.tensor([[c] for c in lens], dtype=torch.int32),
                                  K=2048, ctx_lens=lens)
    key_bytes = bench.indexer_bytes(w) - 60 * 2048 * 4     # the score kernel's share
    assert key_bytes == sum(c * 256 + -(-c // 64) * 4 for c in lens) + 60 * (64 * 260 + 4)
    assert key_bytes == 418_830_540


def test_roofline_record_arithmetic():
    w = workloads.tiny()
    part_bytes, _ = bench.workload_bytes(w)
    rec = bench.roofline(w, 4, 0.01, "tiny", 6650.0, 1590.0, "fallback")
    achieved = part_bytes / 10e-6 / 1e9
    assert rec["achieved"] == round(achieved, 1) and rec["frac"] == round(achieved / 6650.0, 4)
    assert rec["algorithmic_bytes_per_launch"] == part_bytes and rec["partial_us_median"] == 10.0
    assert rec["kernel"] == "smla_partial_small_kernel" and rec["traffic"] is None
    flops = 2 * w.H * w.n_valid() * (576 + 512)
    assert rec["tensor_tflops"] == round(flops / 10e-6 / 1e12, 2)
    assert rec["peak_source"] == "fallback" and rec["bound"] == "hbm"
