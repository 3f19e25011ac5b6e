"""GPU parity of the top-k indexer (through the C ABI) against its fp64 oracle.

The selection is integer output decided by floating-point scores, so the
checks are layered:
  * exact-integer inputs: every score is an exact integer in fp32 and in fp64
    whatever the summation order, so the whole selection -- ties to the
    smaller position included -- must match the oracle bit for bit;
  * general inputs: the kernel's fp32 scores must lie within the fp32
    rounding bound of the oracle's fp64 scores; the selection step applied to
    the kernel's own scores must match the oracle's selection rule applied to
    the same scores bit for bit (the decision taken in the kernel's
    precision); and the end-to-end selection must be a valid top-k of the
    exact scores: everything clearly above the K-th score in, everything
    clearly below it out, exactly min(K, candidates) entries, ascending.
"""
import numpy as np
import pytest
import torch

from oracle import indexer as ix_oracle
from parity_util import bits
from sparse_mla_decode_partial_b200 import binding, build, workloads

pytestmark = pytest.mark.gpu

DEV = torch.device("cuda:0")


@pytest.fixture(scope="module", autouse=True)
def _built():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    build.build()
    binding.lib()
    binding.check_device(clear=True)
    yield
    st, _ = binding.check_device(clear=True)
    assert st in (0, 5), binding.status_string(st)


def oracle_args(w):
    return (bits(w.q_index), w.w.numpy(), bits(w.k_index), w.page_table.numpy(), w.n_vis.numpy())


def gpu_topk(w, K=None, max_n=None):
    wd = w.to(DEV)
    out = binding.indexer_topk(wd.q_index, wd.w, wd.k_index, wd.page_table, wd.n_vis,
                               K or w.K, w.max_n if max_n is None else max_n)
    torch.cuda.synchronize()
    return out.cpu().numpy()


def gpu_scores(w):
    wd = w.to(DEV)
    sc = binding.indexer_scores(wd.q_index, wd.w, wd.k_index, wd.page_table, wd.n_vis, w.max_n)
    torch.cuda.synchronize()
    return sc


def magnitude(w):
    """sum_j |w_j| sum_d |q_jd k_sd| per (b, t, s): the scale of the fp32
    rounding error of a score (fp64, from the inputs only)."""
    q = w.q_index.double().abs().numpy()
    k = w.k_index.double().abs().reshape(-1, 128).numpy()
    wa = w.w.double().abs().numpy()
    pt = w.page_table.numpy()
    out = np.zeros((w.B, w.T, w.max_n))
    for b in range(w.B):
        rows = pt[b, np.arange(w.max_n) // 64].astype(np.int64) * 64 + np.arange(w.max_n) % 64
        rows = np.clip(rows, 0, k.shape[0] - 1)
        for t in range(w.T):
            out[b, t] = (wa[b, t][:, None] * (q[b, t] @ k[rows].T)).sum(0)
    return out


INT_CASES = [
    # name, kwargs
    ("64 heads, two contexts", dict(B=2, T=1, HI=64, K=256, ctx_lens=[3000, 700])),
    ("16 heads", dict(B=2, T=1, HI=16, K=100, ctx_lens=[1000, 1500])),
    ("32 heads, n < K", dict(B=3, T=1, HI=32, K=512, ctx_lens=[130, 300, 700])),
    ("5 heads, causal drafts", dict(B=2, T=3, HI=5, K=64, ctx_lens=[777, 129], causal=True)),
    ("40 heads, ragged tails", dict(B=2, T=2, HI=40, K=33, ctx_lens=[64, 193])),
    ("one head, K = 1", dict(B=1, T=2, HI=1, K=1, ctx_lens=[5000])),
]


@pytest.mark.parametrize("name,kw", INT_CASES, ids=[c[0] for c in INT_CASES])
def test_exact_integer_inputs_bit_exact(name, kw):
    w = workloads.make_indexer_workload("ix_int", seed=len(name), integer=True, **kw)
    want, bad = ix_oracle.topk(*oracle_args(w), w.K)
    assert bad == 0
    got = gpu_topk(w)
    assert np.array_equal(got, want), name
    # the scores themselves are exact integers
    sc = gpu_scores(w).cpu().numpy()
    ref, _ = ix_oracle.scores(*oracle_args(w))
    for b in range(w.B):
        for t in range(w.T):
            n = int(w.n_vis[b, t])
            assert np.array_equal(sc[b, t, :n].astype(np.float64), ref[b, t, :n])


def test_many_ties_go_to_the_smaller_position():
    # keys drawn from {-1, 0, 1} and one index head: scores take few values
    w = workloads.make_indexer_workload("ix_ties", B=2, T=1, HI=1, K=300, ctx_lens=[2000, 4100],
                                        seed=3, integer=True)
    w.k_index.clamp_(-1, 1)
    w.q_index.clamp_(-1, 1)
    w.w.fill_(1.0)
    want, _ = ix_oracle.topk(*oracle_args(w), w.K)
    assert np.array_equal(gpu_topk(w), want)


def test_zero_visible_and_bad_pages_counted():
    w = workloads.make_indexer_workload("ix_bad", B=3, T=1, HI=16, K=40, ctx_lens=[500, 300, 200],
                                        seed=5, integer=True)
    w.n_vis[2, 0] = 0                           # nothing visible: all -1
    w.page_table[0, 2] = w.num_pages + 7        # positions 128..191 of sequence 0 map nowhere
    binding.check_device(clear=True)
    want, bad = ix_oracle.topk(*oracle_args(w), w.K)
    got = gpu_topk(w)
    st, n_bad = binding.check_device(clear=True)
    assert np.array_equal(got, want)
    assert np.all(got[2, 0] == -1)
    assert bad == 64 and st == 5 and n_bad == 64


@pytest.mark.parametrize("HI,T", [(64, 1), (16, 2), (48, 3)])
def test_scores_within_fp32_rounding_of_the_oracle(HI, T):
    w = workloads.make_indexer_workload("ix_sc", B=2, T=T, HI=HI, K=128, ctx_lens=[2500, 900],
                                        seed=HI + T, causal=T > 1)
    sc = gpu_scores(w).cpu().numpy().astype(np.float64)
    ref, _ = ix_oracle.scores(*oracle_args(w))
    mag = magnitude(w)
    for b in range(w.B):
        for t in range(w.T):
            n = int(w.n_vis[b, t])
            err = np.abs(sc[b, t, :n] - ref[b, t, :n])
            assert np.all(err <= 2e-5 * mag[b, t, :n] + 1e-6), (b, t, float(err.max()))


@pytest.mark.parametrize("seed", [0, 1])
def test_selection_bit_exact_on_the_kernels_own_scores(seed):
    w = workloads.make_indexer_workload("ix_sel", B=3, T=2, HI=64, K=700, ctx_lens=[6000, 1000, 650],
                                        seed=40 + seed, causal=True)
    sc = gpu_scores(w)
    nv = w.n_vis.to(DEV)
    got = binding.indexer_select(sc, nv, w.K)
    torch.cuda.synchronize()
    want = ix_oracle.select(sc.cpu().numpy(), w.n_vis.numpy(), w.K)
    assert np.array_equal(got.cpu().numpy(), want)
    # the fused path selects from the same scores
    assert np.array_equal(gpu_topk(w), want)


def crafted_scores(rng, B, T, max_n, kind):
    """Score rows that stress the selection: special values, heavy ties that
    straddle chunk boundaries, one value everywhere."""
    sc = np.full((B, T, max_n), np.nan, np.float32)
    for b in range(B):
        for t in range(T):
            if kind == "special":
                row = rng.choice(np.array([np.nan, np.inf, -np.inf, 0.0, -0.0, 1.0, -1.0, 3.0e38,
                                           -3.0e38, 1e-45, -1e-45, 2.0, 2.0], np.float32), max_n)
            elif kind == "ties":
                row = rng.integers(-3, 4, max_n).astype(np.float32)
            elif kind == "constant":
                row = np.full(max_n, 0.25, np.float32)
            else:
                row = rng.standard_normal(max_n).astype(np.float32)
            sc[b, t] = row
    return sc


SELECT_CASES = [
    # kind, n_vis rows, K
    ("special", [[20000], [8192], [8193], [1]], 700),
    ("ties", [[30000, 7], [16384, 100]], 2048),
    ("constant", [[40000], [9000]], 300),      # crossing bucket holds every position
    ("normal", [[65536], [12345], [0]], 2048),
    ("normal", [[5000], [4999]], 5000),        # K >= n: everything, in order
]


@pytest.mark.parametrize("kind,nv,K", SELECT_CASES,
                         ids=[f"{c[0]}-{len(c[1])}x{len(c[1][0])}-K{c[2]}" for c in SELECT_CASES])
def test_selection_on_crafted_scores_bit_exact(kind, nv, K):
    rng = np.random.default_rng(len(kind) * 1000 + K)
    n_vis = np.array(nv, np.int32)
    B, T = n_vis.shape
    max_n = int(n_vis.max()) or 1
    sc = crafted_scores(rng, B, T, max_n, kind)
    got = binding.indexer_select(torch.from_numpy(sc).to(DEV), torch.from_numpy(n_vis).to(DEV), K)
    torch.cuda.synchronize()
    want = ix_oracle.select(sc, n_vis, K)
    assert np.array_equal(got.cpu().numpy(), want)


def test_selection_at_the_maximum_length():
    """max_n = SMLA_INDEXER_MAX_N: the finishing kernel's largest shared-memory
    configuration (position bitmaps of 524288 positions), the chunked passes'
    longest grid row, and a K that takes every candidate of a shorter row."""
    rng = np.random.default_rng(2024)
    max_n = binding.INDEXER_MAX_N
    n_vis = np.array([[max_n], [max_n - 37], [1000]], np.int32)
    sc = rng.standard_normal((3, 1, max_n)).astype(np.float32)
    sc[1, 0, ::7] = np.nan                        # non-candidates spread over the row
    scd, nvd = torch.from_numpy(sc).to(DEV), torch.from_numpy(n_vis).to(DEV)
    for K in (2048, 4096):
        got = binding.indexer_select(scd, nvd, K)
        torch.cuda.synchronize()
        assert np.array_equal(got.cpu().numpy(), ix_oracle.select(sc, n_vis, K)), K


def test_selection_many_short_tokens():
    """Thousands of query tokens with short rows (most chunk CTAs of the 1-D
    grid have no positions; many tokens take everything)."""
    rng = np.random.default_rng(99)
    B, T, max_n = 512, 8, 700
    n_vis = rng.integers(0, max_n + 1, (B, T)).astype(np.int32)
    sc = rng.integers(-4, 5, (B, T, max_n)).astype(np.float32)   # many ties
    got = binding.indexer_select(torch.from_numpy(sc).to(DEV), torch.from_numpy(n_vis).to(DEV), 300)
    torch.cuda.synchronize()
    assert np.array_equal(got.cpu().numpy(), ix_oracle.select(sc, n_vis, 300))


def test_select_workspace_is_scratch_only():
    """A workspace left dirty by an earlier call (or filled with garbage)
    gives the same selection."""
    rng = np.random.default_rng(77)
    n_vis = np.array([[30000], [9000], [500]], np.int32)
    sc = crafted_scores(rng, 3, 1, 30000, "ties")
    scd, nvd = torch.from_numpy(sc).to(DEV), torch.from_numpy(n_vis).to(DEV)
    ws = torch.full((binding.indexer_select_workspace_bytes(3, 1, 30000),), 0xA5, dtype=torch.uint8,
                    device=DEV)
    want = ix_oracle.select(sc, n_vis, 1000)
    for _ in range(2):
        got = binding.indexer_select(scd, nvd, 1000, workspace=ws)
        torch.cuda.synchronize()
        assert np.array_equal(got.cpu().numpy(), want)


def valid_topk(sel, exact, n, K, eps):
    """sel is a valid top-K of the exact scores up to eps: ascending, unique,
    exactly min(K, candidates) entries, and nothing is misplaced by more than
    the rounding band around the K-th score."""
    cand = np.where(~np.isneginf(exact[:n]))[0]
    take = min(K, len(cand))
    s = sel[sel >= 0]
    assert len(s) == take and np.all(sel[take:] == -1)
    assert np.all(np.diff(s) > 0) and np.all(np.isin(s, cand))
    if take == 0 or take == len(cand):
        return 0
    tau = np.sort(exact[cand])[::-1][take - 1]
    inside = np.zeros(n, bool)
    inside[s] = True
    must_in = cand[exact[cand] > tau + 2 * eps]
    must_out = cand[exact[cand] < tau - 2 * eps]
    assert inside[must_in].all(), "a clearly larger score was left out"
    assert not inside[must_out].any(), "a clearly smaller score was taken"
    return int(len(cand) - len(must_in) - len(must_out))


def test_end_to_end_selection_is_a_valid_topk():
    w = workloads.make_indexer_workload("ix_valid", B=4, T=1, HI=64, K=2048,
                                        ctx_lens=[65536, 5000, 2048, 1500], seed=9)
    got = gpu_topk(w)
    ref, _ = ix_oracle.scores(*oracle_args(w))
    mag = magnitude(w)
    for b in range(w.B):
        n = int(w.n_vis[b, 0])
        valid_topk(got[b, 0], ref[b, 0, :n], n, w.K, eps=float(2e-5 * mag[b, 0, :n].max() + 1e-6))


def test_mixed_lengths_full_size():
    """B60 contexts 1K..128K (the mixed-length decode's shape), 64 index heads,
    top-2048: every token's selection is a valid top-k of the exact scores,
    and bit-exact against the oracle's rule on the kernel's own scores."""
    w = workloads.indexer_mixed()
    wd = w.to(DEV)
    got = binding.indexer_topk(wd.q_index, wd.w, wd.k_index, wd.page_table, wd.n_vis, w.K, w.max_n)
    sc = binding.indexer_scores(wd.q_index, wd.w, wd.k_index, wd.page_table, wd.n_vis, w.max_n)
    torch.cuda.synchronize()
    want = ix_oracle.select(sc.cpu().numpy(), w.n_vis.numpy(), w.K)
    assert np.array_equal(got.cpu().numpy(), want)
    ref, bad = ix_oracle.scores(*oracle_args(w))
    assert bad == 0
    gs = sc.cpu().numpy().astype(np.float64)
    for b in range(w.B):
        n = int(w.n_vis[b, 0])
        # scores within the fp32 band (a loose, magnitude-free bound here)
        assert np.all(np.abs(gs[b, 0, :n] - ref[b, 0, :n]) <= 1e-4 * (1 + np.abs(ref[b, 0, :n])))
        valid_topk(got[b, 0].cpu().numpy(), ref[b, 0, :n], n, w.K, eps=1e-4 * (1 + np.abs(ref[b, 0, :n]).max()))


def test_indexer_feeds_the_decode():
    """The indexer's lists drive smla_decode exactly as the oracle's lists
    drive the oracle decode (exact-integer index scores, so the lists agree)."""
    import oracle
    from parity_util import check_o_lse
    iw = workloads.make_indexer_workload("ix_feed", B=2, T=1, HI=32, K=512, ctx_lens=[4000, 3000],
                                         seed=17, integer=True)
    dw = workloads.make_workload("ix_feed_decode", B=2, T=1, H=16, K=512, ctx_lens=[4000, 3000],
                                 seed=18)
    assert dw.cache.shape[0] == iw.k_index.shape[0]
    dw.page_table = iw.page_table.clone()       # one page numbering for both caches
    idx = torch.from_numpy(gpu_topk(iw)).view(2, 1, 512)
    want, _ = ix_oracle.topk(*oracle_args(iw), 512)
    assert np.array_equal(idx.numpy(), want)
    dw.idx = idx
    wd = dw.to(DEV)
    o, lse = binding.decode(wd.q, wd.cache, wd.page_table, wd.idx, dw.scale, 0)
    torch.cuda.synchronize()
    o_ref, lse_ref, bad = oracle.decode(bits(dw.q), bits(dw.cache), dw.page_table.numpy(), want,
                                        dw.scale)
    assert bad == 0
    check_o_lse(o, lse, o_ref, lse_ref, "indexer -> decode")


@pytest.mark.parametrize("H", [16, 64])
def test_selection_feeds_the_decode_on_one_stream(H):
    """The production chain: the top-k indexer writes the selection and the
    decode consumes it on the same stream with no synchronisation in between
    (the indexer's last kernel lets its dependents launch early; the decode's
    first kernel waits before it reads).  Two query sets alternate, so a
    decode that read the previous call's selection would differ; each decode
    must equal, bit for bit, a decode of the same selection taken after a
    synchronisation."""
    B, HI, K = 3, 32, 512
    wi = workloads.make_indexer_workload("chain", B=B, T=1, HI=HI, K=K,
                                         ctx_lens=[3000, 9000, 20000], seed=21)
    g = torch.Generator().manual_seed(22)
    qi2 = (torch.randn(wi.q_index.shape, generator=g) * 0.5).to(torch.bfloat16)
    cache = (torch.randn(wi.num_pages, 64, 576, generator=g) * 0.5).to(torch.bfloat16).to(DEV)
    q = (torch.randn(B, 1, H, 576, generator=g) * 0.5).to(torch.bfloat16).to(DEV)
    wd = wi.to(DEV)
    qsets = [wd.q_index, qi2.to(DEV)]
    idx = torch.empty((B, 1, K), dtype=torch.int32, device=DEV)
    scale = 576 ** -0.5
    binding.indexer_topk(qsets[0], wd.w, wd.k_index, wd.page_table, wd.n_vis, K, wi.max_n, out=idx)
    binding.decode(q, cache, wd.page_table, idx, scale, 0)  # allocator warm-up
    torch.cuda.synchronize()
    picks = []
    for c in range(8):
        binding.indexer_topk(qsets[c % 2], wd.w, wd.k_index, wd.page_table, wd.n_vis, K, wi.max_n,
                             out=idx)
        o, lse = binding.decode(q, cache, wd.page_table, idx, scale, 0)
        torch.cuda.synchronize()
        sel = idx.clone()
        o_ref, lse_ref = binding.decode(q, cache, wd.page_table, sel, scale, 0)
        torch.cuda.synchronize()
        assert torch.equal(o, o_ref) and torch.equal(lse, lse_ref), f"call {c}"
        picks.append(sel.cpu())
    assert not torch.equal(picks[0], picks[1])  # the two query sets select differently
    assert all(torch.equal(picks[c], picks[c % 2]) for c in range(8))
