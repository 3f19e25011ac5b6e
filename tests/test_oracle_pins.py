"""Pins for the fp64 CPU oracle: checks against what the mathematics fixes.

Each test fixes the oracle to something other than itself: hand-derived
closed forms (tests/golden/closed_forms.json), special cases whose answer is
known (top-k = 1, equal scores, an all-padding list, a peaked softmax),
invariances the definition implies (index order, padding placement, page
relabelling, split count) and a brute-force evaluation on tiny inputs.

The operation: "The Moment of Truth: Validating Split-K Parallelization for
Blackwell MLA Decode", section "The Split-K Imperative" (top-k candidate
rows, split-K partials, LSE combine); "The Occupancy Hypothesis ...",
section "The Occupancy Insight" (NSPLIT chunks of one query's work).
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from sparse_mla_decode_partial_b200 import workloads

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "closed_forms.json")


def to_bits(x) -> np.ndarray:
    """float values -> bf16 bit patterns; asserts the values are bf16-exact."""
    t = torch.as_tensor(np.asarray(x, np.float32))
    b = t.to(torch.bfloat16)
    assert torch.equal(b.to(torch.float32), t), "value not exact in bf16"
    return b.view(torch.int16).numpy().view(np.uint16)


def bits_to_f64(bits) -> np.ndarray:
    return (np.asarray(bits, np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def torch_bits(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def wl_arrays(w):
    return (torch_bits(w.q), torch_bits(w.cache), w.page_table.numpy(), w.idx.numpy())


def small_workload(seed=11, B=2, T=2, H=4, K=40, ctx=300, **kw):
    return workloads.make_workload("pin", B=B, T=T, H=H, K=K, ctx_lens=[ctx] * B,
                                   seed=seed, **kw)


def parse_num(s):
    if isinstance(s, (int, float)):
        return float(s)
    table = {"ln3": math.log(3.0), "ln4": math.log(4.0), "2.5+ln2": 2.5 + math.log(2.0),
             "-inf": -math.inf}
    return table[s] if s in table else float(s)


# ---------------------------------------------------------------- closed forms
@pytest.mark.parametrize("case", json.load(open(GOLDEN))["cases"], ids=lambda c: c["name"])
def test_golden_closed_forms(case):
    dc, dr, ps = case["dc"], case["dr"], case["page_size"]
    q = to_bits(case["q"]).reshape(1, 1, -1, dc + dr)
    cache = to_bits(case["rows"]).reshape(-1, dc + dr)
    pt = np.asarray([case["page_table"]], np.int32)
    idx = np.asarray([[case["idx"]]], np.int32)
    o, lse, _ = oracle.decode(q, cache, pt, idx, parse_num(case["scale"]),
                              dc=dc, dr=dr, page_size=ps)
    np.testing.assert_allclose(o[0, 0], np.asarray(case["expect_o"]), rtol=1e-14, atol=1e-14)
    exp_lse = [parse_num(v) for v in case["expect_lse"]]
    for got, want in zip(lse[0, 0], exp_lse):
        if want == -math.inf:
            assert got == -math.inf
        else:
            assert abs(got - want) <= 1e-14 * max(1.0, abs(want))


def test_integer_scores_full_width():
    """Full 512+64 width: q_nope.c = 2*5, q_pe.k_pe = -3, scale 0.25 -> s = 1.75."""
    D = 576
    q = np.zeros((1, 1, 1, D), np.float32)
    row = np.zeros((1, D), np.float32)
    for d in (0, 100, 255, 256, 511):       # five matches of 1*2 in the latent part
        q[0, 0, 0, d] = 1.0
        row[0, d] = 2.0
    for d in (512, 540, 575):               # three matches of 1*(-1) in the rope part
        q[0, 0, 0, d] = 1.0
        row[0, d] = -1.0
    cache = np.zeros((64, D), np.float32)
    cache[17] = row[0]
    o, lse, bad = oracle.decode(to_bits(q), to_bits(cache), np.zeros((1, 1), np.int32),
                                np.asarray([[[17]]], np.int32), 0.25)
    assert bad == 0
    assert lse[0, 0, 0] == 0.25 * (10.0 - 3.0)
    np.testing.assert_array_equal(o[0, 0, 0], cache[17, :512].astype(np.float64))


# ---------------------------------------------------------------- special cases
def test_topk1_returns_that_row_exactly():
    w = small_workload(K=1, H=3)
    q, cache, pt, idx = wl_arrays(w)
    o, lse, bad = oracle.decode(q, cache, pt, idx, w.scale)
    assert bad == 0
    rows = cache.reshape(-1, 576)
    for b in range(w.B):
        for t in range(w.T):
            i = int(idx[b, t, 0])
            r = int(pt[b, i // 64]) * 64 + i % 64
            want = bits_to_f64(rows[r, :512])
            for h in range(w.H):
                np.testing.assert_array_equal(o[b, t, h], want)
                assert np.isfinite(lse[b, t, h])


def test_equal_scores_give_mean_and_log_count():
    w = small_workload(K=33)
    q, cache, pt, idx = wl_arrays(w)
    q = np.zeros_like(q)                     # every score is 0
    idx = idx.copy()
    idx[0, 0, ::4] = -1                      # interleaved padding
    o, lse, _ = oracle.decode(q, cache, pt, idx, w.scale)
    rows = bits_to_f64(cache.reshape(-1, 576))
    for b in range(w.B):
        for t in range(w.T):
            sel = [int(pt[b, i // 64]) * 64 + i % 64 for i in idx[b, t] if i >= 0]
            mean = rows[sel, :512].mean(axis=0)
            for h in range(w.H):
                np.testing.assert_allclose(o[b, t, h], mean, rtol=1e-13, atol=1e-15)
                assert abs(lse[b, t, h] - math.log(len(sel))) < 1e-14


def test_shared_rope_key_equal_scores():
    """q_nope = 0 and one shared k_pe: equal scores s = scale*q_pe.k_pe, o = mean c."""
    w = small_workload(K=20, B=1, T=1, H=2)
    q, cache, pt, idx = wl_arrays(w)
    q = q.copy()
    q[..., :512] = 0
    cache = cache.copy().reshape(-1, 576)
    cache[:, 512:] = cache[0, 512:]          # every row shares row 0's rope key
    o, lse, _ = oracle.decode(q, cache, pt, idx, w.scale)
    rows = bits_to_f64(cache)
    sel = [int(pt[0, i // 64]) * 64 + i % 64 for i in idx[0, 0]]
    mean = rows[sel, :512].mean(axis=0)
    for h in range(2):
        s = w.scale * float(np.dot(bits_to_f64(q[0, 0, h, 512:]), rows[0, 512:]))
        np.testing.assert_allclose(o[0, 0, h], mean, rtol=1e-13, atol=1e-15)
        assert abs(lse[0, 0, h] - (s + math.log(len(sel)))) < 1e-13


def test_all_padding_gives_zero_and_minus_inf():
    w = small_workload()
    q, cache, pt, idx = wl_arrays(w)
    idx = np.full_like(idx, -1)
    o, lse, bad = oracle.decode(q, cache, pt, idx, w.scale)
    assert bad == 0
    assert np.all(o == 0.0) and np.all(lse == -np.inf)


def test_peaked_softmax_selects_argmax_row():
    """A huge scale makes one score dominate by > 700: o is that row, lse its score."""
    w = small_workload(K=16, B=1, T=1, H=3)
    q, cache, pt, idx = wl_arrays(w)
    rows = bits_to_f64(cache.reshape(-1, 576))
    sel = [int(pt[0, i // 64]) * 64 + i % 64 for i in idx[0, 0]]
    for scale in (1e4, -1e4):
        o, lse, _ = oracle.decode(q, cache, pt, idx, scale)
        for h in range(3):
            qh = bits_to_f64(q[0, 0, h])
            dots = np.array([float(np.dot(qh, rows[r])) for r in sel])
            s = scale * dots
            top = int(np.argmax(s))
            gap = s[top] - np.partition(s, -2)[-2]
            assert gap > 745                  # exp(-745) underflows to 0 in fp64
            np.testing.assert_array_equal(o[0, 0, h], rows[sel[top], :512])
            assert lse[0, 0, h] == s[top]
            assert np.all(np.isfinite(o))


# ---------------------------------------------------------------- invariances
def test_index_order_invariance():
    w = small_workload(K=64)
    q, cache, pt, idx = wl_arrays(w)
    o1, l1, _ = oracle.decode(q, cache, pt, idx, w.scale)
    rng = np.random.default_rng(5)
    idx2 = np.stack([[rng.permutation(idx[b, t]) for t in range(w.T)] for b in range(w.B)])
    o2, l2, _ = oracle.decode(q, cache, pt, idx2, w.scale)
    np.testing.assert_allclose(o2, o1, rtol=1e-12, atol=1e-15)
    np.testing.assert_allclose(l2, l1, rtol=1e-13)


def test_padding_equals_compacted():
    w = small_workload(K=30)
    q, cache, pt, idx = wl_arrays(w)
    o1, l1, _ = oracle.decode(q, cache, pt, idx, w.scale)
    rng = np.random.default_rng(7)
    padded = np.full((w.B, w.T, 50), -1, np.int32)
    for b in range(w.B):
        for t in range(w.T):
            slots = np.sort(rng.choice(50, 30, replace=False))
            padded[b, t, slots] = idx[b, t]
    o2, l2, bad = oracle.decode(q, cache, pt, padded, w.scale)
    assert bad == 0
    np.testing.assert_allclose(o2, o1, rtol=1e-12, atol=1e-15)
    np.testing.assert_allclose(l2, l1, rtol=1e-13)


def test_page_relabelling_invariance():
    """Identity page table over cache C == shuffled table over C permuted to match."""
    w = small_workload(K=50, paged=False)
    q, cache, pt, idx = wl_arrays(w)
    o1, l1, _ = oracle.decode(q, cache, pt, idx, w.scale)
    P = cache.shape[0]
    perm = np.random.default_rng(3).permutation(P).astype(np.int32)
    cache2 = np.empty_like(cache)
    cache2[perm] = cache                     # logical page p now lives at perm[p]
    pt2 = perm[pt]
    o2, l2, _ = oracle.decode(q, cache2, pt2, idx, w.scale)
    np.testing.assert_array_equal(o2, o1)
    np.testing.assert_array_equal(l2, l1)


def test_out_of_range_entries_are_masked_and_counted():
    w = small_workload(K=12, B=1, T=1, H=2)
    q, cache, pt, idx = wl_arrays(w)
    ref_idx = idx.copy()
    ref_idx[0, 0, :3] = -1
    o1, l1, bad1 = oracle.decode(q, cache, pt, ref_idx, w.scale)
    assert bad1 == 0
    bad_idx = idx.copy()
    bad_idx[0, 0, 0] = -7                                  # negative, not -1
    bad_idx[0, 0, 1] = pt.shape[1] * 64                    # past the page table
    pt2 = np.concatenate([pt, np.asarray([[cache.shape[0] + 3]], np.int32)], axis=1)
    bad_idx[0, 0, 2] = pt.shape[1] * 64 + 5                # page entry out of range
    o2, l2, bad2 = oracle.decode(q, cache, pt2, bad_idx, w.scale)
    assert bad2 == 3 * 2                                   # counted per head
    np.testing.assert_array_equal(o2, o1)
    np.testing.assert_array_equal(l2, l1)


# ---------------------------------------------------------------- split-K algebra
@pytest.mark.parametrize("nsplit", [1, 2, 3, 4, 7, 16, 64, 72, 77])
def test_split_combine_equals_unsplit(nsplit):
    w = small_workload(K=72, B=1, T=2, H=3)
    q, cache, pt, idx = wl_arrays(w)
    idx = idx.copy()
    idx[0, 1, 40:] = -1                      # a tail of padding: some splits empty
    o, lse, _ = oracle.decode(q, cache, pt, idx, w.scale)
    po, pm, pl, _ = oracle.partial(q, cache, pt, idx, w.scale, nsplit)
    assert po.shape == (1, 2, 3, nsplit, 512)
    oc, lc = oracle.combine(po, pm, pl)
    assert np.all(np.isfinite(oc)) and np.all(np.isfinite(lc))
    np.testing.assert_allclose(oc, o, rtol=1e-12, atol=1e-15)
    np.testing.assert_allclose(lc, lse, rtol=1e-13)


def test_partial_split_boundaries_and_empty_splits():
    """Kc = ceil(K/S); split s holds positions [s*Kc, (s+1)*Kc); beyond K it is empty."""
    w = small_workload(K=10, B=1, T=1, H=1)
    q, cache, pt, idx = wl_arrays(w)
    po, pm, pl, _ = oracle.partial(q, cache, pt, idx, w.scale, 4)   # Kc = 3: 3,3,3,1
    for s, (j0, j1) in enumerate([(0, 3), (3, 6), (6, 9), (9, 10)]):
        o1, l1, _ = oracle.decode(q, cache, pt, idx[:, :, j0:j1], w.scale)
        # a single split's normalised output and lse equal the decode of its slice
        np.testing.assert_allclose(po[0, 0, 0, s] * np.exp(pm[0, 0, 0, s] - pl[0, 0, 0, s]),
                                   o1[0, 0, 0], rtol=1e-12, atol=1e-15)
        assert abs(pl[0, 0, 0, s] - l1[0, 0, 0]) < 1e-13
    po, pm, pl, _ = oracle.partial(q, cache, pt, idx, w.scale, 13)  # Kc = 1: splits 10..12 empty
    assert np.all(pm[..., 10:] == -np.inf) and np.all(pl[..., 10:] == -np.inf)
    assert np.all(po[..., 10:, :] == 0.0)
    assert np.all(np.isfinite(pm[..., :10]))


def test_combine_closed_form_with_empty_split():
    """Two one-row splits with scores ln3 and 0 plus an empty split: weights 3/4, 1/4."""
    c1 = np.arange(512, dtype=np.float64) * 0.5 - 7
    c2 = np.cos(np.arange(512, dtype=np.float64))
    a, b = math.log(3.0), 0.0
    po = np.stack([c1, np.zeros(512), c2])[None]       # O_s = exp(s - m_s) c = c
    pm = np.asarray([[a, -np.inf, b]])
    pl = np.asarray([[a, -np.inf, b]])
    o, lse = oracle.combine(po, pm, pl)
    np.testing.assert_allclose(o[0], 0.75 * c1 + 0.25 * c2, rtol=1e-14, atol=1e-14)
    assert abs(lse[0] - math.log(4.0)) < 1e-15
    o, lse = oracle.combine(np.zeros((1, 2, 512)), np.full((1, 2), -np.inf),
                            np.full((1, 2), -np.inf))
    assert np.all(o == 0) and lse[0] == -np.inf


# ---------------------------------------------------------------- brute force
def brute_force(q, rows, pt, idx, scale, dc, dr, ps):
    """exp(s_j) / sum_k exp(s_k) with no max shift, pure Python, math.fsum."""
    B, T, H, _ = q.shape
    o = np.zeros((B, T, H, dc))
    lse = np.zeros((B, T, H))
    for b in range(B):
        for t in range(T):
            sel = []
            for i in idx[b, t]:
                i = int(i)
                if i == -1:
                    continue
                sel.append(int(pt[b][i // ps]) * ps + i % ps)
            for h in range(H):
                e = [math.exp(scale * math.fsum(float(q[b, t, h, d]) * float(rows[r, d])
                                                 for d in range(dc + dr))) for r in sel]
                Z = math.fsum(e)
                lse[b, t, h] = math.log(Z) if sel else -math.inf
                for d in range(dc):
                    o[b, t, h, d] = math.fsum(e[k] * float(rows[sel[k], d])
                                              for k in range(len(sel))) / Z if sel else 0.0
    return o, lse


@pytest.mark.parametrize("seed", [0, 1, 2, 3])
def test_brute_force_tiny(seed):
    rng = np.random.default_rng(seed)
    dc, dr, ps = 6, 3, 4
    B, T, H, K, pages = 2, 2, 2, 7, 5
    qf = (rng.integers(-8, 9, size=(B, T, H, dc + dr)) * 0.25).astype(np.float32)
    rf = (rng.integers(-8, 9, size=(pages * ps, dc + dr)) * 0.25).astype(np.float32)
    pt = np.stack([rng.permutation(pages)[:3] for _ in range(B)]).astype(np.int32)
    idx = np.stack([[rng.permutation(12)[:K] for _ in range(T)] for _ in range(B)]).astype(np.int32)
    idx[0, 1, [1, 4]] = -1
    scale = 0.37
    o, lse, bad = oracle.decode(to_bits(qf), to_bits(rf), pt, idx, scale, dc=dc, dr=dr,
                                page_size=ps)
    assert bad == 0
    ob, lb = brute_force(qf.astype(np.float64), rf.astype(np.float64), pt, idx, scale,
                         dc, dr, ps)
    np.testing.assert_allclose(o, ob, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(lse, lb, rtol=1e-13)
    for nsplit in (2, 3, 5, 9):
        oc, lc = oracle.combine(*oracle.partial(to_bits(qf), to_bits(rf), pt, idx, scale,
                                                nsplit, dc=dc, dr=dr, page_size=ps)[:3])
        np.testing.assert_allclose(oc, ob, rtol=1e-12, atol=1e-14)
        np.testing.assert_allclose(lc, lb, rtol=1e-13)


def test_large_scores_no_overflow():
    """Scores near +-1e4 would overflow a shift-free exp; the oracle stays finite."""
    w = small_workload(K=24, B=1, T=1, H=2)
    q, cache, pt, idx = wl_arrays(w)
    o, lse, _ = oracle.decode(q, cache, pt, idx, 300.0)
    assert np.all(np.isfinite(o)) and np.all(np.isfinite(lse))
    assert np.abs(lse).max() > 700           # exp(lse) itself would overflow
    po, pm, pl, _ = oracle.partial(q, cache, pt, idx, 300.0, 5)
    oc, lc = oracle.combine(po, pm, pl)
    np.testing.assert_allclose(oc, o, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(lc, lse, rtol=1e-13)


# ---------------------------------------------------------------- dense-context variant
# "The Occupancy Hypothesis: How One Kernel Parameter Unlocked 1.8x Decode
# Speedup on Blackwell", sections "The Occupancy Insight" and "The Broader
# Context": the verify kernel splits each query token's whole visible KV
# sequence.  The oracle builds the positions 0 .. n-1 as an index list and
# runs the sparse definition pinned above; these pins fix the list.
def dense_workload(B=2, T=3, H=3, ctx=(200, 130), seed=21):
    return workloads.make_dense_workload("pin_dense", B=B, T=T, H=H, ctx_lens=list(ctx), seed=seed)


def dense_arrays(w):
    return torch_bits(w.q), torch_bits(w.cache), w.page_table.numpy(), w.seq_lens.numpy()


def test_dense_positions_hand_case():
    got = oracle.dense_positions([[3, 0], [4, 1]], 4)
    want = [[[0, 1, 2, -1], [-1, -1, -1, -1]], [[0, 1, 2, 3], [0, -1, -1, -1]]]
    np.testing.assert_array_equal(got, np.asarray(want, np.int32))
    for bad in ([[5]], [[-1]]):
        with pytest.raises(ValueError):
            oracle.dense_positions(bad, 4)


def test_dense_workload_lengths_are_causal():
    """Draft token t of a sequence of n tokens sees n - T + t + 1 positions."""
    w = dense_workload()
    np.testing.assert_array_equal(w.seq_lens.numpy(), [[198, 199, 200], [128, 129, 130]])


def test_dense_single_position_returns_first_row_exactly():
    w = dense_workload()
    q, cache, pt, _ = dense_arrays(w)
    o, lse, bad = oracle.decode_dense(q, cache, pt, np.ones((2, 3), np.int32), w.scale)
    assert bad == 0
    rows = cache.reshape(-1, 576)
    for b in range(2):
        want = bits_to_f64(rows[int(pt[b, 0]) * 64, :512])   # position 0 = page pt[b,0], slot 0
        for t in range(3):
            for h in range(3):
                np.testing.assert_array_equal(o[b, t, h], want)
                assert np.isfinite(lse[b, t, h])


def test_dense_equal_scores_give_mean_of_prefix():
    w = dense_workload()
    q, cache, pt, lens = dense_arrays(w)
    q = np.zeros_like(q)                      # every score is 0
    lens = lens.copy()
    lens[1, 0] = 0                            # an empty prefix
    o, lse, _ = oracle.decode_dense(q, cache, pt, lens, w.scale, K=int(lens.max()) + 5)
    rows = bits_to_f64(cache.reshape(-1, 576))
    for b in range(2):
        for t in range(3):
            n = int(lens[b, t])
            if n == 0:
                assert np.all(o[b, t] == 0) and np.all(lse[b, t] == -np.inf)
                continue
            sel = [int(pt[b, i // 64]) * 64 + i % 64 for i in range(n)]
            mean = rows[sel, :512].mean(axis=0)
            for h in range(3):
                np.testing.assert_allclose(o[b, t, h], mean, rtol=1e-13, atol=1e-15)
                assert abs(lse[b, t, h] - math.log(n)) < 1e-13


def test_dense_is_causal():
    """Token t's output depends on the positions below its length only."""
    w = dense_workload(B=1, T=4, H=2, ctx=(150,), seed=23)
    q, cache, pt, lens = dense_arrays(w)              # lens 147, 148, 149, 150
    o1, l1, _ = oracle.decode_dense(q, cache, pt, lens, w.scale)
    cache2 = cache.copy().reshape(-1, 576)
    rng = np.random.default_rng(4)
    for i in (147, 148, 149):                         # the rows of the last three draft tokens
        r = int(pt[0, i // 64]) * 64 + i % 64
        cache2[r] = to_bits(rng.integers(-8, 8, 576) / 4.0)
    o2, l2, _ = oracle.decode_dense(q, cache2.reshape(cache.shape), pt, lens, w.scale)
    np.testing.assert_array_equal(o2[0, 0], o1[0, 0])
    np.testing.assert_array_equal(l2[0, 0], l1[0, 0])
    for t in (1, 2, 3):
        assert np.abs(o2[0, t] - o1[0, t]).max() > 1e-6

