"""Pins of the fp64 top-k indexer oracle (CPU only).

The indexer is named on "The Negative Result That Refined the Hunt: Disabling
the MMA FlashMLA Kernel" (section "The Context: A Systematic Bisection
Campaign": an indexer kernel and a bf16 index-key path run ahead of the
sparse decode).  The oracle's reading -- I[s] = sum_j w[j] max(0, qI[j].kI[s]),
the min(K, n) largest scores, ties to the smaller position, output ascending
then -1 -- is pinned here by a hand-worked case, brute force in pure Python on
exact (integer-valued) inputs, invariances and properties; the second half
plants plausible mistakes in a copy of the C source and checks that a pin
fails for each.
"""
import json
import math
import os

import numpy as np
import pytest

from oracle import indexer

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "indexer_hand_case.json")


def to_bits(x):
    """float values -> bf16 bit patterns (values must be exactly representable)."""
    f = np.asarray(x, np.float32)
    b = (f.view(np.uint32) >> 16).astype(np.uint16)
    assert np.array_equal((b.astype(np.uint32) << 16).view(np.float32), f), "not bf16-exact"
    return b


def hand_case():
    c = json.load(open(GOLDEN))
    q = to_bits(c["qI"]).reshape(1, 1, 2, 2)
    w = np.asarray([[c["w"]]], np.float32)
    k = to_bits(c["rows"])
    pt = np.asarray([c["page_table"]], np.int32)
    return c, q, w, k, pt


def random_case(rng, B=2, T=2, HI=4, DI=8, pages=6, page_size=4, integer=True, spread=2):
    """Small random inputs; integer-valued ones make every score exact in
    fp64 and in pure Python alike."""
    if integer:
        q = rng.integers(-spread, spread + 1, (B, T, HI, DI)).astype(np.float32)
        k = rng.integers(-spread, spread + 1, (pages * page_size, DI)).astype(np.float32)
        w = rng.integers(-3, 4, (B, T, HI)).astype(np.float32)
    else:
        # multiples of 1/16 below 8 in magnitude: at most 7 significant bits, bf16-exact
        q = np.clip(np.round(rng.normal(size=(B, T, HI, DI)) * 16), -127, 127) / 16
        k = np.clip(np.round(rng.normal(size=(pages * page_size, DI)) * 16), -127, 127) / 16
        w = rng.normal(size=(B, T, HI)).astype(np.float32)
    pt_stride = pages
    pt = np.stack([rng.permutation(pages) for _ in range(B)]).astype(np.int32)
    n = rng.integers(0, pt_stride * page_size + 1, (B, T)).astype(np.int32)
    return to_bits(q), w.astype(np.float32), to_bits(k), pt, n, page_size


def brute(q_bits, w, k_bits, pt, n, K, page_size):
    """Pure-Python restatement: math.fsum scores, Python's sort on
    (-score, position), ascending output."""
    f = lambda b: float((np.uint32(b) << np.uint32(16)).view(np.float32))
    B, T, HI, DI = q_bits.shape
    out = np.full((B, T, K), -1, np.int32)
    for b in range(B):
        for t in range(T):
            cand = []
            for s in range(int(n[b, t])):
                page = int(pt[b, s // page_size])
                r = page * page_size + s % page_size
                total = []
                for j in range(HI):
                    logit = math.fsum(f(q_bits[b, t, j, d]) * f(k_bits[r, d]) for d in range(DI))
                    total.append(float(w[b, t, j]) * max(0.0, logit))
                cand.append((-math.fsum(total), s))
            cand.sort()
            sel = sorted(s for _, s in cand[:K])
            out[b, t, :len(sel)] = sel
    return out


# ---------------------------------------------------------------- pins
def test_hand_case_scores():
    c, q, w, k, pt = hand_case()
    sc, bad = indexer.scores(q, w, k, pt, np.asarray([[6]], np.int32), page_size=c["page_size"])
    assert bad == 0
    assert sc[0, 0].tolist() == c["expect_scores"]


@pytest.mark.parametrize("i", range(7))
def test_hand_case_selection(i):
    c, q, w, k, pt = hand_case()
    case = c["cases"][i]
    idx, bad = indexer.topk(q, w, k, pt, np.asarray([[case["n"]]], np.int32), case["K"],
                            page_size=c["page_size"])
    assert bad == 0
    assert idx[0, 0].tolist() == case["expect"]


@pytest.mark.parametrize("seed", range(6))
def test_brute_force_integer_inputs(seed):
    rng = np.random.default_rng(seed)
    q, w, k, pt, n, ps = random_case(rng, spread=1 + seed % 3)
    for K in (1, 5, 13, 40):
        got, bad = indexer.topk(q, w, k, pt, n, K, page_size=ps)
        assert bad == 0
        assert np.array_equal(got, brute(q, w, k, pt, n, K, ps)), (seed, K)


@pytest.mark.parametrize("seed", range(4))
def test_brute_force_scores_general_inputs(seed):
    rng = np.random.default_rng(100 + seed)
    q, w, k, pt, n, ps = random_case(rng, integer=False)
    sc, _ = indexer.scores(q, w, k, pt, n, page_size=ps)
    f = lambda b: float((np.uint32(b) << np.uint32(16)).view(np.float32))
    for b in range(q.shape[0]):
        for t in range(q.shape[1]):
            for s in range(int(n[b, t])):
                r = int(pt[b, s // ps]) * ps + s % ps
                want = math.fsum(float(w[b, t, j]) * max(0.0, math.fsum(
                    f(q[b, t, j, d]) * f(k[r, d]) for d in range(q.shape[3])))
                    for j in range(q.shape[2]))
                assert abs(sc[b, t, s] - want) <= 1e-12 * (1 + abs(want))
            assert np.all(np.isneginf(sc[b, t, int(n[b, t]):]))


def test_ties_go_to_the_smaller_position():
    # every key identical: every score equal, so the first K positions win
    rng = np.random.default_rng(7)
    q = to_bits(rng.integers(-2, 3, (1, 3, 4, 8)).astype(np.float32))
    k = to_bits(np.tile(np.arange(8, dtype=np.float32) - 3, (40, 1)))
    w = np.ones((1, 3, 4), np.float32)
    pt = np.asarray([rng.permutation(10)], np.int32)
    n = np.asarray([[40, 17, 3]], np.int32)
    idx, _ = indexer.topk(q, w, k, pt, n, 5, page_size=4)
    assert idx[0, 0].tolist() == [0, 1, 2, 3, 4]
    assert idx[0, 1].tolist() == [0, 1, 2, 3, 4]
    assert idx[0, 2].tolist() == [0, 1, 2, -1, -1]


def test_relu_clips_negative_logits_and_weights_sign_matters():
    # one head, one dimension: logit = q * k.  With w > 0 the largest positive
    # keys win; every negative key scores 0 (not its negative logit), so the
    # zero-score positions then fill by position.  With w < 0 the positive
    # keys are the worst.
    k = to_bits(np.asarray([[-5], [3], [-1], [7], [2], [-8]], np.float32))
    q = to_bits(np.asarray([[[[1]]]], np.float32))
    pt = np.asarray([[0]], np.int32)
    n = np.asarray([[6]], np.int32)
    pos, _ = indexer.topk(q, np.asarray([[[1.0]]], np.float32), k, pt, n, 4, page_size=6)
    assert pos[0, 0].tolist() == [0, 1, 3, 4]          # 7, 3, 2, then position 0 (score 0)
    neg, _ = indexer.topk(q, np.asarray([[[-1.0]]], np.float32), k, pt, n, 3, page_size=6)
    assert neg[0, 0].tolist() == [0, 2, 5]             # the score-0 (negative-logit) keys


def test_invariant_to_page_relabelling():
    rng = np.random.default_rng(11)
    q, w, k, pt, n, ps = random_case(rng, B=2, T=2, pages=8, integer=False)
    base, _ = indexer.topk(q, w, k, pt, n, 9, page_size=ps)
    perm = rng.permutation(8)                          # physical page p moves to perm[p]
    k2 = np.empty_like(k).reshape(8, ps, -1)
    k2[perm] = k.reshape(8, ps, -1)
    pt2 = perm[pt].astype(np.int32)
    moved, _ = indexer.topk(q, w, k2.reshape(k.shape), pt2, n, 9, page_size=ps)
    assert np.array_equal(base, moved)


def test_positive_weight_scale_keeps_the_selection():
    rng = np.random.default_rng(12)
    q, w, k, pt, n, ps = random_case(rng, integer=True)
    a, _ = indexer.topk(q, w, k, pt, n, 11, page_size=ps)
    b, _ = indexer.topk(q, w * 4.0, k, pt, n, 11, page_size=ps)
    assert np.array_equal(a, b)


def test_selection_properties_and_nesting():
    rng = np.random.default_rng(13)
    q, w, k, pt, n, ps = random_case(rng, B=3, T=2, pages=10, integer=False)
    prev = None
    for K in range(1, 30, 3):
        idx, _ = indexer.topk(q, w, k, pt, n, K, page_size=ps)
        for b in range(3):
            for t in range(2):
                row = idx[b, t]
                sel = row[row >= 0]
                assert len(sel) == min(K, int(n[b, t]))
                assert np.all(row[len(sel):] == -1)
                assert np.all(np.diff(sel) > 0) and (len(sel) == 0 or sel[-1] < n[b, t])
                if prev is not None:                   # the K-selection grows by nesting
                    p = prev[b, t]
                    assert set(p[p >= 0].tolist()) <= set(sel.tolist())
        prev = idx


def test_bad_pages_are_not_candidates_and_are_counted():
    c, q, w, k, pt, = hand_case()
    pt_bad = np.asarray([[2, 9, 1]], np.int32)         # logical page 1 (s2, s3) maps nowhere
    idx, bad = indexer.topk(q, w, k, pt_bad, np.asarray([[6]], np.int32), 3,
                            page_size=c["page_size"])
    assert bad == 2
    assert idx[0, 0].tolist() == [1, 4, 5]             # s4 (2), s1 (0), s5 (0)
    sc, bad2 = indexer.scores(q, w, k, pt_bad, np.asarray([[6]], np.int32),
                              page_size=c["page_size"])
    assert bad2 == 2 and np.isneginf(sc[0, 0, 2]) and np.isneginf(sc[0, 0, 3])
    # positions past the page table's width are not candidates either
    idx, bad = indexer.topk(q, w, k, pt, np.asarray([[8]], np.int32), 8,
                            page_size=c["page_size"])
    assert bad == 2 and idx[0, 0].tolist() == [0, 1, 2, 3, 4, 5, -1, -1]


def test_select_from_scores_matches_the_whole_oracle():
    """The selection rule on given scores (NaN = not a candidate) picks what
    the whole oracle picks from its own scores, on general inputs and on
    integer ones full of ties; NaN positions are skipped."""
    for seed, integer in ((21, False), (22, True), (23, True)):
        rng = np.random.default_rng(seed)
        q, w, k, pt, n, ps = random_case(rng, B=3, T=2, pages=9, integer=integer)
        sc, _ = indexer.scores(q, w, k, pt, n, page_size=ps)
        sc = np.where(np.isneginf(sc), np.nan, sc)
        for K in (1, 4, 17, 50):
            want, _ = indexer.topk(q, w, k, pt, n, K, page_size=ps)
            assert np.array_equal(indexer.select(sc, n, K), want), (seed, K)
    # NaN skipped; fp32 scores compared as stored
    sc = np.asarray([[[1.5, np.nan, 1.5, 0.25, np.nan, 9.0]]], np.float32)
    assert indexer.select(sc, np.asarray([[6]], np.int32), 3).tolist() == [[[0, 2, 5]]]
    assert indexer.select(sc, np.asarray([[6]], np.int32), 6).tolist() == [[[0, 2, 3, 5, -1, -1]]]
    assert indexer.select(sc, np.asarray([[2]], np.int32), 2).tolist() == [[[0, -1]]]


# ---------------------------------------------------------------- planted mistakes
MUTATIONS = {
    "no_relu": ("double relu = logit > 0.0 ? logit : 0.0;", "double relu = logit;"),
    "weights_dropped": ("total += (double)w_t[j] * relu;", "total += relu;"),
    "ties_to_larger_position": ("return (x->pos < y->pos) ? -1 : (x->pos > y->pos);",
                                "return (x->pos > y->pos) ? -1 : (x->pos < y->pos);"),
    "smallest_scores": ("if (x->score > y->score)\n        return -1;",
                        "if (x->score < y->score)\n        return -1;"),
    "ignore_page_table": ("return (int64_t)page * page_size + s % page_size;", "return s;"),
    "slot_from_page_number": ("return (int64_t)page * page_size + s % page_size;",
                              "return (int64_t)page * page_size + s / page_size;"),
    "one_position_too_few": ("for (int64_t s = 0; s < n; ++s) {\n            int64_t r = ix_row",
                             "for (int64_t s = 0; s + 1 < n; ++s) {\n            int64_t r = ix_row"),
    "output_in_score_order": ("qsort(o, (size_t)take, sizeof(int32_t), ix_by_pos);", "(void)ix_by_pos;"),
    "query_head_stride": ("ix_bf16(q_t[(int64_t)j * DI + d])", "ix_bf16(q_t[d])"),
}


def pins_failing(lib):
    failures = []

    def check(name, fn):
        try:
            fn()
        except AssertionError:
            failures.append(name)

    def hand():
        c, q, w, k, pt = hand_case()
        for case in c["cases"]:
            idx, bad = indexer.topk(q, w, k, pt, np.asarray([[case["n"]]], np.int32), case["K"],
                                    page_size=c["page_size"], lib=lib)
            assert idx[0, 0].tolist() == case["expect"]

    def brute_int():
        for seed in range(3):
            rng = np.random.default_rng(seed)
            q, w, k, pt, n, ps = random_case(rng, spread=1 + seed)
            got, _ = indexer.topk(q, w, k, pt, n, 13, page_size=ps, lib=lib)
            assert np.array_equal(got, brute(q, w, k, pt, n, 13, ps))

    def ties():
        k = to_bits(np.tile(np.arange(8, dtype=np.float32) - 3, (40, 1)))
        q = to_bits(np.ones((1, 1, 4, 8), np.float32))
        idx, _ = indexer.topk(q, np.ones((1, 1, 4), np.float32), k,
                              np.asarray([np.arange(10)], np.int32), np.asarray([[40]], np.int32),
                              5, page_size=4, lib=lib)
        assert idx[0, 0].tolist() == [0, 1, 2, 3, 4]

    check("hand", hand)
    check("brute_int", brute_int)
    check("ties", ties)
    return failures


def test_pins_pass_on_the_real_oracle():
    assert pins_failing(None) == []


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_mistake_is_caught(name, tmp_path):
    old, new = MUTATIONS[name]
    src = open(indexer.SRC).read()
    assert src.count(old) == 1, f"mutation anchor for {name} not unique"
    mutated = tmp_path / "mutant.c"
    mutated.write_text(src.replace(old, new))
    lib = indexer.load_library(indexer.build(force=True, src=str(mutated),
                                             out=str(tmp_path / "libmutant.so")))
    assert pins_failing(lib), f"no pin fails with the planted mistake {name}"
