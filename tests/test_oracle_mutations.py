"""The oracle's pins catch plausible mistakes.

Each case plants one mistake in a copy of the oracle's C source (on the CPU,
in a temporary directory), builds it, and checks that at least one pin from
``test_oracle_pins`` fails against the planted build while all of them pass
against the real one.
"""
import math
import os
import subprocess
import tempfile

import numpy as np
import pytest

import oracle
from oracle.oracle import load_library

from test_oracle_pins import (GOLDEN, bits_to_f64, brute_force, parse_num, small_workload,
                              to_bits, wl_arrays)

SRC = os.path.join(os.path.dirname(oracle.__file__), "smla_oracle.c")

MUTATIONS = {
    "drop_rope_term": ("return scale * (dot_nope + dot_pe);", "return scale * (dot_nope);"),
    "rope_sign": ("return scale * (dot_nope + dot_pe);", "return scale * (dot_nope - dot_pe);"),
    "ignore_page_table": ("return (int64_t)page * page_size + (i % page_size);",
                          "return (int64_t)i;"),
    "slot_from_page_number": ("return (int64_t)page * page_size + (i % page_size);",
                              "return (int64_t)page * page_size + (i / page_size);"),
    "log2_lse": ("lse[u] = m + log(l);", "lse[u] = m + log2(l);"),
    "no_normalise": ("oh[d] /= l;", "oh[d] /= 1.0;"),
    "split_boundary_off_by_one": ("int j1 = j0 + Kc;", "int j1 = j0 + Kc - 1;"),
    "combine_weight_uses_lse": ("const double w = exp(m_u[s] - M);",
                                "const double w = exp(lse_u[s] - M);"),
    "padding_counted_as_error": ("if (i == -1)\n        return -1;", "if (i == -2)\n        return -1;"),
    "rope_reads_latent_q": ("bf16_bits_to_double(qh[dc + d])", "bf16_bits_to_double(qh[d])"),
    "output_reads_shifted_row": ("out[d] += w * bf16_bits_to_double(c[d]);",
                                 "out[d] += w * bf16_bits_to_double(c[d + 1]);"),
    "scale_outside_softmax": ("double w = exp(s_buf[v] - m);", "double w = exp((s_buf[v] - m) / scale);"),
}


def run_pins(lib) -> list:
    """Run a compact set of the pins against ``lib``; return the names that fail."""
    import json
    failures = []

    def check(name, fn):
        try:
            fn()
        except AssertionError:
            failures.append(name)

    def golden():
        for case in json.load(open(GOLDEN))["cases"]:
            dc, dr, ps = case["dc"], case["dr"], case["page_size"]
            q = to_bits(case["q"]).reshape(1, 1, -1, dc + dr)
            cache = to_bits(case["rows"]).reshape(-1, dc + dr)
            pt = np.asarray([case["page_table"]], np.int32)
            idx = np.asarray([[case["idx"]]], np.int32)
            o, lse, bad = oracle.decode(q, cache, pt, idx, parse_num(case["scale"]), dc=dc,
                                        dr=dr, page_size=ps, lib=lib)
            assert bad == 0
            np.testing.assert_allclose(o[0, 0], np.asarray(case["expect_o"]), rtol=1e-14,
                                       atol=1e-14)
            want = parse_num(case["expect_lse"][0])
            got = lse[0, 0, 0]
            assert (got == want) if want == -math.inf else abs(got - want) < 1e-13

    def topk1():
        w = small_workload(K=1, H=3)
        q, cache, pt, idx = wl_arrays(w)
        o, lse, bad = oracle.decode(q, cache, pt, idx, w.scale, lib=lib)
        assert bad == 0
        rows = cache.reshape(-1, 576)
        for b in range(w.B):
            for t in range(w.T):
                i = int(idx[b, t, 0])
                r = int(pt[b, i // 64]) * 64 + i % 64
                for h in range(w.H):
                    np.testing.assert_array_equal(o[b, t, h], bits_to_f64(rows[r, :512]))

    def split():
        w = small_workload(K=72, B=1, T=2, H=3)
        q, cache, pt, idx = wl_arrays(w)
        o, lse, _ = oracle.decode(q, cache, pt, idx, w.scale, lib=lib)
        for nsplit in (3, 7, 16):
            po, pm, pl, _ = oracle.partial(q, cache, pt, idx, w.scale, nsplit, lib=lib)
            oc, lc = oracle.combine(po, pm, pl, lib=lib)
            np.testing.assert_allclose(oc, o, rtol=1e-12, atol=1e-15)
            np.testing.assert_allclose(lc, lse, rtol=1e-13)

    def brute():
        rng = np.random.default_rng(0)
        dc, dr, ps = 6, 3, 4
        qf = (rng.integers(-8, 9, size=(2, 2, 2, dc + dr)) * 0.25).astype(np.float32)
        rf = (rng.integers(-8, 9, size=(20, dc + dr)) * 0.25).astype(np.float32)
        pt = np.stack([rng.permutation(5)[:3] for _ in range(2)]).astype(np.int32)
        idx = np.stack([[rng.permutation(12)[:7] for _ in range(2)] for _ in range(2)]).astype(np.int32)
        o, lse, _ = oracle.decode(to_bits(qf), to_bits(rf), pt, idx, 0.37, dc=dc, dr=dr,
                                  page_size=ps, lib=lib)
        ob, lb = brute_force(qf.astype(np.float64), rf.astype(np.float64), pt, idx, 0.37,
                             dc, dr, ps)
        np.testing.assert_allclose(o, ob, rtol=1e-12, atol=1e-14)
        np.testing.assert_allclose(lse, lb, rtol=1e-13)

    for name, fn in [("golden", golden), ("topk1", topk1), ("split", split), ("brute", brute)]:
        check(name, fn)
    return failures


def build_variant(src_text: str, tmpdir: str, tag: str):
    c_path = os.path.join(tmpdir, f"{tag}.c")
    so_path = os.path.join(tmpdir, f"lib{tag}.so")
    with open(c_path, "w") as f:
        f.write(src_text)
    subprocess.run(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", c_path, "-o",
                    so_path, "-lm"], check=True)
    return load_library(so_path)


def test_unmutated_oracle_passes_every_pin():
    assert run_pins(None) == []


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_mistake_is_caught(name):
    old, new = MUTATIONS[name]
    src = open(SRC).read()
    assert src.count(old) >= 1, f"mutation anchor for {name} not found"
    with tempfile.TemporaryDirectory() as d:
        lib = build_variant(src.replace(old, new), d, name)
        failures = run_pins(lib)
    assert failures, f"no pin caught the planted mistake '{name}'"


# ---------------------------------------------------------------- dense-context variant
def _dense_mutant(kind):
    """A copy of the oracle's position-list construction with one mistake."""
    def dense_positions(seq_lens, K):
        seq_lens = np.asarray(seq_lens, np.int64)
        if seq_lens.size and (seq_lens.min() < 0 or seq_lens.max() > K):
            raise ValueError("seq_lens must lie in [0, K]")
        j = np.arange(K, dtype=np.int64)[None, None, :]
        n = seq_lens[..., None]
        if kind == "prefix_one_too_long":
            return np.where(j <= n, j, -1).astype(np.int32)
        if kind == "prefix_one_too_short":
            return np.where(j < n - 1, j, -1).astype(np.int32)
        if kind == "positions_from_one":
            return np.where(j < n, j + 1, -1).astype(np.int32)
        raise AssertionError(kind)
    return dense_positions


def run_dense_pins() -> list:
    import test_oracle_pins as pins
    failures = []
    for name in ("test_dense_positions_hand_case", "test_dense_single_position_returns_first_row_exactly",
                 "test_dense_equal_scores_give_mean_of_prefix", "test_dense_is_causal"):
        try:
            getattr(pins, name)()
        except (AssertionError, ValueError):
            failures.append(name)
    return failures


def test_unmutated_dense_oracle_passes_its_pins():
    assert run_dense_pins() == []


@pytest.mark.parametrize("kind", ["prefix_one_too_long", "prefix_one_too_short",
                                  "positions_from_one"])
def test_planted_dense_mistake_is_caught(kind, monkeypatch):
    mutant = _dense_mutant(kind)
    monkeypatch.setattr(oracle.oracle, "dense_positions", mutant)
    monkeypatch.setattr(oracle, "dense_positions", mutant)
    assert run_dense_pins(), f"no pin caught the planted dense mistake '{kind}'"
