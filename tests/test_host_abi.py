"""Host-side checks of the C ABI that need no GPU: the library loads, exports
every function include/smla.h declares, rejects bad arguments before any CUDA
call, sizes workspaces as documented, and the NSPLIT heuristic behaves as
its model says."""
import ctypes
import math
import os
import re

import pytest

from sparse_mla_decode_partial_b200 import binding, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER_DIR = os.path.join(ROOT, "include")


@pytest.fixture(scope="module")
def lib():
    build.build()
    return binding.lib()


def declared_functions():
    names = set()
    for fn in os.listdir(HEADER_DIR):
        if fn.endswith(".h"):
            text = open(os.path.join(HEADER_DIR, fn)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names |= set(re.findall(r"\b(smla_\w+)\s*\(", text))
    return sorted(names)


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert "smla_decode" in names and "smla_decode_partial" in names
    for n in names:
        assert hasattr(lib, n), f"{n} declared but not exported"
        assert n in binding.SIGNATURES, f"{n} has no binding signature"


def test_status_strings(lib):
    for code, name in binding.STATUS.items():
        assert binding.status_string(code).startswith(name)
    assert lib.smla_version() >= 100


def test_binding_constants_match_the_header():
    """The binding's shape constants are the header's #defines."""
    import re
    text = open(os.path.join(ROOT, "include", "smla.h")).read()
    want = {name: int(v) for name, v in re.findall(r"#define (SMLA_\w+) \(?(\d+)", text)}
    assert want["SMLA_PAGE_SIZE"] == binding.PAGE_SIZE
    assert want["SMLA_MAX_NSPLIT"] == binding.MAX_NSPLIT
    assert want["SMLA_INDEXER_DIM"] == binding.INDEXER_DIM
    assert want["SMLA_INDEXER_MAX_HEADS"] == binding.INDEXER_MAX_HEADS
    assert want["SMLA_INDEXER_MAX_N"] == binding.INDEXER_MAX_N
    assert want["SMLA_MAX_K"] == binding.MAX_K == 2**30 - 64


def test_workspace_bytes_formula(lib):
    r = lambda x: (x + 255) // 256 * 256
    for B, T, H, S in [(1, 1, 16, 64), (64, 1, 16, 8), (60, 1, 64, 3), (1, 9, 8, 16), (2, 3, 5, 7)]:
        n = B * T * H * S
        assert binding.workspace_bytes(B, T, H, S) == r(n * 512 * 4) + 2 * r(n * 4)
    assert binding.workspace_bytes(1, 1, 1, 0) == 0
    assert binding.workspace_bytes(-1, 1, 1, 1) == 0
    assert binding.workspace_bytes(1, 1, 1, 1025) == 0


FAKE = 0x10000000  # an aligned address that is never dereferenced: every call
                   # below fails its host-side argument check before any CUDA call


def call_partial(lib, q=FAKE, cache=FAKE, num_pages=10, pt=FAKE, pt_stride=4, idx=FAKE, B=1, T=1,
                 H=16, K=64, ps=64, scale=0.1, nsplit=2, po=FAKE, pm=FAKE, pl=FAKE):
    return lib.smla_decode_partial(q, cache, num_pages, pt, pt_stride, idx, B, T, H, K, ps, scale,
                                   nsplit, po, pm, pl, None)


def call_decode(lib, q=FAKE, cache=FAKE, num_pages=10, pt=FAKE, pt_stride=4, idx=FAKE, B=1, T=1,
                H=16, K=64, ps=64, scale=0.1, nsplit=2, ws=FAKE, ws_bytes=1 << 30, o=FAKE,
                lse=FAKE):
    return lib.smla_decode(q, cache, num_pages, pt, pt_stride, idx, B, T, H, K, ps, scale, nsplit,
                           ws, ws_bytes, o, lse, None)


@pytest.mark.parametrize("kw,expect", [
    (dict(ps=32), 2), (dict(H=65), 2), (dict(B=-1), 1), (dict(K=-2), 1), (dict(nsplit=0), 1),
    (dict(nsplit=1025), 1), (dict(q=0), 1), (dict(q=FAKE + 8), 3), (dict(cache=FAKE + 4), 3),
    (dict(idx=FAKE + 2), 3), (dict(po=FAKE + 4), 3), (dict(pm=FAKE + 2), 3), (dict(po=0), 1),
    (dict(num_pages=0), 1), (dict(pt_stride=0), 1), (dict(scale=math.inf), 1),
    (dict(scale=math.nan), 1), (dict(cache=0), 1), (dict(pt=0), 1),
])
def test_partial_rejects_bad_arguments(lib, kw, expect):
    assert call_partial(lib, **kw) == expect


@pytest.mark.parametrize("kw", [dict(B=0), dict(T=0), dict(H=0)])
def test_empty_problem_is_a_noop(lib, kw):
    assert call_partial(lib, **kw) == 0
    assert call_decode(lib, **kw) == 0


@pytest.mark.parametrize("kw,expect", [
    (dict(ws_bytes=100), 4), (dict(ws=0), 1), (dict(ws=FAKE + 8), 3), (dict(o=FAKE + 8), 3),
    (dict(lse=FAKE + 2), 3), (dict(o=0), 1), (dict(nsplit=-1), 1), (dict(ps=16), 2),
])
def test_decode_rejects_bad_arguments(lib, kw, expect):
    assert call_decode(lib, **kw) == expect


def call_dense(lib, q=FAKE, cache=FAKE, num_pages=10, pt=FAKE, pt_stride=4, lens=FAKE, B=1, T=9,
               H=8, K=200, ps=64, scale=0.1, nsplit=2, ws=FAKE, ws_bytes=1 << 30, o=FAKE,
               lse=FAKE):
    return lib.smla_decode_dense(q, cache, num_pages, pt, pt_stride, lens, B, T, H, K, ps, scale,
                                 nsplit, ws, ws_bytes, o, lse, None)


@pytest.mark.parametrize("kw,expect", [
    (dict(ws_bytes=100), 4), (dict(ws=0), 1), (dict(ws=FAKE + 8), 3), (dict(o=FAKE + 8), 3),
    (dict(lse=FAKE + 2), 3), (dict(o=0), 1), (dict(lens=0), 1), (dict(lens=FAKE + 2), 3),
    (dict(nsplit=-1), 1), (dict(nsplit=1025), 1), (dict(ps=16), 2), (dict(H=65), 2),
    (dict(K=-1), 1), (dict(scale=math.nan), 1), (dict(cache=0), 1), (dict(pt=0), 1),
    (dict(B=0), 0), (dict(T=0), 0), (dict(H=0), 0),
])
def test_decode_dense_rejects_bad_arguments(lib, kw, expect):
    assert call_dense(lib, **kw) == expect


def test_dense_workspace_bytes_formula(lib):
    """The split-K partials of [B, T, H, S] (none at nsplit 1)."""
    for B, T, H, K, S in [(1, 9, 8, 46089, 74), (1, 9, 8, 46089, 1), (2, 3, 16, 777, 5),
                          (1, 1, 64, 0, 4)]:
        want = binding.workspace_bytes(B, T, H, S) if S > 1 else 0
        assert binding.dense_workspace_bytes(B, T, H, K, S) == want
    assert binding.dense_workspace_bytes(1, 1, 1, 1, 0) == 0
    assert binding.dense_workspace_bytes(1, 1, 1, -1, 1) == 0


@pytest.mark.parametrize("shape", [(1, 9, 8, 46089), (1, 9, 8, 4105), (2, 3, 16, 777),
                                   (2, 2, 64, 1500), (2, 4, 8, 40), (1, 1, 16, 65536),
                                   (2, 5, 24, 2100), (3, 17, 4, 999)])
def test_dense_nsplit_packs_tokens_into_64_rows(lib, shape, monkeypatch):
    """Up to 64 / H query tokens share a pass, in balanced groups; the NSPLIT
    is the heuristic's for that many units at the one-CTA-per-SM kernel."""
    monkeypatch.delenv("SMLA_NSPLIT", raising=False)
    B, T, H, K = shape
    gmax = max(1, min(T, 64 // H))
    units = -(-T // gmax)
    assert units * gmax >= T and (units - 1) * gmax < T
    assert binding.dense_nsplit(B, T, H, K) == binding.choose_nsplit(B, units, 64, K, 0)


def call_dense_partial(lib, q=FAKE, cache=FAKE, num_pages=10, pt=FAKE, pt_stride=4, lens=FAKE, B=1,
                       T=9, H=8, K=200, ps=64, scale=0.1, nsplit=2, po=FAKE, pm=FAKE, pl=FAKE):
    return lib.smla_decode_dense_partial(q, cache, num_pages, pt, pt_stride, lens, B, T, H, K, ps,
                                         scale, nsplit, po, pm, pl, None)


@pytest.mark.parametrize("kw,expect", [
    (dict(nsplit=0), 1), (dict(nsplit=1025), 1), (dict(po=0), 1), (dict(po=FAKE + 4), 3),
    (dict(pm=FAKE + 2), 3), (dict(lens=0), 1), (dict(H=65), 2), (dict(ps=32), 2),
    (dict(q=FAKE + 8), 3), (dict(B=0), 0),
])
def test_decode_dense_partial_rejects_bad_arguments(lib, kw, expect):
    assert call_dense_partial(lib, **kw) == expect


def test_combine_rejects_bad_arguments(lib):
    c = lambda **kw: lib.smla_lse_combine(kw.get("po", FAKE), kw.get("pm", FAKE),
                                          kw.get("pl", FAKE), kw.get("B", 1), 1, 16,
                                          kw.get("S", 4), kw.get("o", FAKE), kw.get("lse", FAKE),
                                          None)
    assert c(S=0) == 1 and c(S=2000) == 1 and c(B=-1) == 1 and c(po=0) == 1
    assert c(po=FAKE + 4) == 3 and c(o=FAKE + 8) == 3 and c(B=0) == 0


# ------------------------------------------------------------------ NSPLIT heuristic
def model(B, T, H, K, sms):
    """The cost model the library documents, restated for a table check."""
    base = B * T
    slots = sms * (2 if H <= 16 else 1)
    s_max = max(1, min(1024, -(-K // 32)))
    best, best_s = None, 1
    for s in range(1, s_max + 1):
        ctas = base * s
        t = math.ceil(ctas / slots) * (48.0 + math.ceil(K / s))
        if s > 1:
            t += 0.5 * ctas * H * (514 * 4.0) * 2.0 / 1152 / slots
        if best is None or t < best * (1 - 1e-9):
            best, best_s = t, s
    # balanced schedule: one full wave of `slots` CTAs, base + slots pieces
    s_bal = math.ceil(slots / base) + 1
    units = base * -(-K // 32)
    latency_kernel = H <= 32 and math.ceil(K / s_bal) <= 64
    if H <= 32 and 2 <= s_bal <= s_max and units >= 4 * slots and not latency_kernel:
        pieces = base + slots
        t = 48.0 * pieces / slots + units * 32.0 / slots
        t += 0.5 * pieces * H * (514 * 4.0) * 2.0 / 1152 / slots
        if t < best * (1 - 0.15):
            best_s = s_bal
    return best_s


@pytest.mark.parametrize("shape", [(1, 1, 16, 2048), (1, 9, 8, 2048), (64, 1, 16, 2048),
                                   (60, 1, 64, 2048), (1, 1, 8, 256), (4, 1, 16, 100),
                                   (128, 1, 16, 2048), (1, 1, 16, 31), (64, 1, 24, 2048),
                                   (8, 1, 16, 2048), (20, 3, 16, 4096)])
def test_nsplit_heuristic_matches_model(lib, shape, monkeypatch):
    monkeypatch.delenv("SMLA_NSPLIT", raising=False)
    B, T, H, K = shape
    assert binding.choose_nsplit(B, T, H, K, 148) == model(B, T, H, K, 148)


def test_nsplit_heuristic_properties(lib, monkeypatch):
    monkeypatch.delenv("SMLA_NSPLIT", raising=False)
    # one query token on an idle GPU: split as far as the 32-rows floor allows
    assert binding.choose_nsplit(1, 1, 16, 2048, 148) == 64
    # the split count never drops a split below 32 rows (except a single split)
    for K in (1, 20, 33, 64, 65, 1000):
        s = binding.choose_nsplit(1, 1, 16, K, 148)
        assert s == 1 or math.ceil(K / s) >= 32 or s <= -(-K // 32)
    # batched decode on mma.sync (2 CTAs per SM): 4 splits fill one wave well
    # enough that the balanced schedule (6 slots) does not pay
    assert binding.choose_nsplit(64, 1, 16, 2048, 148) == 4
    # a batch that already fills the GPU is not split
    assert binding.choose_nsplit(296, 1, 16, 2048, 148) == 1
    assert binding.choose_nsplit(148, 1, 64, 2048, 148) == 1
    # degenerate sizes
    assert binding.choose_nsplit(0, 1, 16, 2048, 148) == 1
    assert binding.choose_nsplit(1, 1, 16, 0, 148) == 1


def test_nsplit_env_override(lib, monkeypatch):
    monkeypatch.setenv("SMLA_NSPLIT", "37")
    assert binding.choose_nsplit(64, 1, 16, 2048, 148) == 37
    monkeypatch.setenv("SMLA_NSPLIT", "99999")
    assert binding.choose_nsplit(64, 1, 16, 2048, 148) == 1024
    monkeypatch.setenv("SMLA_NSPLIT", "junk")
    assert binding.choose_nsplit(1, 1, 16, 2048, 148) == 64


def balanced_items(B, T, K, grid):
    """Work pieces of the balanced schedule, as the kernels enumerate them."""
    tpt = -(-K // 32)
    U = B * T * tpt
    owner = lambda u: ((u + 1) * grid - 1) // U
    out = []
    for c in range(grid):
        u, u_end = c * U // grid, (c + 1) * U // grid
        while u < u_end:
            bt = u // tpt
            ue = min(u_end, (bt + 1) * tpt)
            out.append((c, bt, (u - bt * tpt) * 32, min(K, (ue - bt * tpt) * 32),
                        c - owner(bt * tpt), ue == (bt + 1) * tpt))
            u = ue
    return out


@pytest.mark.parametrize("B,T,K,grid,S", [(64, 1, 2048, 296, 6), (60, 1, 2048, 148, 4),
                                          (7, 3, 1000, 148, 9), (128, 1, 2048, 296, 4),
                                          (5, 1, 33, 2, 2)])
def test_balanced_schedule_covers_every_row_once(B, T, K, grid, S):
    items = balanced_items(B, T, K, grid)
    rows = {}
    for c, bt, j0, j1, slot, last in items:
        assert 0 <= slot < S and j0 < j1
        for j in range(j0, j1):
            assert (bt, j) not in rows
            rows[(bt, j)] = slot
    assert len(rows) == B * T * K
    # per token: slots 0..n-1 in row order, exactly one piece marked last
    for bt in range(B * T):
        pieces = sorted((j0, slot, last) for c, b, j0, j1, slot, last in items if b == bt)
        assert [sl for _, sl, _ in pieces] == list(range(len(pieces)))
        assert [la for _, _, la in pieces] == [False] * (len(pieces) - 1) + [True]
    # every CTA has the same number of tiles, +-1
    per_cta = {}
    for c, bt, j0, j1, slot, last in items:
        per_cta[c] = per_cta.get(c, 0) + -(-(j1 - j0) // 32)
    assert max(per_cta.values()) - min(per_cta.values()) <= 1 + (K % 32 != 0)


def test_binding_refuses_cpu_tensors():
    import torch
    q = torch.zeros((1, 1, 16, 576), dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        binding.decode(q, torch.zeros((1, 64, 576), dtype=torch.bfloat16),
                       torch.zeros((1, 1), dtype=torch.int32), torch.zeros((1, 1, 4), dtype=torch.int32),
                       0.1, 1)


def test_workspace_host_bytes_formula(lib):
    r = lambda x: (x + 255) // 256 * 256
    for B, T, H, K, P, S in [(1, 1, 16, 2048, 1024, 64), (64, 1, 16, 2048, 256, 4), (2, 3, 5, 7, 9, 1)]:
        base = binding.workspace_bytes(B, T, H, S) if S > 1 else 0
        want = r(base) + r(B * T * H * 576 * 2) + r(B * T * K * 4) + r(B * P * 4)
        assert binding.workspace_host_bytes(B, T, H, K, P, S) == want
    assert binding.workspace_host_bytes(1, 1, 1, 1, 1, 0) == 0
    assert binding.workspace_host_bytes(1, 1, 1, -1, 1, 1) == 0


# ------------------------------------------------------------------ binding buffer checks
def _cpu_as_device(monkeypatch):
    """Let CPU tensors through the binding's device test, so that its shape
    checks (which run before any library call) can be exercised here."""
    monkeypatch.setattr(binding, "_on_device", lambda t, name, device: None)


def test_need_checks_shape_before_device():
    import torch
    with pytest.raises(ValueError, match="out must have shape"):
        binding._need(torch.zeros((2, 3), dtype=torch.int32), torch.int32, "out", shape=(2, 4))
    with pytest.raises(ValueError, match="CUDA tensor"):
        binding._need(torch.zeros((2, 4), dtype=torch.int32), torch.int32, "out", shape=(2, 4))


def _decode_inputs(B=2, T=3, H=16, K=40, P=2):
    import torch
    return (torch.zeros((B, T, H, 576), dtype=torch.bfloat16), torch.zeros((P, 64, 576), dtype=torch.bfloat16),
            torch.zeros((B, 1), dtype=torch.int32), torch.zeros((B, T, K), dtype=torch.int32))


def test_binding_rejects_wrong_output_shapes(lib, monkeypatch):
    """Every caller-supplied buffer the library writes through must have the
    shape the call implies; a wrong one is refused before anything runs."""
    import torch
    _cpu_as_device(monkeypatch)
    q, cache, pt, idx = _decode_inputs()
    bf, f32 = torch.bfloat16, torch.float32
    o_ok, lse_ok = torch.zeros((2, 3, 16, 512), dtype=bf), torch.zeros((2, 3, 16), dtype=f32)
    o_bad, lse_bad = torch.zeros((2, 3, 8, 512), dtype=bf), torch.zeros((2, 3, 17), dtype=f32)
    calls = [
        ("o", lambda: binding.decode(q, cache, pt, idx, 0.1, 2, o=o_bad, lse=lse_ok)),
        ("lse", lambda: binding.decode(q, cache, pt, idx, 0.1, 2, o=o_ok, lse=lse_bad)),
        ("o", lambda: binding.decode_noalloc(q, cache, pt, idx, 0.1, 2, o=o_bad, lse=lse_ok)),
        ("part_o", lambda: binding.decode_partial(q, cache, pt, idx, 0.1, 3,
                                                  part_o=torch.zeros((2, 3, 16, 2, 512), dtype=f32))),
        ("part_m", lambda: binding.decode_partial(q, cache, pt, idx, 0.1, 3,
                                                  part_m=torch.zeros((2, 3, 16, 4), dtype=f32))),
        ("o", lambda: binding.lse_combine(torch.zeros((2, 3, 16, 4, 512), dtype=f32),
                                          torch.zeros((2, 3, 16, 4), dtype=f32),
                                          torch.zeros((2, 3, 16, 4), dtype=f32), o=o_bad)),
    ]
    seq_lens = torch.full((2, 3), 30, dtype=torch.int32)
    calls += [
        ("lse", lambda: binding.decode_dense(q, cache, pt, seq_lens, 0.1, 2, K=40, o=o_ok,
                                             lse=lse_bad)),
        ("part_lse", lambda: binding.decode_dense_partial(
            q, cache, pt, seq_lens, 0.1, 2, K=40, part_lse=torch.zeros((2, 3, 16, 3), dtype=f32))),
    ]
    qi = torch.zeros((2, 3, 4, 128), dtype=bf)
    wi, ki, nv = torch.zeros((2, 3, 4), dtype=f32), torch.zeros((2, 64, 128), dtype=bf), \
        torch.zeros((2, 3), dtype=torch.int32)
    calls += [
        ("out", lambda: binding.indexer_topk(qi, wi, ki, pt, nv, 16, 100,
                                             out=torch.zeros((2, 3, 8), dtype=torch.int32))),
        ("scores", lambda: binding.indexer_scores(qi, wi, ki, pt, nv, 100,
                                                  scores=torch.zeros((2, 3, 64), dtype=f32))),
        ("n_vis", lambda: binding.indexer_select(torch.zeros((2, 3, 100), dtype=f32),
                                                 torch.zeros((6,), dtype=torch.int32), 16)),
        ("out", lambda: binding.indexer_select(torch.zeros((2, 3, 100), dtype=f32), nv, 16,
                                               out=torch.zeros((2, 3, 17), dtype=torch.int32))),
    ]
    for name, call in calls:
        with pytest.raises(ValueError, match=f"^{name} must have shape"):
            call()
    with pytest.raises(ValueError, match="scores must be"):
        binding.indexer_select(torch.zeros((6, 100), dtype=f32), nv, 16)


def test_binding_enforces_the_k_limit(lib, monkeypatch):
    """K above the library's 32-bit split arithmetic is refused by the
    binding; at the limit the host heuristics stay in range."""
    import torch
    _cpu_as_device(monkeypatch)
    monkeypatch.delenv("SMLA_NSPLIT", raising=False)
    big = binding.MAX_K + 1
    for call in (lambda: binding.choose_nsplit(1, 1, 16, big, 148),
                 lambda: binding.dense_nsplit(1, 1, 8, big),
                 lambda: binding.indexer_select(torch.zeros((1, 1, 8), dtype=torch.float32),
                                                torch.zeros((1, 1), dtype=torch.int32), big)):
        with pytest.raises(ValueError, match="above the library's limit"):
            call()
    assert 1 <= binding.choose_nsplit(1, 1, 16, binding.MAX_K, 148) <= 1024
    assert 1 <= binding.dense_nsplit(1, 1, 8, binding.MAX_K) <= 1024
    ws = binding.dense_workspace_bytes(1, 1, 8, binding.MAX_K, 1)
    assert ws == 0


# ------------------------------------------------------------------ indexer entry points
def call_topk(lib, q=FAKE, w=FAKE, k=FAKE, num_pages=10, pt=FAKE, pt_stride=4, nv=FAKE, B=2, T=1,
              HI=64, max_n=256, K=64, ps=64, ws=FAKE, ws_bytes=1 << 30, out=FAKE):
    return lib.smla_indexer_topk(q, w, k, num_pages, pt, pt_stride, nv, B, T, HI, max_n, K, ps,
                                 ws, ws_bytes, out, None)


def call_scores(lib, q=FAKE, w=FAKE, k=FAKE, num_pages=10, pt=FAKE, pt_stride=4, nv=FAKE, B=2,
                T=1, HI=64, max_n=256, ps=64, ws=FAKE, ws_bytes=1 << 30, scores=FAKE):
    return lib.smla_indexer_scores(q, w, k, num_pages, pt, pt_stride, nv, B, T, HI, max_n, ps, ws,
                                   ws_bytes, scores, None)


def call_select(lib, scores=FAKE, nv=FAKE, B=2, T=1, max_n=256, K=64, ws=FAKE, ws_bytes=1 << 30,
                out=FAKE):
    return lib.smla_indexer_select(scores, nv, B, T, max_n, K, ws, ws_bytes, out, None)


# shared by the two entry points that score
INDEXER_INPUT_ERRORS = [
    (dict(ps=32), 2), (dict(HI=65), 2), (dict(HI=0), 1), (dict(B=-1), 1), (dict(max_n=-1), 1),
    (dict(max_n=binding.INDEXER_MAX_N + 1), 2), (dict(B=1048577), 2), (dict(q=0), 1),
    (dict(w=0), 1), (dict(nv=0), 1), (dict(q=FAKE + 8), 3), (dict(w=FAKE + 2), 3),
    (dict(nv=FAKE + 2), 3), (dict(k=0), 1), (dict(pt=0), 1), (dict(num_pages=0), 1),
    (dict(pt_stride=0), 1), (dict(num_pages=33554432), 2), (dict(k=FAKE + 8), 3),
    (dict(pt=FAKE + 2), 3), (dict(ws_bytes=100), 4), (dict(ws=0), 1), (dict(ws=FAKE + 8), 3),
]


@pytest.mark.parametrize("kw,expect", INDEXER_INPUT_ERRORS + [
    (dict(K=0), 1), (dict(out=0), 1), (dict(out=FAKE + 2), 3), (dict(B=0), 0), (dict(T=0), 0),
])
def test_indexer_topk_rejects_bad_arguments(lib, kw, expect):
    assert call_topk(lib, **kw) == expect


@pytest.mark.parametrize("kw,expect", INDEXER_INPUT_ERRORS + [
    (dict(scores=0), 1), (dict(scores=FAKE + 2), 3), (dict(B=0), 0), (dict(max_n=0), 0),
])
def test_indexer_scores_rejects_bad_arguments(lib, kw, expect):
    assert call_scores(lib, **kw) == expect


@pytest.mark.parametrize("kw,expect", [
    (dict(K=0), 1), (dict(B=-1), 1), (dict(max_n=-1), 1), (dict(max_n=binding.INDEXER_MAX_N + 1), 2),
    (dict(B=1048577), 2), (dict(nv=0), 1), (dict(out=0), 1), (dict(scores=0), 1),
    (dict(nv=FAKE + 2), 3), (dict(out=FAKE + 2), 3), (dict(scores=FAKE + 2), 3),
    (dict(ws_bytes=100), 4), (dict(ws=0), 1), (dict(ws=FAKE + 8), 3), (dict(B=0), 0),
    (dict(T=0), 0),
])
def test_indexer_select_rejects_bad_arguments(lib, kw, expect):
    assert call_select(lib, **kw) == expect


def test_indexer_workspace_sizes(lib):
    """The top-k workspace is the tile plan, the fp32 score rows and the
    selection scratch, each 256-byte rounded; the scratch holds per token a
    16 KiB digit histogram, a bitmap of max_n positions and max_n candidates
    of (key, position)."""
    r = lambda x: (x + 255) // 256 * 256
    for B, T, n in [(60, 1, 123434), (1, 9, 46089), (3, 2, 1), (512, 8, 700), (1, 1, 0)]:
        sel = binding.indexer_select_workspace_bytes(B, T, n)
        assert sel >= B * T * (16384 + -(-n // 32) * 4 + n * 8)
        assert sel == r(sel)
        assert binding.indexer_workspace_bytes(B, T, n) == r((B * T + 1) * 4) + r(B * T * n * 4) + sel
    assert binding.indexer_workspace_bytes(-1, 1, 1) == 0
    assert binding.indexer_select_workspace_bytes(1, 1, -1) == 0
    # the scores entry point needs only the plan
    assert binding.indexer_workspace_bytes(4, 2, 0) >= r(9 * 4)


# ------------------------------------------------------------------ the other decode entry points
def call_noalloc(lib, q=FAKE, cache=FAKE, num_pages=10, pt=FAKE, pt_stride=4, idx=FAKE, B=1, T=1,
                 H=16, K=64, ps=64, scale=0.1, nsplit=2, o=FAKE, lse=FAKE):
    return lib.smla_decode_noalloc(q, cache, num_pages, pt, pt_stride, idx, B, T, H, K, ps, scale,
                                   nsplit, o, lse, None)


@pytest.mark.parametrize("kw,expect", [
    (dict(ps=32), 2), (dict(H=65), 2), (dict(B=-1), 1), (dict(q=0), 1), (dict(q=FAKE + 8), 3),
    (dict(scale=math.nan), 1), (dict(nsplit=-1), 1), (dict(nsplit=1025), 1), (dict(B=0), 0),
])
def test_noalloc_rejects_bad_arguments(lib, kw, expect):
    assert call_noalloc(lib, **kw) == expect


def test_noalloc_refuses_partials_beyond_its_scratch_on_the_host(lib):
    """64 tokens x 64 heads x 8 splits of partials need about 67 MB: refused
    with a message before the scratch array is even looked up."""
    assert binding.workspace_bytes(64, 1, 64, 8) > binding.NOALLOC_SCRATCH_BYTES
    assert call_noalloc(lib, B=64, H=64, K=256, nsplit=8) == 4
    assert b"scratch" in lib.smla_last_error()


def call_host(lib, q=FAKE, cache=FAKE, num_pages=10, pt=FAKE, pt_stride=4, idx=FAKE, B=1, T=1,
              H=16, K=64, ps=64, scale=0.1, nsplit=2, ws=FAKE, ws_bytes=1 << 30, o=FAKE, lse=FAKE):
    return lib.smla_decode_host(q, cache, num_pages, pt, pt_stride, idx, B, T, H, K, ps, scale,
                                nsplit, ws, ws_bytes, o, lse, None)


@pytest.mark.parametrize("kw,expect", [
    (dict(ps=32), 2), (dict(H=65), 2), (dict(B=-1), 1), (dict(q=0), 1), (dict(cache=FAKE + 4), 3),
    (dict(scale=math.inf), 1), (dict(nsplit=-1), 1), (dict(nsplit=1025), 1), (dict(o=0), 1),
    (dict(lse=0), 1), (dict(num_pages=0), 1), (dict(B=0), 0),
])
def test_decode_host_rejects_bad_arguments_before_any_launch(lib, kw, expect):
    assert call_host(lib, **kw) == expect


def test_nsplit_of_every_bench_workload(lib, monkeypatch):
    """The split counts the heuristic gives the benchmark's shapes on a
    148-SM B200 (the values the results tables are measured at)."""
    monkeypatch.delenv("SMLA_NSPLIT", raising=False)
    assert binding.choose_nsplit(1, 1, 16, 2048, 148) == 64      # single_request
    assert binding.choose_nsplit(1, 9, 8, 2048, 148) == 32       # spec_verify
    assert binding.choose_nsplit(64, 1, 16, 2048, 148) == 4      # batched
    assert binding.choose_nsplit(60, 1, 64, 2048, 148) == 2      # mixed
    assert binding.dense_nsplit(1, 9, 8, 46089) == 74            # dense_verify (148 CTAs)
