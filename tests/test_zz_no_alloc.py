"""GPU test of smla_decode_noalloc, the entry point for callers that cannot
allocate device memory while they decode (it takes no workspace; the split-K
partials go to a scratch array the library keeps on each device).

Each case calls the allocation-free entry point twice in a row and the
ordinary smla_decode (with a workspace it is given) on the same inputs, and
requires the outputs to agree within the tolerances the parity tests use.  The
file is named so that pytest collects it last; it also passes on its own in a
fresh process.
"""
import numpy as np
import pytest
import torch

from parity_util import LSE_MAX_ABS, O_MAX_ABS, O_REL_L2
from sparse_mla_decode_partial_b200 import binding, build, workloads

pytestmark = pytest.mark.gpu

DEV = torch.device("cuda:0")


@pytest.fixture(scope="module", autouse=True)
def _lib():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    build.build()
    binding.lib()


def agree(o_a, lse_a, o_b, lse_b, what):
    a = o_a.float().cpu().numpy().astype(np.float64)
    b = o_b.float().cpu().numpy().astype(np.float64)
    assert np.all(np.isfinite(a)), f"{what}: non-finite o"
    err = np.abs(a - b).max()
    denom = np.linalg.norm(b)
    rel = np.linalg.norm(a - b) / denom if denom > 0 else np.linalg.norm(a)
    la, lb = lse_a.cpu().numpy(), lse_b.cpu().numpy()
    assert np.array_equal(np.isneginf(la), np.isneginf(lb)), f"{what}: -inf pattern"
    fin = ~np.isneginf(lb)
    lerr = np.abs(la[fin] - lb[fin]).max() if fin.any() else 0.0
    assert err <= O_MAX_ABS and rel <= O_REL_L2 and lerr <= LSE_MAX_ABS, (what, err, rel, lerr)


CASES = [
    # (name, builder kwargs, nsplit)
    ("one token, 16 heads, S=16", dict(B=1, T=1, H=16, K=2048, ctx=65536), 16),
    ("batch 8, 16 heads, heuristic S", dict(B=8, T=1, H=16, K=2048, ctx=16384), 0),
    ("verify shape, 8 heads, S=32", dict(B=1, T=9, H=8, K=2048, ctx=46089, causal=True), 32),
    ("batch 4, 64 heads, S=4", dict(B=4, T=1, H=64, K=2048, ctx=8000), 4),
]


@pytest.mark.parametrize("name,kw,nsplit", CASES, ids=[c[0] for c in CASES])
def test_noalloc_matches_decode_twice(name, kw, nsplit):
    kw = dict(kw)
    ctx = kw.pop("ctx")
    w = workloads.make_workload("noalloc", ctx_lens=[ctx] * kw["B"], seed=21, **kw).to(DEV)
    ref_o, ref_lse = binding.decode(w.q, w.cache, w.page_table, w.idx, w.scale, nsplit)
    torch.cuda.synchronize()
    outs = []
    for _ in range(2):  # two calls in a row share (and reuse) the library's scratch
        o = torch.empty_like(ref_o)
        lse = torch.empty_like(ref_lse)
        binding.decode_noalloc(w.q, w.cache, w.page_table, w.idx, w.scale, nsplit, o=o, lse=lse)
        torch.cuda.synchronize()
        outs.append((o, lse))
    for i, (o, lse) in enumerate(outs):
        agree(o, lse, ref_o, ref_lse, f"{name}: call {i + 1}")


def test_noalloc_rejects_work_beyond_its_scratch():
    # 64 tokens x 64 heads x 8 splits of partials need ~67 MB > the 16 MiB scratch
    w = workloads.make_workload("big", B=64, T=1, H=64, K=256, ctx_lens=[300] * 64,
                                seed=3).to(DEV)
    assert binding.workspace_bytes(64, 1, 64, 8) > binding.NOALLOC_SCRATCH_BYTES
    o = torch.full((64, 1, 64, 512), 3.0, dtype=torch.bfloat16, device=DEV)
    lse = torch.full((64, 1, 64), 3.0, dtype=torch.float32, device=DEV)
    with pytest.raises(binding.SmlaError) as exc:
        binding.decode_noalloc(w.q, w.cache, w.page_table, w.idx, w.scale, 8, o=o, lse=lse)
    assert exc.value.status == 4
    assert "scratch" in binding.lib().smla_last_error().decode()
    torch.cuda.synchronize()
    assert torch.all(o == 3.0) and torch.all(lse == 3.0)   # nothing was launched
