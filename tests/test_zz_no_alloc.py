"""GPU test of smla_decode_noalloc, the entry point for callers that cannot
allocate device memory while they decode (it takes no workspace; the split-K
partials go to a scratch array the library keeps on each device).

Each case calls the allocation-free entry point twice in a row and the
ordinary smla_decode (with a workspace it is given) on the same inputs at the
same split count.  Both run the same kernels in the same schedule, so the
outputs must be bit-identical; a stale value left in the shared scratch by an
earlier call would show up as a difference.  One case is also compared with
the fp64 oracle, and the free device memory must not change across the calls
after the first.  The file is named so that pytest collects it last; it also
passes on its own in a fresh process.
"""
import pytest
import torch

from parity_util import check_o_lse, oracle_decode
from sparse_mla_decode_partial_b200 import binding, build, workloads

pytestmark = pytest.mark.gpu

DEV = torch.device("cuda:0")


@pytest.fixture(scope="module", autouse=True)
def _lib():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    build.build()
    binding.lib()


def noalloc_nsplit(B, T, H, K):
    """The split count smla_decode_noalloc uses for nsplit = 0: the
    heuristic's, lowered until its partials fit the scratch array."""
    S = binding.choose_nsplit(B, T, H, K, 0)
    while S > 1 and binding.workspace_bytes(B, T, H, S) > binding.NOALLOC_SCRATCH_BYTES:
        S -= 1
    return S


CASES = [
    # (name, builder kwargs, nsplit)
    ("one token, 16 heads, S=16", dict(B=1, T=1, H=16, K=2048, ctx=65536), 16),
    ("batch 8, 16 heads, heuristic S", dict(B=8, T=1, H=16, K=2048, ctx=16384), 0),
    ("verify shape, 8 heads, S=32", dict(B=1, T=9, H=8, K=2048, ctx=46089, causal=True), 32),
    ("batch 4, 64 heads, S=4", dict(B=4, T=1, H=64, K=2048, ctx=8000), 4),
    # the heuristic's S (9) needs 18 MiB of partials: nsplit = 0 lowers it
    ("batch 16, 64 heads, heuristic S lowered", dict(B=16, T=1, H=64, K=2048, ctx=3000), 0),
]


@pytest.mark.parametrize("name,kw,nsplit", CASES, ids=[c[0] for c in CASES])
def test_noalloc_matches_decode_twice(name, kw, nsplit):
    kw = dict(kw)
    ctx = kw.pop("ctx")
    w = workloads.make_workload("noalloc", ctx_lens=[ctx] * kw["B"], seed=21, **kw).to(DEV)
    S = nsplit or noalloc_nsplit(w.B, w.T, w.H, w.K)
    assert binding.workspace_bytes(w.B, w.T, w.H, S) <= binding.NOALLOC_SCRATCH_BYTES
    if name.endswith("lowered"):
        assert S < binding.choose_nsplit(w.B, w.T, w.H, w.K, 0)
    ref_o, ref_lse = binding.decode(w.q, w.cache, w.page_table, w.idx, w.scale, S)
    torch.cuda.synchronize()
    for call in range(2):  # two calls in a row share (and reuse) the library's scratch
        o = torch.full_like(ref_o, 9.0)
        lse = torch.full_like(ref_lse, 9.0)
        binding.decode_noalloc(w.q, w.cache, w.page_table, w.idx, w.scale, nsplit, o=o, lse=lse)
        torch.cuda.synchronize()
        assert torch.equal(o, ref_o), f"{name}: o differs from smla_decode on call {call + 1}"
        assert torch.equal(lse, ref_lse), f"{name}: lse differs from smla_decode on call {call + 1}"


def test_noalloc_against_oracle_and_free_memory_steady():
    w = workloads.make_workload("noalloc_oracle", B=3, T=2, H=64, K=1500, ctx_lens=[5000] * 3,
                                seed=23)
    w.idx[1, 0, 700:] = -1                       # padding, and a short split
    wd = w.to(DEV)
    o = torch.empty((3, 2, 64, 512), dtype=torch.bfloat16, device=DEV)
    lse = torch.empty((3, 2, 64), dtype=torch.float32, device=DEV)
    binding.decode_noalloc(wd.q, wd.cache, wd.page_table, wd.idx, w.scale, 3, o=o, lse=lse)
    torch.cuda.synchronize()
    o_ref, lse_ref, _ = oracle_decode(w)
    check_o_lse(o, lse, o_ref, lse_ref, "noalloc vs oracle")
    # after the first call on the device, further calls reserve nothing
    free0 = torch.cuda.mem_get_info(DEV)[0]
    for _ in range(3):
        binding.decode_noalloc(wd.q, wd.cache, wd.page_table, wd.idx, w.scale, 3, o=o, lse=lse)
        torch.cuda.synchronize()
        assert torch.cuda.mem_get_info(DEV)[0] == free0
    check_o_lse(o, lse, o_ref, lse_ref, "noalloc vs oracle, fourth call")


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
