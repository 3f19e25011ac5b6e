"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle.

Every case feeds the same seeded inputs to both sides.  Tolerances are the
problem statement's: o max-abs <= 1e-2 and relative L2 <= 5e-3, lse <= 1e-3
(see parity_util), plus the relative-L2 bound on every output row.  Small
cases and the full-size batched and mixed-length workloads, the latter run in
the launch configuration the benchmark times (heuristic NSPLIT), compare every
output; a few many-token schedule tests compare sampled query tokens.
"""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
from parity_util import (bits, check_o_lse, normalised_partials, oracle_decode, sample_bt)
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
    st, n = binding.check_device(clear=True)
    assert st in (0, 5), binding.status_string(st)


def run_decode(w, nsplit, **kw):
    wd = w.to(DEV)
    o, lse = binding.decode(wd.q, wd.cache, wd.page_table, wd.idx, w.scale, nsplit, **kw)
    torch.cuda.synchronize()
    return o, lse


def small(name="s", seed=5, B=2, T=2, H=16, K=300, ctx=2000, **kw):
    return workloads.make_workload(name, B=B, T=T, H=H, K=K, ctx_lens=[ctx] * B, seed=seed, **kw)


# ------------------------------------------------------------------ the five configurations
@pytest.mark.parametrize("nsplit", [4, 1, 0])
def test_tiny(nsplit):
    w = workloads.tiny()
    o, lse = run_decode(w, nsplit)
    o_ref, lse_ref, _ = oracle_decode(w)
    check_o_lse(o, lse, o_ref, lse_ref, f"tiny S={nsplit}")


@pytest.fixture(scope="module")
def single_request():
    return workloads.single_request()


@pytest.mark.parametrize("nsplit", [1, 4, 16, 32, 64, 0])
def test_single_request_nsplit_sweep(single_request, nsplit):
    w = single_request
    o, lse = run_decode(w, nsplit)
    o_ref, lse_ref, _ = oracle_decode(w)
    check_o_lse(o, lse, o_ref, lse_ref, f"single_request S={nsplit}")


@pytest.mark.parametrize("nsplit", [16, 64, 0])
def test_spec_verify(nsplit):
    w = workloads.spec_verify()
    o, lse = run_decode(w, nsplit)
    o_ref, lse_ref, _ = oracle_decode(w)
    check_o_lse(o, lse, o_ref, lse_ref, f"spec_verify S={nsplit}")


def test_batched_full_size_every_token():
    """B64 H16 K2048 at the heuristic NSPLIT (the launch the benchmark times):
    every query token, head and output element against the oracle."""
    w = workloads.batched()
    o, lse = run_decode(w, 0)
    o_ref, lse_ref, bad = oracle_decode(w)
    assert bad == 0
    check_o_lse(o, lse, o_ref, lse_ref, "batched, every token")


def test_mixed_full_size_every_token():
    """B60 H64 K2048, contexts 1K..128K with -1 tails, at the heuristic NSPLIT
    (the launch the benchmark times): every output against the oracle."""
    w = workloads.mixed()
    assert any(c < 2048 for c in w.ctx_lens), "the draw has no padded token"
    o, lse = run_decode(w, 0)
    o_ref, lse_ref, bad = oracle_decode(w)
    assert bad == 0
    check_o_lse(o, lse, o_ref, lse_ref, "mixed, every token")


def test_batched_reduced_full_compare():
    w = workloads.batched(B=6)
    for nsplit in (0, 2, 8):
        o, lse = run_decode(w, nsplit)
        o_ref, lse_ref, _ = oracle_decode(w)
        check_o_lse(o, lse, o_ref, lse_ref, f"batched B=6 S={nsplit}")


def test_mixed_reduced_full_compare():
    w = workloads.mixed(B=5)
    for nsplit in (0, 3, 8):
        o, lse = run_decode(w, nsplit)
        o_ref, lse_ref, _ = oracle_decode(w)
        check_o_lse(o, lse, o_ref, lse_ref, f"mixed B=5 S={nsplit}")


# ------------------------------------------------------------------ the two passes separately
@pytest.mark.parametrize("H", [8, 16, 64])
def test_partial_pass_against_oracle_partials(H):
    w = small(H=H, K=200, B=1, T=2)
    w.idx[0, 1, 64:128] = -1          # one whole split (Kc = 50) of padding and more
    nsplit = 4
    wd = w.to(DEV)
    po, pm, pl = binding.decode_partial(wd.q, wd.cache, wd.page_table, wd.idx, w.scale, nsplit)
    torch.cuda.synchronize()
    rpo, rpm, rpl, _ = oracle.partial(bits(w.q), bits(w.cache), w.page_table.numpy(),
                                      w.idx.numpy(), w.scale, nsplit)
    got = normalised_partials(po.cpu().numpy(), pm.cpu().numpy(), pl.cpu().numpy())
    ref = normalised_partials(rpo, rpm, rpl)
    assert np.abs(got - ref).max() <= 1e-2
    assert np.linalg.norm(got - ref) / np.linalg.norm(ref) <= 5e-3
    plg = pl.cpu().numpy()
    assert np.array_equal(np.isneginf(plg), np.isneginf(rpl))
    fin = ~np.isneginf(rpl)
    assert np.abs(plg[fin] - rpl[fin]).max() <= 1e-3


@pytest.mark.parametrize("nsplit", [2, 5, 8, 16, 70])
def test_combine_pass_against_oracle_combine(nsplit):
    w = small(H=16, K=256, B=2, T=1)
    w.idx[1, 0, 100:] = -1
    rpo, rpm, rpl, _ = oracle.partial(bits(w.q), bits(w.cache), w.page_table.numpy(),
                                      w.idx.numpy(), w.scale, nsplit)
    o_ref, lse_ref = oracle.combine(rpo, rpm, rpl)
    t = lambda a: torch.tensor(a, dtype=torch.float32, device=DEV).contiguous()
    o, lse = binding.lse_combine(t(rpo), t(rpm), t(rpl))
    torch.cuda.synchronize()
    check_o_lse(o, lse, o_ref, lse_ref, f"combine S={nsplit}")


# ------------------------------------------------------------------ edge cases
@pytest.mark.parametrize("H", [1, 5, 16, 17, 33, 48, 64])
@pytest.mark.parametrize("K", [1, 31, 33, 100])
def test_ragged_heads_and_topk(H, K):
    w = small(H=H, K=K, B=2, T=1, ctx=500, seed=H * 131 + K)
    for nsplit in (1, 3, K + 3):
        o, lse = run_decode(w, nsplit)
        o_ref, lse_ref, _ = oracle_decode(w)
        check_o_lse(o, lse, o_ref, lse_ref, f"H={H} K={K} S={nsplit}")


@pytest.mark.parametrize("pattern", ["trailing", "interleaved", "whole_split", "all", "leading"])
def test_padding_placements(pattern):
    w = small(H=16, K=256, B=2, T=2, seed=9)
    if pattern == "trailing":
        w.idx[:, :, 200:] = -1
    elif pattern == "interleaved":
        w.idx[:, :, ::3] = -1
    elif pattern == "whole_split":
        w.idx[:, :, 64:128] = -1      # S = 4 -> split 1 is entirely padding
    elif pattern == "leading":
        w.idx[:, :, :130] = -1
    else:
        w.idx[0, 1, :] = -1
        w.idx[1, 0, :] = -1
    for nsplit in (1, 4, 7):
        o, lse = run_decode(w, nsplit)
        o_ref, lse_ref, _ = oracle_decode(w)
        check_o_lse(o, lse, o_ref, lse_ref, f"{pattern} S={nsplit}")
    if pattern == "all":
        assert torch.all(o[0, 1] == 0) and torch.all(torch.isneginf(lse[0, 1]))


def test_empty_topk():
    w = small(H=16, K=0, B=2, T=1)
    o, lse = run_decode(w, 1)
    assert torch.all(o == 0) and torch.all(torch.isneginf(lse))


def test_bounded_wait_gives_up_and_context_survives():
    """A wait nothing will end (a barrier no thread arrives at) gives up after
    its limit, raises the timeout status and the kernel returns; the context
    then decodes normally."""
    binding.check_device(clear=True)
    with pytest.raises(binding.SmlaError):
        binding.selftest_wait_timeout(10)                 # below the 1 us floor: refused
    binding.selftest_wait_timeout(5_000_000)              # 5 ms
    st, _ = binding.check_device(clear=False)
    assert st == 7, binding.status_string(st)
    assert binding.check_device(clear=True)[0] == 7
    assert binding.check_device(clear=True)[0] == 0
    w = small(seed=11, B=1, T=1, K=200)
    o, lse = run_decode(w, 4)
    assert binding.check_device(clear=True)[0] == 0
    o_ref, lse_ref, _ = oracle_decode(w)
    check_o_lse(o, lse, o_ref, lse_ref, "after timeout self-test")


def test_out_of_range_entries_masked_and_counted():
    w = small(H=16, K=128, B=1, T=1)
    w.idx[0, 0, 3] = -5
    w.idx[0, 0, 10] = w.pt_stride * 64 + 1
    w.page_table[0, 0] = 10 ** 6                      # every index on logical page 0 goes bad
    n_page0 = int(((w.idx[0, 0] >= 0) & (w.idx[0, 0] < 64)).sum())
    binding.check_device(clear=True)
    o, lse = run_decode(w, 4)
    st, n = binding.check_device(clear=True)
    o_ref, lse_ref, bad = oracle_decode(w)
    check_o_lse(o, lse, o_ref, lse_ref, "out of range")
    assert st == 5, binding.status_string(st)
    assert n == 2 + n_page0 == bad // w.H


def test_deterministic():
    w = workloads.single_request()
    o1, l1 = run_decode(w, 16)
    o2, l2 = run_decode(w, 16)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_output_guards_untouched():
    w = small(H=16, K=300, B=2, T=3)
    wd = w.to(DEV)
    n_o, n_l = w.B * w.T * w.H * 512, w.B * w.T * w.H
    o_buf = torch.full((n_o + 4096,), 7.0, dtype=torch.bfloat16, device=DEV)
    l_buf = torch.full((n_l + 2048,), 7.0, dtype=torch.float32, device=DEV)
    o = o_buf[2048:2048 + n_o].view(w.B, w.T, w.H, 512)
    lse = l_buf[1024:1024 + n_l].view(w.B, w.T, w.H)
    for nsplit in (1, 5):
        binding.decode(wd.q, wd.cache, wd.page_table, wd.idx, w.scale, nsplit, o=o, lse=lse)
        torch.cuda.synchronize()
        assert torch.all(o_buf[:2048] == 7) and torch.all(o_buf[2048 + n_o:] == 7)
        assert torch.all(l_buf[:1024] == 7) and torch.all(l_buf[1024 + n_l:] == 7)
    o_ref, lse_ref, _ = oracle_decode(w)
    check_o_lse(o, lse, o_ref, lse_ref, "guarded")


def test_side_stream_and_reused_workspace():
    w = small(H=16, K=512, B=3, T=1)
    wd = w.to(DEV)
    s = torch.cuda.Stream()
    ws = torch.empty(binding.workspace_bytes(3, 1, 16, 8), dtype=torch.uint8, device=DEV)
    with torch.cuda.stream(s):
        o, lse = binding.decode(wd.q, wd.cache, wd.page_table, wd.idx, w.scale, 8, workspace=ws,
                                stream=s)
    s.synchronize()
    o_ref, lse_ref, _ = oracle_decode(w)
    check_o_lse(o, lse, o_ref, lse_ref, "side stream")


def test_device_error_paths():
    w = small(H=16, K=64, B=1, T=1).to(DEV)
    lib = binding.lib()
    o = torch.empty((1, 1, 16, 512), dtype=torch.bfloat16, device=DEV)
    lse = torch.empty((1, 1, 16), dtype=torch.float32, device=DEV)
    qbytes = torch.empty(w.q.numel() * 2 + 64, dtype=torch.uint8, device=DEV)
    mis = qbytes.data_ptr() + 2                      # 2-byte aligned, not 16
    st = lib.smla_decode(mis, w.cache.data_ptr(), w.num_pages, w.page_table.data_ptr(),
                         w.pt_stride, w.idx.data_ptr(), 1, 1, 16, 64, 64, w.scale, 1, None, 0,
                         o.data_ptr(), lse.data_ptr(), None)
    assert st == 3
    st = lib.smla_decode(w.q.data_ptr(), w.cache.data_ptr(), w.num_pages, w.page_table.data_ptr(),
                         w.pt_stride, w.idx.data_ptr(), 1, 1, 16, 64, 64, w.scale, 4, None, 100,
                         o.data_ptr(), lse.data_ptr(), None)
    assert st == 4


# ------------------------------------------------------------------ one-tile splits
# When every split holds at most 32 entries (H <= 32) the partial pass runs the
# latency form of the kernel (one CTA per split, every load in flight at once).
# Whatever a reused workspace held before must not change the result.
@pytest.mark.parametrize("fill", [0x00, 0xFF, 0x5A])
def test_one_tile_splits_arbitrary_workspace_contents(fill):
    w = small("one_tile", seed=11, B=1, T=2, H=16, K=1024, ctx=30000)
    wd = w.to(DEV)
    S = 32                                                # 32 rows per split
    ws = torch.full((binding.workspace_bytes(1, 2, 16, S),), fill, dtype=torch.uint8, device=DEV)
    o_ref, lse_ref, _ = oracle_decode(w)
    for call in range(3):                                 # partials left by the previous call
        o, lse = binding.decode(wd.q, wd.cache, wd.page_table, wd.idx, w.scale, S, workspace=ws)
        torch.cuda.synchronize()
        check_o_lse(o, lse, o_ref, lse_ref, f"fill={fill:#x} call {call}")
    assert binding.check_device(clear=False)[0] == 0


@pytest.mark.parametrize("H,K,S", [(16, 33, 32), (32, 64, 2), (8, 1, 4), (17, 640, 20),
                                   (32, 2048, 64), (1, 100, 7)])
def test_one_tile_split_shapes(H, K, S):
    # empty splits (K=33, S=32 -> 17 one-or-two-row splits and 15 empty ones),
    # both head groups (H <= 16, H <= 32), one row in all, odd S
    w = small("one_tile_shapes", seed=H * 100 + K, B=2, T=1, H=H, K=K, ctx=4000)
    o, lse = run_decode(w, S)
    o_ref, lse_ref, _ = oracle_decode(w)
    check_o_lse(o, lse, o_ref, lse_ref, f"one-tile H={H} K={K} S={S}")


def test_one_tile_splits_many_waves():
    # 64 tokens x 64 splits = 4096 blocks: many waves of the latency form
    w = small("one_tile_big", seed=12, B=64, T=1, H=16, K=2048, ctx=8000)
    o, lse = run_decode(w, 64)
    sample = [(0, 0), (17, 0), (63, 0)]
    o_ref, lse_ref, _ = oracle_decode(w, sample)
    idx = torch.tensor([b for b, _ in sample])
    check_o_lse(o[idx, 0], lse[idx, 0], o_ref, lse_ref, "many waves")


# ------------------------------------------------------------------ balanced schedule
# The whole decode may cover a token's top-k axis with up to nsplit pieces of
# unequal length, one full wave of CTAs with equal work each.  These shapes
# take that path on a 148-SM B200 (checked below with the library's rule).
def balanced_taken(B, T, H, K, S, sms):
    resident = sms * (2 if H <= 16 else 1)
    bt, units = B * T, B * T * -(-K // 32)
    latency = H <= 32 and -(-K // S) <= 64
    return (S >= 2 and H <= 32 and not latency and bt * S > resident
            and (S - 1) * bt >= resident and units >= 4 * resident)


def sms():
    return torch.cuda.get_device_properties(0).multi_processor_count


@pytest.mark.parametrize("B,T,H,K,S", [(64, 1, 16, 2048, 6), (64, 1, 16, 2048, 24),
                                       (40, 1, 24, 1000, 8), (20, 3, 16, 777, 8),
                                       (128, 1, 16, 2048, 4)])
def test_balanced_schedule(B, T, H, K, S):
    w = workloads.make_workload("balanced", B=B, T=T, H=H, K=K, ctx_lens=[6000] * B, seed=B + K)
    S_used = S or binding.choose_nsplit(B, T, H, K, 0)
    assert balanced_taken(B, T, H, K, S_used, sms()), "shape does not exercise the balanced path"
    o, lse = run_decode(w, S)
    sample = sample_bt(w, 6, seed=K)
    o_ref, lse_ref, _ = oracle_decode(w, sample)
    bi = [b for b, _ in sample]
    ti = [t for _, t in sample]
    check_o_lse(o[bi, ti], lse[bi, ti], o_ref, lse_ref, f"balanced B={B} T={T} H={H} K={K} S={S}")
    assert torch.isfinite(o.float()).all() and torch.isfinite(lse).all()


@pytest.mark.parametrize("B,T,H,K,S", [(60, 1, 64, 2048, 4), (64, 1, 16, 2048, 6), (3, 2, 16, 500, 5)])
def test_partial_ws_then_combine_is_the_decode(B, T, H, K, S):
    """smla_decode_partial_ws followed by smla_lse_combine on the workspace
    runs the decode's own kernels in its own schedule: bit-identical o, lse."""
    w = workloads.make_workload("split_decode", B=B, T=T, H=H, K=K, ctx_lens=[3000] * B, seed=B + S)
    wd = w.to(DEV)
    ws = torch.empty(binding.workspace_bytes(B, T, H, S), dtype=torch.uint8, device=DEV)
    o_ref, lse_ref = binding.decode(wd.q, wd.cache, wd.page_table, wd.idx, w.scale, S, workspace=ws)
    ws.fill_(0xFF)
    lib = binding.lib()
    st = lib.smla_decode_partial_ws(wd.q.data_ptr(), wd.cache.data_ptr(), w.num_pages,
                                    wd.page_table.data_ptr(), w.pt_stride, wd.idx.data_ptr(), B, T,
                                    H, K, 64, w.scale, S, ws.data_ptr(), ws.numel(), None)
    assert st == 0
    n = B * T * H * S
    r256 = lambda x: (x + 255) // 256 * 256
    po = ws[:n * 2048].view(torch.float32).view(B, T, H, S, 512)
    pm = ws[r256(n * 2048):r256(n * 2048) + n * 4].view(torch.float32).view(B, T, H, S)
    off = r256(n * 2048) + r256(n * 4)
    pl = ws[off:off + n * 4].view(torch.float32).view(B, T, H, S)
    o, lse = binding.lse_combine(po, pm, pl)
    torch.cuda.synchronize()
    assert torch.equal(o, o_ref) and torch.equal(lse, lse_ref)


def test_balanced_schedule_ignores_stale_workspace():
    # slots no CTA writes keep whatever the workspace held: NaN bit patterns
    # (0xFF bytes) there must not reach o
    B, T, H, K, S = 64, 1, 16, 2048, 9
    w = workloads.make_workload("balanced_nan", B=B, T=T, H=H, K=K, ctx_lens=[5000] * B, seed=77)
    assert balanced_taken(B, T, H, K, S, sms())
    wd = w.to(DEV)
    ws = torch.full((binding.workspace_bytes(B, T, H, S),), 0xFF, dtype=torch.uint8, device=DEV)
    o, lse = binding.decode(wd.q, wd.cache, wd.page_table, wd.idx, w.scale, S, workspace=ws)
    torch.cuda.synchronize()
    assert torch.isfinite(o.float()).all() and torch.isfinite(lse).all()
    sample = [(0, 0), (31, 0), (63, 0)]
    o_ref, lse_ref, _ = oracle_decode(w, sample)
    bi = [b for b, _ in sample]
    check_o_lse(o[bi, 0], lse[bi, 0], o_ref, lse_ref, "balanced, 0xFF workspace")


def test_balanced_schedule_with_padding_and_short_contexts():
    # tokens whose whole top-k is padding, or mostly padding, spread over pieces
    B, H, K, S = 48, 16, 2048, 8
    ctx = [100 if b % 5 == 0 else (1500 if b % 5 == 1 else 9000) for b in range(B)]
    w = workloads.make_workload("balanced_pad", B=B, T=1, H=H, K=K, ctx_lens=ctx, seed=5)
    w.idx[0::7, 0, :] = -1                       # some tokens select nothing at all
    assert balanced_taken(B, 1, H, K, S, sms())
    o, lse = run_decode(w, S)
    sample = [(0, 0), (1, 0), (5, 0), (7, 0), (14, 0), (46, 0), (47, 0)]
    o_ref, lse_ref, _ = oracle_decode(w, sample)
    bi = [b for b, _ in sample]
    check_o_lse(o[bi, 0], lse[bi, 0], o_ref, lse_ref, "balanced with padding")


# ------------------------------------------------------------------ sizes at the edges
@pytest.mark.parametrize("H", [16, 24, 64])
@pytest.mark.parametrize("S", [1, 2])
def test_split_longer_than_one_resolve_chunk(H, S):
    # a split of more than 2048 entries is resolved to rows in several chunks
    w = workloads.make_workload("long_split", B=1, T=1, H=H, K=4500, ctx_lens=[12000], seed=H + S)
    o, lse = run_decode(w, S)
    o_ref, lse_ref, _ = oracle_decode(w)
    check_o_lse(o, lse, o_ref, lse_ref, f"K=4500 H={H} S={S}")


def test_page_table_wider_than_the_latency_kernel_holds():
    # 9000 logical pages (576k positions) over a pool of 96 physical pages
    # (pages aliased): one-tile splits then take the pipelined kernel
    g = torch.Generator().manual_seed(17)
    B, H, K, P, W = 2, 16, 2048, 96, 9000
    q = (torch.randn(B, 1, H, 576, generator=g) * 0.5).to(torch.bfloat16)
    cache = (torch.randn(P, 64, 576, generator=g) * 0.5).to(torch.bfloat16)
    pt = torch.randint(0, P, (B, W), generator=g, dtype=torch.int32)
    idx = torch.stack([torch.randperm(W * 64, generator=g)[:K] for _ in range(B)]).to(torch.int32)
    idx = idx.view(B, 1, K)
    w = workloads.Workload("wide_pt", q, cache, pt, idx, 576 ** -0.5, [W * 64] * B, None, ())
    for S in (64, 16):
        o, lse = run_decode(w, S)
        o_ref, lse_ref, _ = oracle_decode(w)
        check_o_lse(o, lse, o_ref, lse_ref, f"pt_stride {W} S={S}")


@pytest.mark.parametrize("H,W", [(16, 20000), (64, 9000), (64, 60000)])
def test_wide_page_tables_on_the_pipelined_kernels(H, W):
    # Page-table rows of 9000 to 60000 logical pages (up to 3.8M positions)
    # over a pool of 96 physical pages, one logical page mapped past the pool:
    # the mma kernel (H = 16) and the tcgen05 kernel (H = 64) must give the
    # oracle's answer with that page's positions masked and counted.
    g = torch.Generator().manual_seed(W + H)
    B, K, P = 2, 2048, 96
    q = (torch.randn(B, 1, H, 576, generator=g) * 0.5).to(torch.bfloat16)
    cache = (torch.randn(P, 64, 576, generator=g) * 0.5).to(torch.bfloat16)
    pt = torch.randint(0, P, (B, W), generator=g, dtype=torch.int32)
    pt[:, 5] = P + 3  # a page past the pool: its positions are masked and counted
    idx = torch.stack([torch.randperm(W * 64, generator=g)[:K] for _ in range(B)]).to(torch.int32)
    idx[:, 0, ] = 5 * 64 + 7
    idx = idx.view(B, 1, K)
    w = workloads.Workload("pt_row", q, cache, pt, idx, 576 ** -0.5, [W * 64] * B, None, ())
    binding.check_device(clear=True)
    o, lse = run_decode(w, 4)
    st, n = binding.check_device(clear=True)
    o_ref, lse_ref, bad = oracle_decode(w)
    assert st == 5 and n == bad // H and n >= B
    check_o_lse(o, lse, o_ref, lse_ref, f"H={H} pt_stride {W}")


@pytest.mark.parametrize("K,S", [(2048, 1024), (100, 512), (3, 1024)])
def test_maximum_nsplit(K, S):
    # NSPLIT at its maximum: two-entry splits, and mostly empty splits
    w = small("max_nsplit", seed=K, B=1, T=2, H=16, K=K, ctx=5000)
    o, lse = run_decode(w, S)
    o_ref, lse_ref, _ = oracle_decode(w)
    check_o_lse(o, lse, o_ref, lse_ref, f"K={K} S={S}")


@pytest.mark.parametrize("H,K,S", [(16, 2048, 32), (8, 100, 2), (24, 640, 12), (32, 130, 3),
                                   (5, 33, 1), (16, 64, 1), (1, 1000, 16)])
def test_two_tile_splits(H, K, S):
    # 33..64 entries per split: the latency form gathers both tiles at once
    assert 32 < -(-K // S) <= 64
    w = small("two_tiles", seed=H * 7 + K, B=2, T=2, H=H, K=K, ctx=3000)
    w.idx[1, 0, 5::9] = -1                       # interleaved padding in one token
    o, lse = run_decode(w, S)
    o_ref, lse_ref, _ = oracle_decode(w)
    check_o_lse(o, lse, o_ref, lse_ref, f"two tiles H={H} K={K} S={S}")


# ------------------------------------------------------------------ dense-context variant
# ("The Occupancy Hypothesis ...", sections "The Occupancy Insight" and "The
# Broader Context": the verify kernel splits each query token's whole visible
# KV sequence)
def run_dense(w, nsplit, **kw):
    wd = w.to(DEV)
    o, lse = binding.decode_dense(wd.q, wd.cache, wd.page_table, wd.seq_lens, w.scale, nsplit,
                                  K=w.K, **kw)
    torch.cuda.synchronize()
    return o, lse


@pytest.mark.parametrize("H,T,ctx,S", [(8, 9, 3000, 0), (8, 9, 3000, 16), (16, 3, 777, 5),
                                       (64, 2, 1500, 0), (64, 2, 1500, 3), (8, 4, 40, 1),
                                       (16, 2, 100, 64), (24, 5, 2100, 0)])
def test_dense_against_oracle(H, T, ctx, S):
    w = workloads.make_dense_workload("dense", B=2, T=T, H=H, ctx_lens=[ctx, max(T, ctx // 2 + 7)],
                                      seed=H + T + S)
    o, lse = run_dense(w, S)
    o_ref, lse_ref, _ = oracle_decode(w)
    check_o_lse(o, lse, o_ref, lse_ref, f"dense H={H} T={T} ctx={ctx} S={S}")


@pytest.mark.parametrize("H,T,ctx,S", [(8, 9, 3000, 7), (16, 3, 777, 5), (64, 2, 1500, 3),
                                       (24, 5, 2100, 16)])
def test_dense_partial_pass_against_oracle_partials(H, T, ctx, S):
    """Each split's normalised partial and lse against the oracle's partials of
    the equivalent index lists (every visible position, width K)."""
    w = workloads.make_dense_workload("dense_part", B=2, T=T, H=H, ctx_lens=[ctx, ctx // 2 + 40],
                                      seed=3 * H + S)
    wd = w.to(DEV)
    po, pm, pl = binding.decode_dense_partial(wd.q, wd.cache, wd.page_table, wd.seq_lens, w.scale,
                                              S, K=w.K)
    torch.cuda.synchronize()
    lists = oracle.dense_positions(w.seq_lens.numpy(), w.K)
    rpo, rpm, rpl, _ = oracle.partial(bits(w.q), bits(w.cache), w.page_table.numpy(), lists,
                                      w.scale, S)
    got = normalised_partials(po.cpu().numpy(), pm.cpu().numpy(), pl.cpu().numpy())
    want = normalised_partials(rpo, rpm, rpl)
    pl_g = pl.cpu().numpy().astype(np.float64)
    assert np.array_equal(np.isneginf(pl_g), np.isneginf(rpl)), "empty splits differ"
    fin = ~np.isneginf(rpl)
    assert np.abs(pl_g[fin] - rpl[fin]).max() <= 1e-3
    err = np.abs(got - want)
    assert err.max() <= 1e-2
    assert np.linalg.norm(got - want) / np.linalg.norm(want) <= 5e-3


@pytest.fixture(scope="module")
def dense_verify_ref():
    w = workloads.dense_verify()
    o_ref, lse_ref, bad = oracle_decode(w)
    assert bad == 0
    return w, o_ref, lse_ref


@pytest.mark.parametrize("nsplit", [16, 64, 0])
def test_dense_verify_config(dense_verify_ref, nsplit):
    """B1 T9 H8 at 46080 + 9 tokens, every output compared."""
    w, o_ref, lse_ref = dense_verify_ref
    o, lse = run_dense(w, nsplit)
    check_o_lse(o, lse, o_ref, lse_ref, f"dense_verify S={nsplit}")


def test_dense_lengths_out_of_range_are_clamped_and_counted():
    w = workloads.make_dense_workload("dense_bad", B=2, T=2, H=16, ctx_lens=[300, 300], seed=9)
    K = 310                                   # natural lengths 299, 300 lie inside [0, K]
    lens = w.seq_lens.clone()
    lens[0, 1] = K + 7                        # clamped to K (positions 300.. sit on page 4)
    lens[1, 0] = -3                           # clamped to 0: o = 0, lse = -inf
    w = dataclasses.replace(w, seq_lens=lens)
    binding.check_device(clear=True)
    wd = w.to(DEV)
    o, lse = binding.decode_dense(wd.q, wd.cache, wd.page_table, wd.seq_lens, w.scale, 4, K=K)
    st, n = binding.check_device(clear=True)
    assert st == 5 and n == 2, (binding.status_string(st), n)
    ref = dataclasses.replace(w, seq_lens=lens.clamp(0, K))
    o_ref, lse_ref, _ = oracle_decode(ref)
    check_o_lse(o, lse, o_ref, lse_ref, "dense clamped lengths")


def test_dense_positions_past_the_page_table_are_masked_and_counted():
    w = workloads.make_dense_workload("dense_pt", B=1, T=2, H=16, ctx_lens=[100], seed=3)
    lens = torch.tensor([[90, 200]], dtype=torch.int32)   # 2 pages = 128 positions mapped
    w = dataclasses.replace(w, seq_lens=lens)
    binding.check_device(clear=True)
    o, lse = run_dense(w, 4)
    st, n = binding.check_device(clear=True)
    o_ref, lse_ref, bad = oracle_decode(w)
    assert st == 5 and n == 200 - 128 == bad // w.H
    check_o_lse(o, lse, o_ref, lse_ref, "dense past the page table")


# ------------------------------------------------------------------ per-step data in host memory
@pytest.mark.parametrize("name,S", [("single_request", 0), ("spec_verify", 0), ("tiny", 1),
                                    ("tiny", 4)])
def test_decode_host_matches_device_decode(name, S):
    w = workloads.WORKLOADS[name]()
    wd = w.to(DEV)
    o_ref, lse_ref = binding.decode(wd.q, wd.cache, wd.page_table, wd.idx, w.scale, S)
    q_h, pt_h, idx_h = w.q.pin_memory(), w.page_table.pin_memory(), w.idx.pin_memory()
    o_h = torch.full(o_ref.shape, 5.0, dtype=torch.bfloat16).pin_memory()
    lse_h = torch.full(lse_ref.shape, 5.0, dtype=torch.float32).pin_memory()
    for _ in range(2):
        binding.decode_host(q_h, wd.cache, pt_h, idx_h, w.scale, S, o=o_h, lse=lse_h)
        torch.cuda.synchronize()
        # the same kernels on the same bytes: bit-identical to the device path
        assert torch.equal(o_h, o_ref.cpu()) and torch.equal(lse_h, lse_ref.cpu())


def test_decode_host_rejects_unpinned_memory_before_launch():
    w = workloads.tiny()
    wd = w.to(DEV)
    lib = binding.lib()
    o_h = torch.full((1, 1, 8, 512), 5.0, dtype=torch.bfloat16).pin_memory()
    lse_h = torch.full((1, 1, 8), 5.0, dtype=torch.float32).pin_memory()
    ws = torch.empty(binding.workspace_host_bytes(1, 1, 8, 256, w.pt_stride, 4), dtype=torch.uint8,
                     device=DEV)
    q_pageable = w.q.clone()                      # ordinary (pageable) host memory
    q_h, pt_h, idx_h = w.q.pin_memory(), w.page_table.pin_memory(), w.idx.pin_memory()
    st = lib.smla_decode_host(q_pageable.data_ptr(), wd.cache.data_ptr(), w.num_pages,
                              pt_h.data_ptr(), w.pt_stride, idx_h.data_ptr(), 1, 1, 8, 256, 64,
                              w.scale, 4, ws.data_ptr(), ws.numel(), o_h.data_ptr(),
                              lse_h.data_ptr(), None)
    assert st == 1 and "pinned" in lib.smla_last_error().decode()
    # a device pointer where host memory is expected is refused too
    st = lib.smla_decode_host(wd.q.data_ptr(), wd.cache.data_ptr(), w.num_pages, pt_h.data_ptr(),
                              w.pt_stride, idx_h.data_ptr(), 1, 1, 8, 256, 64, w.scale, 4,
                              ws.data_ptr(), ws.numel(), o_h.data_ptr(), lse_h.data_ptr(), None)
    assert st == 1
    st = lib.smla_decode_host(q_h.data_ptr(), wd.cache.data_ptr(), w.num_pages, pt_h.data_ptr(),
                              w.pt_stride, idx_h.data_ptr(), 1, 1, 8, 256, 64, w.scale, 4,
                              ws.data_ptr(), 100, o_h.data_ptr(), lse_h.data_ptr(), None)
    assert st == 4
    torch.cuda.synchronize()
    assert torch.all(o_h == 5.0) and torch.all(lse_h == 5.0)   # nothing ran


@pytest.mark.parametrize("bad", ["page_size", "heads", "scale", "cache_null", "cache_misaligned",
                                 "pt_stride"])
def test_decode_host_checks_every_argument_before_the_copy_kernel(bad):
    """A bad argument that smla_decode would reject is rejected by
    smla_decode_host before its copy kernel runs: the staging area of the
    workspace keeps its sentinel bytes and the host outputs stay untouched."""
    w = workloads.tiny()
    wd = w.to(DEV)
    lib = binding.lib()
    B, T, H, K = 1, 1, 8, 256
    q_h, pt_h, idx_h = w.q.pin_memory(), w.page_table.pin_memory(), w.idx.pin_memory()
    o_h = torch.full((B, T, H, 512), 5.0, dtype=torch.bfloat16).pin_memory()
    lse_h = torch.full((B, T, H), 5.0, dtype=torch.float32).pin_memory()
    ws = torch.full((binding.workspace_host_bytes(B, T, H, K, w.pt_stride, 4),), 0xA5,
                    dtype=torch.uint8, device=DEV)
    cache_raw = torch.empty(wd.cache.numel() * 2 + 64, dtype=torch.uint8, device=DEV)
    args = dict(q=q_h.data_ptr(), cache=wd.cache.data_ptr(), pt=pt_h.data_ptr(),
                pt_stride=w.pt_stride, idx=idx_h.data_ptr(), H=H, page=64, scale=w.scale)
    expect = {"page_size": 2, "heads": 2, "scale": 1, "cache_null": 1, "cache_misaligned": 3,
              "pt_stride": 1}[bad]
    if bad == "page_size":
        args["page"] = 32
    elif bad == "heads":
        args["H"] = 65
    elif bad == "scale":
        args["scale"] = float("nan")
    elif bad == "cache_null":
        args["cache"] = None
    elif bad == "cache_misaligned":
        args["cache"] = cache_raw.data_ptr() + 8
    else:
        args["pt_stride"] = 0
    st = lib.smla_decode_host(args["q"], args["cache"], w.num_pages, args["pt"], args["pt_stride"],
                              args["idx"], B, T, args["H"], K, args["page"], args["scale"], 4,
                              ws.data_ptr(), ws.numel(), o_h.data_ptr(), lse_h.data_ptr(), None)
    torch.cuda.synchronize()
    assert st == expect, binding.status_string(st)
    assert torch.all(ws == 0xA5), "the copy kernel ran before the argument check"
    assert torch.all(o_h == 5.0) and torch.all(lse_h == 5.0)


def test_concurrent_host_threads_on_separate_streams():
    # four host threads decode at once, each on its own stream and workspace,
    # with shapes that take different kernels (latency form, mma, tcgen05);
    # ctypes releases the GIL, so the library's calls really overlap
    import threading
    cases = [small("mt0", seed=40, B=1, T=1, H=16, K=2048, ctx=70000),
             small("mt1", seed=41, B=3, T=2, H=16, K=700, ctx=4000),
             small("mt2", seed=42, B=2, T=1, H=64, K=900, ctx=4000),
             small("mt3", seed=43, B=2, T=3, H=24, K=130, ctx=4000)]
    splits = [64, 3, 2, 5]
    devs = [w.to(DEV) for w in cases]
    torch.cuda.synchronize()
    results, errors = [None] * 4, []

    def run(i):
        try:
            s = torch.cuda.Stream()
            wd = devs[i]
            with torch.cuda.stream(s):
                for _ in range(5):
                    o, lse = binding.decode(wd.q, wd.cache, wd.page_table, wd.idx, cases[i].scale,
                                            splits[i], stream=s)
            s.synchronize()
            results[i] = (o, lse)
        except Exception as e:  # reported below, on the main thread
            errors.append(e)

    threads = [threading.Thread(target=run, args=(i,)) for i in range(4)]
    for t in threads:
        t.start()
    for t in threads:
        t.join()
    assert not errors, errors
    for i, w in enumerate(cases):
        o_ref, lse_ref, _ = oracle_decode(w)
        check_o_lse(results[i][0], results[i][1], o_ref, lse_ref, f"thread {i}")


@pytest.mark.parametrize("name", ["tiny", "spec_verify"])
def test_decode_host_word_aligned_index_and_page_table(name):
    """Index and page-table buffers that are 4-byte but not 16-byte aligned
    (views one int32 into pinned buffers): the copy kernel moves them as
    4-byte words; the result must equal the device decode bit for bit."""
    w = workloads.WORKLOADS[name]()
    wd = w.to(DEV)
    o_ref, lse_ref = binding.decode(wd.q, wd.cache, wd.page_table, wd.idx, w.scale, 0)
    idx_buf = torch.empty(w.idx.numel() + 1, dtype=torch.int32).pin_memory()
    pt_buf = torch.empty(w.page_table.numel() + 3, dtype=torch.int32).pin_memory()
    idx_h = idx_buf[1:].view(w.idx.shape)
    pt_h = pt_buf[3:].view(w.page_table.shape)
    idx_h.copy_(w.idx)
    pt_h.copy_(w.page_table)
    assert idx_h.data_ptr() % 16 != 0 and pt_h.data_ptr() % 16 != 0
    q_h = w.q.pin_memory()
    o_h = torch.empty(o_ref.shape, dtype=torch.bfloat16).pin_memory()
    lse_h = torch.empty(lse_ref.shape, dtype=torch.float32).pin_memory()
    binding.decode_host(q_h, wd.cache, pt_h, idx_h, w.scale, 0, o=o_h, lse=lse_h)
    torch.cuda.synchronize()
    assert torch.equal(o_h, o_ref.cpu()) and torch.equal(lse_h, lse_ref.cpu())


# ------------------------------------------------------------------ inputs rewritten between calls
def _second_inputs(w, seed):
    """Same shapes and cache, another q and another selection (every valid
    position moved to the next one of its sequence, padding kept), so that a
    stale read of either input from the previous call shows in the output."""
    g = torch.Generator().manual_seed(seed)
    q2 = (torch.randn(w.q.shape, generator=g) * 0.5).to(torch.bfloat16)
    ctx = torch.tensor(w.ctx_lens, dtype=torch.int32).view(-1, 1, 1)
    idx2 = torch.where(w.idx >= 0, (w.idx + 1) % ctx, w.idx).to(torch.int32).contiguous()
    return q2, idx2


@pytest.mark.parametrize("name", ["single_request", "spec_verify", "tiny", "batched", "mixed"])
def test_decode_host_inputs_change_every_call(name):
    """The partial pass is a programmatic dependent of the copy kernel that
    fills the workspace's staging area, so every call overwrites inputs that
    the previous call read.  Alternate two input sets on one workspace: each
    call must match the device decode of its own inputs bit for bit."""
    w = workloads.WORKLOADS[name]()
    wd = w.to(DEV)
    q2, idx2 = _second_inputs(w, 11)
    sets = [(w.q, w.idx), (q2, idx2)]
    refs = [binding.decode(q.to(DEV), wd.cache, wd.page_table, i.to(DEV), w.scale, 0) for q, i in sets]
    torch.cuda.synchronize()
    q_h, idx_h, pt_h = w.q.pin_memory(), w.idx.pin_memory(), w.page_table.pin_memory()
    o_h = torch.empty(refs[0][0].shape, dtype=torch.bfloat16).pin_memory()
    lse_h = torch.empty(refs[0][1].shape, dtype=torch.float32).pin_memory()
    B, T, H, K = w.B, w.T, w.H, w.K
    S = binding.choose_nsplit(B, T, H, K, 0)
    ws = torch.empty(binding.workspace_host_bytes(B, T, H, K, w.pt_stride, S), dtype=torch.uint8,
                     device=DEV)
    calls = 12 if name in ("batched", "mixed") else 24
    for c in range(calls):
        q, i = sets[c % 2]
        q_h.copy_(q)
        idx_h.copy_(i)
        binding.decode_host(q_h, wd.cache, pt_h, idx_h, w.scale, S, o=o_h, lse=lse_h, workspace=ws)
        torch.cuda.synchronize()
        o_ref, lse_ref = refs[c % 2]
        assert torch.equal(o_h, o_ref.cpu()) and torch.equal(lse_h, lse_ref.cpu()), f"call {c}"


@pytest.mark.parametrize("name", ["single_request", "spec_verify", "batched", "mixed", "dense_verify"])
def test_decode_right_after_a_kernel_that_rewrites_its_inputs(name):
    """Device path: a copy kernel rewrites q and the selection (or the visible
    lengths) on the stream just before each decode, alternating two sets; the
    decode's first kernel may be scheduled while that copy still runs and
    must still read the new inputs."""
    w = workloads.WORKLOADS[name]()
    wd = w.to(DEV)
    if w.dense:
        g = torch.Generator().manual_seed(12)
        q2 = (torch.randn(w.q.shape, generator=g) * 0.5).to(torch.bfloat16)
        lens2 = (w.seq_lens - 37).clamp(min=0)
        sets = [(w.q.to(DEV), w.seq_lens.to(DEV)), (q2.to(DEV), lens2.to(DEV))]
        refs = [binding.decode_dense(q, wd.cache, wd.page_table, l, w.scale, 0, K=w.K) for q, l in sets]
    else:
        q2, idx2 = _second_inputs(w, 12)
        sets = [(w.q.to(DEV), w.idx.to(DEV)), (q2.to(DEV), idx2.to(DEV))]
        refs = [binding.decode(q, wd.cache, wd.page_table, i, w.scale, 0) for q, i in sets]
    torch.cuda.synchronize()
    q_d, sel_d = sets[0][0].clone(), sets[0][1].clone()
    for c in range(16):
        q, sel = sets[c % 2]
        q_d.copy_(q)
        sel_d.copy_(sel)
        if w.dense:
            o, lse = binding.decode_dense(q_d, wd.cache, wd.page_table, sel_d, w.scale, 0, K=w.K)
        else:
            o, lse = binding.decode(q_d, wd.cache, wd.page_table, sel_d, w.scale, 0)
        torch.cuda.synchronize()
        o_ref, lse_ref = refs[c % 2]
        assert torch.equal(o, o_ref) and torch.equal(lse, lse_ref), f"call {c}"
