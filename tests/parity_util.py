"""Shared helpers for the GPU parity tests: oracle calls on workload tensors and
the tolerance checks (bf16 inputs, fp32 accumulation)."""
import math

import numpy as np
import torch

import oracle

# Tolerances of the problem statement: o max-abs <= 1e-2 and relative L2
# <= 5e-3 over the whole o tensor; lse max-abs <= 1e-3 over finite entries,
# and -inf must match exactly.
O_MAX_ABS = 1e-2
O_REL_L2 = 5e-3
LSE_MAX_ABS = 1e-3


def bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def oracle_decode(w, sample=None):
    """Oracle o/lse for workload ``w``; ``sample`` = list of (b, t) to evaluate
    (returns arrays stacked in that order), or None for the whole batch."""
    if w.dense:
        return oracle_decode_dense(w, sample)
    q, cache, pt, idx = bits(w.q), bits(w.cache), w.page_table.cpu().numpy(), w.idx.cpu().numpy()
    if sample is None:
        o, lse, bad = oracle.decode(q, cache, pt, idx, w.scale)
        return o, lse, bad
    os_, ls_, bad = [], [], 0
    for b, t in sample:
        o, lse, n = oracle.decode(q[b:b + 1, t:t + 1], cache, pt[b:b + 1], idx[b:b + 1, t:t + 1],
                                  w.scale)
        os_.append(o[0, 0])
        ls_.append(lse[0, 0])
        bad += n
    return np.stack(os_), np.stack(ls_), bad


def oracle_decode_dense(w, sample=None):
    q, cache, pt = bits(w.q), bits(w.cache), w.page_table.cpu().numpy()
    lens = w.seq_lens.cpu().numpy()
    if sample is None:
        return oracle.decode_dense(q, cache, pt, lens, w.scale)
    os_, ls_, bad = [], [], 0
    for b, t in sample:
        o, lse, n = oracle.decode_dense(q[b:b + 1, t:t + 1], cache, pt[b:b + 1],
                                        lens[b:b + 1, t:t + 1], w.scale)
        os_.append(o[0, 0])
        ls_.append(lse[0, 0])
        bad += n
    return np.stack(os_), np.stack(ls_), bad


def check_o_lse(o_gpu, lse_gpu, o_ref, lse_ref, what=""):
    """Assert the tolerances; returns (max_abs, rel_l2, lse_err) for reporting."""
    o = o_gpu.detach().float().cpu().numpy().astype(np.float64)
    lse = lse_gpu.detach().float().cpu().numpy().astype(np.float64)
    assert o.shape == o_ref.shape, (o.shape, o_ref.shape)
    assert np.all(np.isfinite(o)), f"{what}: non-finite o"
    err = np.abs(o - o_ref)
    max_abs = float(err.max()) if err.size else 0.0
    denom = float(np.linalg.norm(o_ref))
    rel = float(np.linalg.norm(o - o_ref) / denom) if denom > 0 else float(np.linalg.norm(o))
    ninf_ref = np.isneginf(lse_ref)
    assert np.array_equal(np.isneginf(lse), ninf_ref), f"{what}: -inf lse pattern differs"
    fin = ~ninf_ref
    lse_err = float(np.abs(lse[fin] - lse_ref[fin]).max()) if fin.any() else 0.0
    assert max_abs <= O_MAX_ABS, f"{what}: o max-abs {max_abs:.3e} > {O_MAX_ABS}"
    assert rel <= O_REL_L2, f"{what}: o rel-L2 {rel:.3e} > {O_REL_L2}"
    assert lse_err <= LSE_MAX_ABS, f"{what}: lse err {lse_err:.3e} > {LSE_MAX_ABS}"
    # The same relative-L2 bound per output row (one (b, t, h)): |o| is about
    # |c| / sqrt(valid rows) here, so the max-abs bound alone is loose, and
    # one wrong row among thousands could pass the whole-tensor bound.  A row
    # whose reference is exactly zero (nothing selected) must be zero.
    if o.size:
        o2, r2 = o.reshape(-1, o.shape[-1]), o_ref.reshape(-1, o_ref.shape[-1])
        num = np.linalg.norm(o2 - r2, axis=1)
        den = np.linalg.norm(r2, axis=1)
        zero = den == 0
        assert np.all(num[zero] == 0), f"{what}: non-zero o where nothing is selected"
        row_rel = num[~zero] / den[~zero]
        worst = float(row_rel.max()) if row_rel.size else 0.0
        assert worst <= O_REL_L2, f"{what}: o rel-L2 of one row {worst:.3e} > {O_REL_L2}"
    return max_abs, rel, lse_err


def normalised_partials(po, pm, pl):
    """part_o * exp(part_m - part_lse): each split's normalised output (0 if empty)."""
    po = np.asarray(po, np.float64)
    pm = np.asarray(pm, np.float64)
    pl = np.asarray(pl, np.float64)
    w = np.where(np.isneginf(pl), 0.0, np.exp(np.where(np.isneginf(pl), 0.0, pm - pl)))
    return po * w[..., None]


def sample_bt(w, n, seed=0):
    rng = np.random.default_rng(seed)
    pairs = [(b, t) for b in range(w.B) for t in range(w.T)]
    if len(pairs) <= n:
        return pairs
    sel = rng.choice(len(pairs), n, replace=False)
    return [pairs[i] for i in sorted(sel)]


def lse_is_close(a, b, tol=LSE_MAX_ABS):
    return (a == b) or (math.isfinite(a) and math.isfinite(b) and abs(a - b) <= tol)
