#!/usr/bin/env python
"""Benchmark of split-K sparse MLA decode on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                    [--nsplit S] [--impl ours|reference]

One step = one whole decode (partial pass + LSE combine, through the C ABI)
over one batch of the named synthetic workload, inputs resident in HBM.  L2
is flushed before every step; each step is timed with CUDA events on the
launching stream; `ms_per_step` is the median (the mean is reported beside
it).  Rank 0 prints one JSON line.  Under torchrun every rank runs an
independent replica (its own seed), so per-GPU work is fixed (weak scaling)
and the step time is the max over ranks.

On one GPU the line also carries a `workloads` record: the memory-bound
batched and mixed-length configurations and the two verify shapes, each
measured after the headline in the same process under the same protocol
(decode and partial pass at the heuristic NSPLIT, medians, its own roofline
and clock record), plus the top-k indexer ahead of the mixed-length decode.

The metric (query tokens per second, us per call and achieved HBM GB/s,
against NSPLIT) follows "The Occupancy Hypothesis ..." (section "The
Experiment": decode throughput measured against NSPLIT) and "The Moment of
Truth ..." (section "The Split-K Imperative": the C=1 single-request case).
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "sparse MLA decode query-tokens/s, µs/call and achieved HBM GB/s vs NSPLIT"
UNIT = "query-tokens/s"
DEFAULT_WORKLOAD = "single_request"
L2_FLUSH_BYTES = 256 << 20
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0


def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawTextHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=400)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--nsplit", type=int, default=0, help="0 = the library's heuristic")
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-sweep", action="store_true", help="skip the NSPLIT sweep")
    ap.add_argument("--no-workloads", action="store_true",
                    help="skip the other configurations measured beside the headline")
    ap.add_argument("--cpu-seconds", type=float, default=6.0,
                    help="seconds of oracle CPU time for the baseline sample")
    return ap.parse_args(argv)


# ----------------------------------------------------------------------------- workload facts
def workload_bytes(w):
    """Algorithmic bytes of one step.

    partial pass, per query token: every valid selected row once (1152 B),
    its page-table entry (4 B), the K index entries (4 B each) and q
    (H * 1152 B); the combine adds o (H * 1024 B) and lse (H * 4 B).
    Dense variant: the T query tokens of a sequence attend to nested prefixes
    of the same rows, so each row of the longest prefix counts once (with its
    page-table entry), plus the visible lengths (4 B per query token).
    """
    BT = w.B * w.T
    if w.dense:
        rows = int(w.seq_lens.max(dim=1).values.to(__import__("torch").int64).sum())
        partial = rows * (1152 + 4) + BT * 4 + BT * w.H * 1152
    else:
        partial = w.n_valid() * (1152 + 4) + BT * w.K * 4 + BT * w.H * 1152
    step = partial + BT * w.H * (1024 + 4)
    return partial, step


def workload_flops(w):
    """2 * H * valid * (576 + 512): QK^T over 576 dims and PV over 512."""
    return 2 * w.H * w.n_valid() * (576 + 512)


def describe(w):
    sel = (f"dense causal prefixes of {int(w.seq_lens.min())}..{w.K} positions" if w.dense
           else f"K{w.K}")
    return (f"B{w.B} T{w.T} H{w.H} {sel} dc512+dr64 bf16, paged cache page64, "
            f"{w.num_pages} pages, ctx {min(w.ctx_lens)}..{max(w.ctx_lens)}")


def data_note(w):
    sel = ("every visible position of each draft token (dense causal verify)" if w.dense
           else "distinct random top-k indices")
    return f"synthetic (seeded N(0,1)*0.5 bf16 q and cache, {sel})"


# The sources each partial kernel's code and launch shape come from: a
# recorded ncu traffic figure stays valid while these files are unchanged.
KERNEL_SOURCES = {
    "smla_partial_small_kernel": ["smla_api.cu", "smla_partial_mma.cuh", "smla_ptx.cuh"],
    "smla_partial_mma_kernel": ["smla_api.cu", "smla_partial_mma.cuh", "smla_ptx.cuh"],
    "smla_partial_tc_kernel": ["smla_api.cu", "smla_partial_mma.cuh", "smla_partial_tc.cuh",
                               "smla_ptx.cuh", "smla_tc_ptx.cuh"],
    "smla_ix_score_kernel": ["smla_api.cu", "smla_indexer.cuh", "smla_ptx.cuh", "smla_tc_ptx.cuh"],
}


def kernel_sources_hash(kernel: str) -> str:
    """sha256[:16] over the kernel's source files (KERNEL_SOURCES), in order,
    with comments and whitespace removed (a comment edit does not change the
    kernel)."""
    import hashlib
    import re
    h = hashlib.sha256()
    for name in KERNEL_SOURCES[kernel]:
        with open(os.path.join(ROOT, "sparse_mla_decode_partial_b200", "csrc", name)) as f:
            text = f.read()
        text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)   # block comments
        text = re.sub(r"//[^\n]*", " ", text)                 # line comments
        h.update(re.sub(r"\s+", "", text).encode())
    return h.hexdigest()[:16]


def measured_traffic(workload: str):
    """DRAM bytes (read + write) per launch of the partial kernel for this
    workload from the committed ncu capture, or None when no capture exists
    or that kernel's sources changed since it was taken."""
    try:
        with open(os.path.join(ROOT, "profiles", "ncu_traffic.json")) as f:
            rec = json.load(f)[workload]
        ok = kernel_sources_hash(rec["kernel"]) == rec["sources_sha256_16"]
    except (OSError, KeyError, ValueError):
        return None
    return rec["traffic_bytes_per_launch"] if ok else None


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), float(p["bf16_tflops"]), "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, "fallback"


# ----------------------------------------------------------------------------- clocks
def partial_kernel_name(H: int, K: int, nsplit: int, pt_stride: int, dense: bool = False) -> str:
    """The partial kernel the library launches for this shape (its dispatch rule;
    the dense variant always runs the tcgen05 kernel)."""
    if dense:
        return "smla_partial_tc_kernel"
    kc = -(-K // nsplit) if K > 0 else 0
    if H <= 32 and K > 0 and kc <= 64 and pt_stride <= 8192:
        return "smla_partial_small_kernel"
    return "smla_partial_tc_kernel" if H > 32 else "smla_partial_mma_kernel"


class ClockSampler:
    """Samples SM clock and throttle reasons through NVML while running."""

    HW = {"hw_slowdown": 0x8, "hw_thermal_slowdown": 0x40, "sw_thermal_slowdown": 0x20,
          "sw_power_cap": 0x4, "hw_power_brake_slowdown": 0x80}

    def __init__(self, device_index: int, period_s: float = 0.002):
        self.period = period_s
        self.samples = []
        self.reasons = 0
        self.max_mhz = None
        self._stop = threading.Event()
        self._thread = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception:  # NVML missing: no clock record
            self._nv = None
        if self._nv is not None:
            # the first queries of a process can take longer than a short timed
            # region; pay for them here, before it starts
            try:
                self._nv.nvmlDeviceGetClockInfo(self._h, self._nv.NVML_CLOCK_SM)
                self._nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
            except Exception:
                pass
        self.after_region = False

    def _run(self):
        nv = self._nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                self.reasons |= nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self._nv is not None:
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()
        return self

    def __exit__(self, *exc):
        self._stop.set()
        if self._thread is not None:
            self._thread.join()
        if self._nv is not None and not self.samples:
            # nothing landed inside the region: one read right after it, flagged
            try:
                self.samples.append(self._nv.nvmlDeviceGetClockInfo(self._h, self._nv.NVML_CLOCK_SM))
                self.reasons |= self._nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                self.after_region = True
            except Exception:
                pass

    def summary(self):
        if self._nv is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvml unavailable"]}
        names = [k for k, bit in self.HW.items() if self.reasons & bit]
        out = {"sm_mhz": statistics.median(self.samples) if self.samples else None,
               "sm_max_mhz": self.max_mhz, "reasons": names, "samples": len(self.samples)}
        if self.after_region:
            out["sampled"] = "once, right after the timed region (no sample landed inside it)"
        return out


# ----------------------------------------------------------------------------- distributed
def dist_init():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return world, rank, local


def replica_workload(name: str, rank: int, world: int):
    """The workload one rank runs: rank r of an N-rank job draws an independent
    replica of the named workload (seed offset 1000 * r), so every GPU has the
    same amount of work (weak scaling) and no data crosses ranks."""
    import inspect
    from sparse_mla_decode_partial_b200 import workloads
    builder = workloads.WORKLOADS[name]
    if world == 1:
        return builder()
    base_seed = inspect.signature(builder).parameters["seed"].default
    return builder(seed=base_seed + 1000 * rank)


def aggregate(tokens_local: float, ms_local: float, world: int):
    """Whole-job throughput: query tokens of all ranks / the slowest rank's
    step time.  Returns (tokens_all, ms_max, tokens per second)."""
    ms_max = max_over_ranks(ms_local, world)
    tokens_all = sum_over_ranks(tokens_local, world)
    return tokens_all, ms_max, tokens_all / (ms_max * 1e-3)


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    dev = torch.device("cuda", torch.cuda.current_device()) if torch.cuda.is_available() else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    dev = torch.device("cuda", torch.cuda.current_device()) if torch.cuda.is_available() else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


# ----------------------------------------------------------------------------- oracle baseline
def cpu_baseline(w, seconds: float):
    """The fp64 oracle as it stands, on this host's cores, over whole steps of
    the same workload (or the first query tokens of one step when a step alone
    exceeds that time)."""
    import numpy as np
    import oracle
    bits = lambda t: t.contiguous().view(__import__("torch").int16).numpy().view(np.uint16)
    q, cache = bits(w.q), bits(w.cache)
    pt = w.page_table.numpy()
    # the dense variant's lists are every visible position (the oracle's own
    # construction); the sparse workloads carry theirs
    idx = oracle.dense_positions(w.seq_lens.numpy(), w.K) if w.dense else w.idx.numpy()
    threads = oracle.max_threads()
    units = w.B * w.T * w.H
    # one query token first, to size the sample
    t0 = time.perf_counter()
    oracle.decode(q[:1, :1], cache, pt[:1], idx[:1, :1], w.scale)
    per_token = time.perf_counter() - t0
    n_tok = max(1, min(w.B * w.T, int(seconds / max(per_token, 1e-9))))
    bt = [(b, t) for b in range(w.B) for t in range(w.T)][:n_tok]
    reps = 0
    t0 = time.perf_counter()
    while True:
        for b, t in bt:
            oracle.decode(q[b:b + 1, t:t + 1], cache, pt[b:b + 1], idx[b:b + 1, t:t + 1], w.scale)
        reps += 1
        if time.perf_counter() - t0 >= seconds * 0.5 or reps >= 50:
            break
    el = time.perf_counter() - t0
    tokens = reps * len(bt)
    sample = (f"{len(bt)} of {w.B * w.T} query tokens of one step (all {w.H} heads, "
              f"{'dense, up to ' if w.dense else ''}K={w.K}) x {reps} repeats")
    # the same oracle on one thread, over the first query token (a few repeats)
    oracle.set_threads(1)
    try:
        n1, t0 = 0, time.perf_counter()
        while n1 < 5 and (n1 == 0 or time.perf_counter() - t0 < seconds * 0.25):
            b, t = bt[0]
            oracle.decode(q[b:b + 1, t:t + 1], cache, pt[b:b + 1], idx[b:b + 1, t:t + 1], w.scale)
            n1 += 1
        one_thread = n1 / (time.perf_counter() - t0)
    finally:
        oracle.set_threads(threads)
    model = ""
    try:
        with open("/proc/cpuinfo") as f:
            model = next((ln.split(":", 1)[1].strip() for ln in f if ln.startswith("model name")), "")
    except OSError:
        pass
    return {"value": tokens / el, "unit": UNIT, "cores": min(threads, w.H), "kind": "oracle",
            "sample": sample, "threads_available": threads, "us_per_token": el / tokens * 1e6,
            "value_1_thread": one_thread, "cpu_model": model}


# ----------------------------------------------------------------------------- GPU arm
# Workloads measured beside the headline in the same invocation: the
# memory-bound configurations the roofline target is stated on (batched,
# mixed) and the two verify shapes.
SIDE_WORKLOADS = ("batched", "mixed", "spec_verify", "dense_verify")


def bench_config(w, workload: str, nsplit_arg: int, world: int) -> dict:
    """The `config` object of the JSON line, identical in both arms for the
    same command line (the split count the library resolves is reported
    beside it, as `nsplit_used`)."""
    return {"workload": workload, "shape": describe(w),
            "nsplit": nsplit_arg if nsplit_arg else "heuristic",
            "batch": w.B, "q_len": w.T, "heads": w.H, "topk": w.K,
            "l2": "flushed before every step: 256 MB write then 256 MB read",
            "parallelism": f"replicas x{world}" if world > 1 else "single GPU"}


INDEXER_DATA = "synthetic (seeded index queries, keys and weights)"


def indexer_shape(w) -> str:
    return (f"B{w.B} T{w.T} HI{w.HI} x128 bf16 index keys, top-{w.K}, ctx "
            f"{min(w.ctx_lens)}..{max(w.ctx_lens)}")


def indexer_config(w, world: int) -> dict:
    """The `config` object of an indexer_mixed line, identical in both arms."""
    return {"workload": "indexer_mixed", "shape": indexer_shape(w),
            "l2": "flushed before every step: 256 MB write then 256 MB read",
            "parallelism": f"replicas x{world}" if world > 1 else "single GPU"}


class Harness:
    """Device-side timing through the C ABI on one stream: L2 flush before
    every step, CUDA events on the launching stream around each step."""

    def __init__(self, dev):
        import torch
        from sparse_mla_decode_partial_b200 import binding
        self.torch, self.binding, self.lib = torch, binding, binding.lib()
        self.dev = dev
        self.stream = torch.cuda.current_stream(dev)
        self.sptr = self.stream.cuda_stream
        self.flush_w = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
        self.flush_r = torch.ones(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
        self.sink = torch.empty(1, dtype=torch.float32, device=dev)

    def flush(self):
        self.flush_w.fill_(1.0)
        self.torch.sum(self.flush_r, dim=0, out=self.sink[0])

    def steps(self, w, S):
        """(decode step, partial-only step) for NSPLIT = S on device workload w;
        each returns (status, kernel launches)."""
        torch, binding, lib, sptr, dev = self.torch, self.binding, self.lib, self.sptr, self.dev
        B, T, H, K = w.B, w.T, w.H, w.K
        n = B * T * H * S
        po = torch.empty(max(n * 512, 4), dtype=torch.float32, device=dev)
        pm = torch.empty(max(n, 1), dtype=torch.float32, device=dev)
        pl = torch.empty(max(n, 1), dtype=torch.float32, device=dev)
        o = torch.empty((B, T, H, 512), dtype=torch.bfloat16, device=dev)
        lse = torch.empty((B, T, H), dtype=torch.float32, device=dev)
        if w.dense:
            ws = torch.empty(max(16, binding.dense_workspace_bytes(B, T, H, K, S)),
                             dtype=torch.uint8, device=dev)
            common = (w.q.data_ptr(), w.cache.data_ptr(), w.num_pages, w.page_table.data_ptr(),
                      w.pt_stride, w.seq_lens.data_ptr(), B, T, H, K, 64, w.scale)
            whole, part = lib.smla_decode_dense, lib.smla_decode_dense_partial
        else:
            ws = torch.empty(max(16, binding.workspace_bytes(B, T, H, S)), dtype=torch.uint8,
                             device=dev)
            common = (w.q.data_ptr(), w.cache.data_ptr(), w.num_pages, w.page_table.data_ptr(),
                      w.pt_stride, w.idx.data_ptr(), B, T, H, K, 64, w.scale)
            whole, part = lib.smla_decode, None

        def decode():
            """One whole decode: partial pass + LSE combine in one call."""
            st = whole(*common, S, ws.data_ptr(), ws.numel(), o.data_ptr(), lse.data_ptr(), sptr)
            return st, (1 if S == 1 else 2)

        def partial():
            """The decode's partial pass alone, as the decode launches it (the
            balanced schedule included); with S = 1 it writes o and lse."""
            if S == 1:
                return whole(*common, 1, None, 0, o.data_ptr(), lse.data_ptr(), sptr), 1
            if part is None:
                return lib.smla_decode_partial_ws(*common, S, ws.data_ptr(), ws.numel(), sptr), 1
            return part(*common, S, po.data_ptr(), pm.data_ptr(), pl.data_ptr(), sptr), 1
        return decode, partial

    def timed(self, step, n):
        """n flushed steps; returns (per-step ms list, kernel launches)."""
        torch = self.torch
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(n)]
        launches = 0
        for i in range(n):
            self.flush()
            ev[i][0].record(self.stream)
            st, nl = step()
            ev[i][1].record(self.stream)
            if st != 0:
                raise RuntimeError(self.binding.status_string(st))
            launches += nl
        torch.cuda.synchronize(self.dev)
        return [e[0].elapsed_time(e[1]) for e in ev], launches

    def warm(self, fns, n):
        for _ in range(max(3, n)):
            for f in fns:
                self.flush()
                f()
        self.torch.cuda.synchronize(self.dev)


def roofline(w_host, nsplit, part_ms, workload, hbm_peak, tc_peak, peak_src):
    """The partial kernel's roofline record: algorithmic bytes per launch over
    its CUDA-event duration, against the measured HBM copy bandwidth."""
    part_bytes, _ = workload_bytes(w_host)
    flops = workload_flops(w_host)
    part_us = part_ms * 1e3
    achieved = part_bytes / (part_us * 1e-6) / 1e9
    tc_achieved = flops / (part_us * 1e-6) / 1e12
    return {"bound": "hbm",
            "kernel": partial_kernel_name(w_host.H, w_host.K, nsplit, w_host.pt_stride,
                                          w_host.dense),
            "achieved": round(achieved, 1), "peak": hbm_peak, "unit": "GB/s",
            "frac": round(achieved / hbm_peak, 4),
            "peak_source": (f"{peak_src} (MEASURED_PEAKS.json hbm_gbs)" if peak_src == "measured"
                            else "fallback"),
            "traffic": measured_traffic(workload),
            "traffic_source": "profiles/ncu_traffic.json (ncu dram__bytes_read.sum + "
                              "dram__bytes_write.sum of one capture of this kernel)",
            "algorithmic_bytes_per_launch": part_bytes,
            "partial_us_median": round(part_us, 3),
            "tensor_tflops": round(tc_achieved, 2),
            "tensor_frac_of_bf16_peak": round(tc_achieved / tc_peak, 4)}


def side_workload(h, name, steps, warmup, peaks):
    """One configuration measured beside the headline: decode and partial pass
    at the heuristic NSPLIT, the same flush protocol, its own clock record."""
    import torch
    from sparse_mla_decode_partial_b200 import binding, workloads
    w_host = workloads.WORKLOADS[name]()
    w = w_host.to(h.dev)
    B, T, H, K = w.B, w.T, w.H, w.K
    S = binding.dense_nsplit(B, T, H, K) if w.dense else binding.choose_nsplit(B, T, H, K, 0)
    decode, partial = h.steps(w, S)
    h.warm([decode, partial], warmup)
    sampler = ClockSampler(h.dev.index)
    with sampler:
        tot, launches = h.timed(decode, steps)
        part, _ = h.timed(partial, steps)
    _, step_bytes = workload_bytes(w_host)
    us = statistics.median(tot) * 1e3
    rec = {"shape": describe(w_host), "nsplit": S, "steps": steps,
           "us_per_call": round(us, 3), "us_per_call_mean": round(statistics.fmean(tot) * 1e3, 3),
           "partial_us": round(statistics.median(part) * 1e3, 3),
           "partial_us_mean": round(statistics.fmean(part) * 1e3, 3),
           "q_tok_s": round(B * T / (us * 1e-6), 1),
           "hbm_gbs_step": round(step_bytes / (us * 1e-6) / 1e9, 1),
           "roofline": roofline(w_host, S, statistics.median(part), name, *peaks),
           "gpu_launches": launches, "clocks": sampler.summary()}
    del w, decode, partial
    torch.cuda.empty_cache()
    return rec


def indexer_bytes(w):
    """Algorithmic bytes of one indexer call: every visible index key once
    (256 B), its page-table entry once per 64 positions, the index queries
    (HI x 256 B) and weights (HI x 4 B) of every query token, its visible
    length, and the K output entries (4 B)."""
    n = w.n_vis.to(__import__("torch").int64).clamp(min=0)
    keys = int(n.sum())
    pages = int(((n + 63) // 64).sum())
    BT = w.B * w.T
    return keys * 256 + pages * 4 + BT * w.HI * (256 + 4) + BT * 4 + BT * w.K * 4


def side_indexer(h, steps, warmup, peaks):
    """The top-k indexer ahead of the mixed-length decode (B60 T1, contexts
    1K..128K, 64 index heads, top-2048), timed through smla_indexer_topk,
    with its scoring and selection steps also timed alone."""
    import torch
    from sparse_mla_decode_partial_b200 import binding, workloads
    w_host = workloads.indexer_mixed()
    w = w_host.to(h.dev)
    B, T, HI, K, max_n = w.B, w.T, w.HI, w.K, w_host.max_n
    lib, sptr = h.lib, h.sptr
    ws = torch.empty(binding.indexer_workspace_bytes(B, T, max_n), dtype=torch.uint8, device=h.dev)
    out = torch.empty((B, T, K), dtype=torch.int32, device=h.dev)
    sc = torch.empty((B, T, max_n), dtype=torch.float32, device=h.dev)
    sel_ws = torch.empty(binding.indexer_select_workspace_bytes(B, T, max_n), dtype=torch.uint8,
                         device=h.dev)
    common = (w.q_index.data_ptr(), w.w.data_ptr(), w.k_index.data_ptr(), w.num_pages,
              w.page_table.data_ptr(), w.pt_stride, w.n_vis.data_ptr(), B, T, HI, max_n)

    def topk():
        return lib.smla_indexer_topk(*common, K, 64, ws.data_ptr(), ws.numel(), out.data_ptr(),
                                     sptr), 4

    def scores():
        return lib.smla_indexer_scores(*common, 64, ws.data_ptr(), ws.numel(), sc.data_ptr(),
                                       sptr), 2

    def select():
        return lib.smla_indexer_select(sc.data_ptr(), w.n_vis.data_ptr(), B, T, max_n, K,
                                       sel_ws.data_ptr(), sel_ws.numel(), out.data_ptr(), sptr), 4
    h.warm([topk, scores, select], warmup)
    sampler = ClockSampler(h.dev.index)
    with sampler:
        t_all, launches = h.timed(topk, steps)
        t_sc, _ = h.timed(scores, steps)
        t_sel, _ = h.timed(select, steps)
    us, us_sc, us_sel = (statistics.median(t) * 1e3 for t in (t_all, t_sc, t_sel))
    nbytes = indexer_bytes(w_host)
    hbm_peak, tc_peak, peak_src = peaks
    key_bytes = nbytes - B * T * K * 4
    flops = 2 * int(w_host.n_vis.clamp(min=0).sum()) * HI * 128
    rec = {"shape": indexer_shape(w_host), "query_tokens": B * T,
           "steps": steps, "us_per_call": round(us, 3),
           "us_per_call_mean": round(statistics.fmean(t_all) * 1e3, 3),
           "q_tok_s": round(B * T / (us * 1e-6), 1),
           "scores_us": round(us_sc, 3), "select_us": round(us_sel, 3),
           "roofline": {"bound": "hbm", "kernel": "smla_ix_score_kernel",
                        "achieved": round(key_bytes / (us_sc * 1e-6) / 1e9, 1),
                        "peak": hbm_peak, "unit": "GB/s",
                        "frac": round(key_bytes / (us_sc * 1e-6) / 1e9 / hbm_peak, 4),
                        "peak_source": peak_src,
                        "traffic": measured_traffic("indexer_mixed"),
                        "algorithmic_bytes_per_launch": key_bytes,
                        "tensor_tflops": round(flops / (us_sc * 1e-6) / 1e12, 2),
                        "tensor_frac_of_bf16_peak": round(flops / (us_sc * 1e-6) / 1e12 / tc_peak, 4),
                        "note": "scoring kernel (plan + scores) timed alone; bytes: keys, page "
                                "entries, queries, weights and lengths, read once"},
           "whole_call_frac_of_hbm": round(nbytes / (us * 1e-6) / 1e9 / hbm_peak, 4),
           "gpu_launches": launches, "clocks": sampler.summary()}
    del w, ws, sc, sel_ws
    torch.cuda.empty_cache()
    return rec


def run_indexer_headline(args, world, rank, local):
    """`--workload indexer_mixed`: the top-k indexer as the timed step (the
    profiling recipe's launch list and captures of the indexer kernels use
    it); the line carries the indexer record's figures.  Under torchrun every
    rank runs the same workload (weak scaling) and the line reports all
    ranks' query tokens over the slowest rank's time."""
    import torch
    from sparse_mla_decode_partial_b200 import build
    build.build()
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    h = Harness(dev)
    barrier(world)
    torch.cuda.synchronize(dev)
    rec = side_indexer(h, args.steps, args.warmup, load_peaks())
    barrier(world)
    torch.cuda.synchronize(dev)
    _, ms_max, value = aggregate(float(rec["query_tokens"]), rec["us_per_call"] * 1e-3, world)
    if rank != 0:
        return None
    from sparse_mla_decode_partial_b200 import workloads
    w = workloads.indexer_mixed()
    return {"metric": "top-k indexer query-tokens/s", "value": round(value, 1),
            "unit": UNIT, "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(ms_max, 6), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": INDEXER_DATA,
            "config": indexer_config(w, world),
            "roofline": rec["roofline"], "clocks": rec["clocks"], "gpu_launches": rec["gpu_launches"],
            "indexer": rec}


def run_ours(args, world, rank, local):
    import torch
    from sparse_mla_decode_partial_b200 import binding, build

    if args.workload == "indexer_mixed":
        return run_indexer_headline(args, world, rank, local)
    build.build()
    lib = binding.lib()
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    h = Harness(dev)
    sptr = h.sptr
    w_host = replica_workload(args.workload, rank, world)
    w = w_host.to(dev)
    B, T, H, K = w.B, w.T, w.H, w.K
    nsplit = args.nsplit or (binding.dense_nsplit(B, T, H, K) if w.dense
                             else binding.choose_nsplit(B, T, H, K, 0))
    stream = h.stream

    _, step_bytes = workload_bytes(w_host)
    peaks = load_peaks()

    step, part_step = h.steps(w, nsplit)
    h.warm([step, part_step], args.warmup)

    sampler = ClockSampler(dev.index)
    barrier(world)
    torch.cuda.synchronize(dev)
    with sampler:
        tot, launches = h.timed(step, args.steps)
        part, _ = h.timed(part_step, args.steps)
    barrier(world)
    torch.cuda.synchronize(dev)

    # median over the timed steps (the mean is reported beside it)
    ms_step = statistics.median(tot)
    ms_part = statistics.median(part)
    tokens_all, ms_step_max, value = aggregate(float(B * T), ms_step, world)
    ms_mean_max = max_over_ranks(statistics.fmean(tot), world)

    # e2e: per-step data in pinned host memory through the C ABI's host entry
    # point (smla_decode_host): the library pulls q, the top-k indices and the
    # page table over the host link with a copy kernel and writes o, lse
    # straight back into host memory; all of it inside the timed region.
    if w_host.dense:
        # the dense entry point takes device buffers: the step's q, visible
        # lengths and page table are copied from pinned host memory first, o
        # and lse back after, all on the launching stream inside the interval
        q_h, len_h = w_host.q.pin_memory(), w_host.seq_lens.pin_memory()
        pt_h = w_host.page_table.pin_memory()
        o_h = torch.empty((B, T, H, 512), dtype=torch.bfloat16).pin_memory()
        lse_h = torch.empty((B, T, H), dtype=torch.float32).pin_memory()
        q_d, len_d, pt_d = torch.empty_like(w.q), torch.empty_like(w.seq_lens), torch.empty_like(w.page_table)
        o_d = torch.empty((B, T, H, 512), dtype=torch.bfloat16, device=dev)
        lse_d = torch.empty((B, T, H), dtype=torch.float32, device=dev)
        ws_e = torch.empty(max(16, binding.dense_workspace_bytes(B, T, H, K, nsplit)),
                           dtype=torch.uint8, device=dev)
        h2d = q_h.numel() * 2 + len_h.numel() * 4 + pt_h.numel() * 4
        d2h = o_h.numel() * 2 + lse_h.numel() * 4

        def e2e_step():
            q_d.copy_(q_h, non_blocking=True)
            len_d.copy_(len_h, non_blocking=True)
            pt_d.copy_(pt_h, non_blocking=True)
            st = lib.smla_decode_dense(q_d.data_ptr(), w.cache.data_ptr(), w.num_pages,
                                       pt_d.data_ptr(), w.pt_stride, len_d.data_ptr(), B, T, H, K,
                                       64, w.scale, nsplit, ws_e.data_ptr(), ws_e.numel(),
                                       o_d.data_ptr(), lse_d.data_ptr(), sptr)
            o_h.copy_(o_d, non_blocking=True)
            lse_h.copy_(lse_d, non_blocking=True)
            return st
        e2e_note = ("smla_decode_dense every step: q, visible lengths and page table copied from "
                    "pinned host memory, o and lse copied back, on the launching stream; the "
                    "latent cache stays resident")
    else:
        q_h = w_host.q.pin_memory()
        idx_h = w_host.idx.pin_memory()
        pt_h = w_host.page_table.pin_memory()
        o_h = torch.empty((B, T, H, 512), dtype=torch.bfloat16).pin_memory()
        lse_h = torch.empty((B, T, H), dtype=torch.float32).pin_memory()
        ws_h = torch.empty(max(16, binding.workspace_host_bytes(B, T, H, K, w.pt_stride, nsplit)),
                           dtype=torch.uint8, device=dev)
        h2d = q_h.numel() * 2 + idx_h.numel() * 4 + pt_h.numel() * 4
        d2h = o_h.numel() * 2 + lse_h.numel() * 4

        def e2e_step():
            return lib.smla_decode_host(q_h.data_ptr(), w.cache.data_ptr(), w.num_pages,
                                        pt_h.data_ptr(), w.pt_stride, idx_h.data_ptr(), B, T, H, K,
                                        64, w.scale, nsplit, ws_h.data_ptr(), ws_h.numel(),
                                        o_h.data_ptr(), lse_h.data_ptr(), sptr)
        e2e_note = ("smla_decode_host every step: q, top-k indices and page table read from "
                    "pinned host memory by the library's copy kernel, o and lse written straight "
                    "into pinned host memory; the latent cache stays resident")
    for _ in range(3):
        e2e_step()
    torch.cuda.synchronize(dev)
    n_e2e = max(10, min(args.steps, 200))
    times = []
    for _ in range(n_e2e):
        h.flush()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        st = e2e_step()
        e1.record(stream)
        stream.synchronize()
        if st != 0:
            raise RuntimeError(binding.status_string(st))
        times.append(e0.elapsed_time(e1))
    e2e_ms = max_over_ranks(statistics.median(times), world)
    e2e = {"value": tokens_all / (e2e_ms * 1e-3), "unit": UNIT, "h2d_bytes_per_step": h2d,
           "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms,
           "ms_per_step_mean": max_over_ranks(statistics.fmean(times), world), "note": e2e_note}

    # Warm-L2 reference (after the timed region, not part of value): the same
    # step back to back without the flush, so the selected rows may still sit
    # in L2 from the previous call.
    warm = []
    for _ in range(3):
        step()
    torch.cuda.synchronize(dev)
    for _ in range(max(20, min(args.steps, 200))):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        step()
        e1.record(stream)
        warm.append((e0, e1))
    torch.cuda.synchronize(dev)
    warm_us = statistics.median(a.elapsed_time(b) for a, b in warm) * 1e3

    # NSPLIT sweep (rank 0 only, after the timed region)
    sweep = []
    if rank == 0 and not args.no_sweep:
        cands = list(w_host.nsplit_sweep) or sorted({1, 2, 4, 8, 16, 32, 64, nsplit})
        for S in sorted(set(cands) | {nsplit}):
            d_fn, p_fn = h.steps(w, S)
            h.warm([d_fn, p_fn], 5)
            nrep = max(20, min(args.steps, 200))
            t, _ = h.timed(d_fn, nrep)
            p_, _ = h.timed(p_fn, nrep)
            us = statistics.median(t) * 1e3
            sweep.append({"nsplit": S, "us_per_call": round(us, 3),
                          "partial_us": round(statistics.median(p_) * 1e3, 3),
                          "q_tok_s": round(B * T / (us * 1e-6), 1),
                          "hbm_gbs": round(step_bytes / (us * 1e-6) / 1e9, 1)})

    if rank != 0:
        return None

    # The other configurations, measured after the headline in the same
    # process (one GPU only: under torchrun the ranks would wait on rank 0)
    side = {}
    if world == 1 and not args.no_workloads:
        del w
        torch.cuda.empty_cache()
        for name in SIDE_WORKLOADS:
            if name != args.workload:
                side[name] = side_workload(h, name, min(args.steps, 200), args.warmup, peaks)
        side["indexer_mixed"] = side_indexer(h, min(args.steps, 100), args.warmup, peaks)

    line = {
        "metric": METRIC, "value": round(value, 2), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step_max, 6),
        "ms_per_step_mean": round(ms_mean_max, 6),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": data_note(w_host),
        "config": bench_config(w_host, args.workload, args.nsplit, world),
        "nsplit_used": nsplit,
        "us_per_call": round(ms_step_max * 1e3, 3),
        "hbm_gbs_step": round(step_bytes / (ms_step * 1e-3) / 1e9, 1),
        "kernel_us": {"partial": round(ms_part * 1e3, 3),
                      "partial_mean": round(statistics.fmean(part) * 1e3, 3),
                      "note": "the decode's partial pass timed alone (smla_decode_partial_ws, "
                              "the same kernel and schedule) in a second loop of the same "
                              "length (medians); the step runs it and the combine through one "
                              "smla_decode call"},
        "roofline": roofline(w_host, nsplit, ms_part, args.workload, *peaks),
        "warm_l2": {"us_per_call": round(warm_us, 3),
                    "note": "same step back to back without the L2 flush (labelled reference, "
                            "not the headline: repeated inputs leave the selected rows in L2)"},
        "gpu_launches": launches,
        "clocks": sampler.summary(),
        "e2e": e2e,
        "nsplit_sweep": sweep,
        "workloads": side,
    }
    return line


def indexer_cpu_baseline(seconds: float, w=None):
    """The fp64 indexer oracle on this host's cores over the first query
    tokens of the indexer workload (one token at a time until the time is
    spent)."""
    import numpy as np
    import torch
    from oracle import indexer as ix_oracle
    from sparse_mla_decode_partial_b200 import workloads
    if w is None:
        w = workloads.indexer_mixed()
    bits = lambda t: t.contiguous().view(torch.int16).numpy().view(np.uint16)
    q, k = bits(w.q_index), bits(w.k_index)
    wt, pt, nv = w.w.numpy(), w.page_table.numpy(), w.n_vis.numpy()
    done, keys = 0, 0
    t0 = time.perf_counter()
    while done < w.B and time.perf_counter() - t0 < seconds:
        b = done
        ix_oracle.topk(q[b:b + 1], wt[b:b + 1], k, pt[b:b + 1], nv[b:b + 1], w.K)
        keys += int(nv[b, 0])
        done += 1
    el = time.perf_counter() - t0
    return {"value": done / el, "unit": UNIT, "cores": __import__("os").cpu_count(),
            "kind": "oracle", "sample": f"the first {done} of {w.B} query tokens ({keys} keys)",
            "us_per_token": el / done * 1e6}


def run_reference(args, world, rank):
    """The oracle (CPU, fp64) as the reference arm, on this host's cores."""
    if rank != 0:
        return None
    from sparse_mla_decode_partial_b200 import workloads
    if args.workload == "indexer_mixed":
        w = workloads.indexer_mixed()
        res = indexer_cpu_baseline(max(2.0, args.cpu_seconds), w)
        return {"metric": "top-k indexer query-tokens/s", "value": round(res["value"], 3),
                "unit": UNIT, "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
                "ms_per_step": round(1e3 / res["value"], 3), "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": INDEXER_DATA,
                "config": indexer_config(w, world), "impl": "reference", "cpu_baseline": res,
                "e2e": {"value": round(res["value"], 3), "unit": UNIT, "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}}
    w = workloads.WORKLOADS[args.workload]()
    seconds = max(2.0, args.cpu_seconds)
    t_all = time.perf_counter()
    res = cpu_baseline(w, seconds)
    value = res["value"]
    return {
        "metric": METRIC, "value": round(value, 3), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(w.B * w.T / value * 1e3, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": data_note(w),
        "config": bench_config(w, args.workload, args.nsplit, world),
        "impl": "reference",
        "cpu_baseline": res,
        "e2e": {"value": round(value, 3), "unit": UNIT, "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
        "wall_s": round(time.perf_counter() - t_all, 2),
    }


def main(argv=None):
    args = parse_args(argv)
    if args.impl == "reference":
        # The CPU oracle as the reference arm: rank 0 alone runs and prints;
        # under torchrun the other ranks exit at once, with no process group.
        rank = int(os.environ.get("RANK", "0"))
        world = int(os.environ.get("WORLD_SIZE", "1"))
        line = run_reference(args, world, rank) if rank == 0 else None
        if line is not None:
            print(json.dumps(line), flush=True)
        return 0
    world, rank, local = dist_init()
    line = run_ours(args, world, rank, local)
    if rank == 0 and line is not None and args.workload != "indexer_mixed":
        from sparse_mla_decode_partial_b200 import workloads
        line["cpu_baseline"] = cpu_baseline(workloads.WORKLOADS[args.workload](),
                                            args.cpu_seconds)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0 and line is not None:
        print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
