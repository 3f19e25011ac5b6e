"""Multi-rank host logic of bench.py on CPU: two gloo ranks (world_size 2).

The decode path shards into independent query tokens with no exchange step,
so N GPUs run N independent replicas; the only cross-rank traffic is the
benchmark's own bookkeeping (max of step times, sum of tokens, barriers).
These tests run that bookkeeping over gloo with no GPU.
"""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    w, r, _ = bench.dist_init()
    assert (w, r) == (world, rank)
    wl = bench.replica_workload("tiny", rank, world)
    # rank-dependent step times: the job is as slow as its slowest rank
    ms_local = 1.0 + rank
    tokens_all, ms_max, value = bench.aggregate(float(wl.B * wl.T), ms_local, world)
    bench.barrier(world)
    digest = float(wl.q.float().sum())
    with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
        json.dump({"tokens_all": tokens_all, "ms_max": ms_max, "value": value,
                   "digest": digest, "idx_first": int(wl.idx[0, 0, 0])}, f)
    import torch.distributed as dist
    dist.destroy_process_group()


def test_two_gloo_ranks_aggregate_weak_scaling(tmp_path):
    port = free_port()
    mp.start_processes(_rank_main, args=(2, port, str(tmp_path)), nprocs=2, join=True,
                       start_method="spawn")
    r0 = json.load(open(tmp_path / "rank0.json"))
    r1 = json.load(open(tmp_path / "rank1.json"))
    for r in (r0, r1):
        assert r["tokens_all"] == 2.0            # one query token per tiny replica
        assert r["ms_max"] == 2.0                # max over ranks, not the local time
        assert abs(r["value"] - 2.0 / 2e-3) < 1e-6
    assert r0["digest"] != r1["digest"]          # independent replicas (own seeds)


def test_single_rank_replica_is_the_canonical_workload():
    sys.path.insert(0, ROOT)
    import bench
    from sparse_mla_decode_partial_b200 import workloads
    a = bench.replica_workload("tiny", 0, 1)
    b = workloads.tiny()
    assert torch.equal(a.q, b.q) and torch.equal(a.idx, b.idx)
    tokens_all, ms_max, value = bench.aggregate(1.0, 4.0, 1)
    assert (tokens_all, ms_max) == (1.0, 4.0) and abs(value - 250.0) < 1e-9


def test_reference_arm_other_ranks_exit_without_work():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1", MASTER_ADDR="127.0.0.1",
               MASTER_PORT=str(free_port()))
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference"],
                       env=env, capture_output=True, text=True, timeout=120)
    assert r.returncode == 0 and r.stdout.strip() == ""


def test_reference_arm_rank0_prints_one_line():
    env = dict(os.environ, RANK="0", WORLD_SIZE="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--workload", "tiny", "--cpu-seconds", "0.5"],
                       env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    lines = [l for l in r.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["cpu_baseline"]["kind"] == "oracle"
    assert d["unit"] == "query-tokens/s" and d["value"] > 0
    assert d["e2e"]["h2d_bytes_per_step"] == 0


def test_dense_replicas_keep_the_shape_and_change_the_data():
    """Weak scaling for the dense verify workload: each rank's replica has the
    same shape and visible lengths (the same work) with its own data."""
    sys.path.insert(0, ROOT)
    import bench
    r0 = bench.replica_workload("dense_verify", 0, 2)
    r1 = bench.replica_workload("dense_verify", 1, 2)
    assert r0.dense and r1.dense
    assert r0.q.shape == r1.q.shape and r0.cache.shape == r1.cache.shape
    assert torch.equal(r0.seq_lens, r1.seq_lens)
    assert not torch.equal(r0.q, r1.q)
    assert bench.workload_bytes(r0) == bench.workload_bytes(r1)


def test_reference_arm_dense_workload(tmp_path):
    env = dict(os.environ, RANK="0", WORLD_SIZE="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--workload", "dense_verify", "--cpu-seconds", "0.5"],
                       env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    d = json.loads([l for l in r.stdout.splitlines() if l.strip()][0])
    assert d["impl"] == "reference" and d["config"]["workload"] == "dense_verify"
    assert "dense" in d["cpu_baseline"]["sample"] and d["value"] > 0


def test_traffic_record_tracks_its_kernel_sources(tmp_path, monkeypatch):
    """roofline.traffic is reported only while the captured kernel's own source
    files are unchanged (comments aside): editing the tcgen05 kernel's code
    drops the tcgen05 figures and keeps the others."""
    import shutil
    sys.path.insert(0, ROOT)
    import bench
    csrc = os.path.join("sparse_mla_decode_partial_b200", "csrc")
    shutil.copytree(os.path.join(ROOT, csrc), tmp_path / csrc)
    (tmp_path / "profiles").mkdir()
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    # a record taken on the sources as they are now
    kernels = {"single_request": "smla_partial_small_kernel", "batched": "smla_partial_mma_kernel",
               "mixed": "smla_partial_tc_kernel"}
    rec = {wl: {"kernel": k, "sources_sha256_16": bench.kernel_sources_hash(k),
                "traffic_bytes_per_launch": 1000 + i} for i, (wl, k) in enumerate(kernels.items())}
    (tmp_path / "profiles" / "ncu_traffic.json").write_text(json.dumps(rec))
    before = {wl: bench.measured_traffic(wl) for wl in kernels}
    assert before == {"single_request": 1000, "batched": 1001, "mixed": 1002}
    tc = tmp_path / csrc / "smla_partial_tc.cuh"
    tc.write_text(tc.read_text() + "\n// a comment edit does not change the kernel\n")
    assert bench.measured_traffic("mixed") == before["mixed"]
    tc.write_text(tc.read_text() + "\nstatic_assert(true, \"a code edit\");\n")
    assert bench.measured_traffic("mixed") is None
    assert bench.measured_traffic("single_request") == before["single_request"]
    assert bench.measured_traffic("batched") == before["batched"]
    assert bench.measured_traffic("tiny") is None          # never captured


class _FakeNvml:
    """Stands in for pynvml: a fixed SM clock and throttle-reason mask; while
    `failing` is set the per-sample queries raise, as a busy driver can."""
    NVML_CLOCK_SM = 1

    def __init__(self, mhz, reasons):
        self.mhz, self.mask, self.failing, self.calls = mhz, reasons, False, []

    def nvmlInit(self):
        self.calls.append("init")

    def nvmlDeviceGetHandleByIndex(self, i):
        return ("dev", i)

    def nvmlDeviceGetMaxClockInfo(self, h, kind):
        return 1965

    def nvmlDeviceGetClockInfo(self, h, kind):
        self.calls.append("clock")
        if self.failing:
            raise RuntimeError("busy")
        return self.mhz

    def nvmlDeviceGetCurrentClocksEventReasons(self, h):
        self.calls.append("reasons")
        if self.failing:
            raise RuntimeError("busy")
        return self.mask


def test_clock_sampler_reads_inside_the_region_and_names_reasons(monkeypatch):
    """The sampler's first NVML queries run when it is made (before the timed
    region); inside the region it samples the SM clock and ORs the throttle
    reasons, which it names."""
    import time
    sys.path.insert(0, ROOT)
    import bench
    fake = _FakeNvml(1800, bench.ClockSampler.HW["sw_power_cap"] | bench.ClockSampler.HW["hw_slowdown"])
    monkeypatch.setitem(sys.modules, "pynvml", fake)
    s = bench.ClockSampler(0, period_s=0.001)
    assert fake.calls[:3] == ["init", "clock", "reasons"]
    n_before = len(fake.calls)
    with s:
        t0 = time.monotonic()
        while len(s.samples) < 2 and time.monotonic() - t0 < 10.0:
            time.sleep(0.005)
    assert len(fake.calls) > n_before
    out = s.summary()
    assert out["sm_mhz"] == 1800 and out["sm_max_mhz"] == 1965 and out["samples"] >= 2
    assert sorted(out["reasons"]) == ["hw_slowdown", "sw_power_cap"]
    assert "sampled" not in out


def test_clock_sampler_flags_a_read_taken_after_the_region(monkeypatch):
    """When no sample lands inside the region, the one read taken right after
    it is reported as such, never as a sample from inside."""
    import time
    sys.path.insert(0, ROOT)
    import bench
    fake = _FakeNvml(1965, 0)
    monkeypatch.setitem(sys.modules, "pynvml", fake)
    s = bench.ClockSampler(0, period_s=0.001)
    fake.failing = True
    with s:
        time.sleep(0.01)
        s._stop.set()             # the region's sampling ends with nothing read
        s._thread.join()
        fake.failing = False      # the driver answers again only after it
    out = s.summary()
    assert out["samples"] == 1 and out["sm_mhz"] == 1965 and out["reasons"] == []
    assert out["sampled"].startswith("once, right after the timed region")


def test_reference_arm_indexer_workload_prints_the_same_config():
    """The indexer's reference line carries the config and data note the
    GPU arm prints for the same command (one helper builds both)."""
    sys.path.insert(0, ROOT)
    import bench
    from sparse_mla_decode_partial_b200 import workloads
    env = dict(os.environ, RANK="0", WORLD_SIZE="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--workload", "indexer_mixed", "--cpu-seconds", "0.5"],
                       env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    d = json.loads([l for l in r.stdout.splitlines() if l.strip()][0])
    w = workloads.indexer_mixed()
    assert d["impl"] == "reference" and d["config"] == bench.indexer_config(w, 1)
    assert d["data"] == bench.INDEXER_DATA and d["value"] > 0
    assert d["config"]["shape"].startswith(f"B{w.B} T{w.T} HI{w.HI} ")
    assert bench.indexer_config(w, 4)["parallelism"] == "replicas x4"


def test_indexer_headline_reports_the_job_from_the_timed_record(monkeypatch):
    """The indexer line's value is query tokens over the timed call's
    duration, with the shared config (timing faked: the record the timed
    region produces is given, CUDA calls are stubbed)."""
    sys.path.insert(0, ROOT)
    import bench
    from sparse_mla_decode_partial_b200 import build, workloads
    w = workloads.indexer_mixed()
    rec = {"shape": bench.indexer_shape(w), "query_tokens": w.B * w.T, "us_per_call": 100.0,
           "roofline": {"frac": 0.8}, "clocks": {"sm_mhz": 1965}, "gpu_launches": 40}
    monkeypatch.setattr(build, "build", lambda: None)
    monkeypatch.setattr(bench, "Harness", lambda dev: None)
    monkeypatch.setattr(bench, "side_indexer", lambda h, steps, warmup, peaks: rec)
    monkeypatch.setattr(torch.cuda, "set_device", lambda dev: None)
    monkeypatch.setattr(torch.cuda, "synchronize", lambda dev=None: None)

    class A:
        steps, warmup = 10, 3
    line = bench.run_indexer_headline(A(), 1, 0, 0)
    assert line["value"] == round(w.B * w.T / 100e-6, 1) and line["ms_per_step"] == 0.1
    assert line["config"] == bench.indexer_config(w, 1) and line["data"] == bench.INDEXER_DATA
    assert line["n_gpus"] == 1 and line["indexer"] is rec


def test_side_indexer_record_from_fixed_timings(monkeypatch):
    """The indexer record of the default bench line, built from fixed step
    times (the harness is a stand-in: every call returns status 0, every
    timed loop reports 100 / 75 / 30 us per step), so its arithmetic can be
    checked without a GPU."""
    sys.path.insert(0, ROOT)
    import types
    import bench
    from sparse_mla_decode_partial_b200 import workloads

    calls = []

    class FakeLib:
        def __getattr__(self, name):
            def fn(*args):
                calls.append(name)
                return 0
            return fn

    per_step = {"topk": 0.100, "scores": 0.075, "select": 0.030}

    class FakeHarness:
        dev = torch.device("cpu")
        lib, sptr = FakeLib(), 0

        def warm(self, fns, n):
            for f in fns:
                assert f()[0] == 0

        def timed(self, step, n):
            st, nl = step()
            return [per_step[step.__name__]] * n, nl * n

    monkeypatch.setattr(torch.cuda, "empty_cache", lambda: None)
    rec = bench.side_indexer(FakeHarness(), 10, 3, (6650.0, 1590.0, "fallback"))
    w = workloads.indexer_mixed()
    key_bytes = bench.indexer_bytes(w) - w.B * w.T * w.K * 4
    assert rec["shape"] == bench.indexer_shape(w) and rec["query_tokens"] == w.B * w.T
    assert rec["us_per_call"] == 100.0 and rec["scores_us"] == 75.0 and rec["select_us"] == 30.0
    assert rec["q_tok_s"] == round(w.B * w.T / 100e-6, 1)
    r = rec["roofline"]
    assert r["kernel"] == "smla_ix_score_kernel" and r["algorithmic_bytes_per_launch"] == key_bytes
    assert r["achieved"] == round(key_bytes / 75e-6 / 1e9, 1)
    assert r["frac"] == round(key_bytes / 75e-6 / 1e9 / 6650.0, 4)
    assert rec["gpu_launches"] == 40                      # 10 top-k calls x 4 kernels
    assert {"smla_indexer_topk", "smla_indexer_scores", "smla_indexer_select"} <= set(calls)
