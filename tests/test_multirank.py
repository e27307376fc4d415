"""The N > 1 plumbing of bench.py on CPU: two ranks over gloo (spawned
processes, 127.0.0.1 rendezvous). Each rank owns a different copy of the
workload (weak scaling, no data-path collective); the only collectives are
the barrier and the max over ranks of the timed duration; the reference arm
prints from rank 0 alone."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world),
                      RANK=str(rank), LOCAL_RANK=str(rank))
    w_, r_, l_ = bench.dist_env()
    dist = bench.init_dist(w_, "gloo")
    bench.barrier(dist)
    slowest = bench.max_over_ranks(10.0 + 5.0 * rank, dist, torch.device("cpu"))
    from exact_attention_125_b200.inputs import WORKLOADS
    q, k, v = bench._rank_inputs(WORKLOADS["single_head_128"], rank)
    out.put((rank, w_, r_, slowest, float(q.float().sum()), float(k.float().sum())))
    bench.barrier(dist)
    dist.destroy_process_group()


def test_two_ranks_share_only_timing():
    ctx = mp.get_context("spawn")
    out = ctx.SimpleQueue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    got = sorted(out.get() for _ in range(2))
    assert [g[0] for g in got] == [0, 1] and all(g[1] == 2 for g in got)
    assert all(g[3] == 15.0 for g in got)          # max over ranks seen by both
    assert got[0][4] != got[1][4] and got[0][5] != got[1][5]  # each rank owns different inputs


def test_aggregate_is_weak_scaling_over_the_slowest_rank():
    one = bench.aggregate_tflops(4.0e12, 1, 10, 20.0)
    assert one == pytest.approx(4.0e12 * 10 / 0.02 / 1e12)
    # two ranks doing the same per-rank work in the same slowest time: twice the throughput
    assert bench.aggregate_tflops(4.0e12, 2, 10, 20.0) == pytest.approx(2 * one)


def test_reference_arm_prints_from_rank_zero_only():
    env = dict(os.environ, WORLD_SIZE="2", RANK="1", LOCAL_RANK="1", MASTER_ADDR="127.0.0.1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--gpus", "2", "--steps", "1", "--warmup", "0"],
                       capture_output=True, text=True, env=env, timeout=300)
    assert r.returncode == 0 and r.stdout.strip() == ""


def test_reference_arm_line_on_rank_zero():
    env = dict(os.environ, WORLD_SIZE="1", RANK="0", LOCAL_RANK="0")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "0", "--cpu-seconds", "1"],
                       capture_output=True, text=True, env=env, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["unit"] == "TFLOP/s" and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["e2e"]["h2d_bytes_per_step"] == 0
    assert line["config"]["workload"] == "long_8192_causal"


def test_profiled_traffic_is_gated_by_source_hash_and_workload(tmp_path, monkeypatch):
    good = tmp_path / "good.txt"
    good.write_text(f"# header\nkernel_source_sha256_16: {bench.source_hash()}\n"
                    "workload: long_8192_causal\ndram_bytes_per_launch_full_workload: 123\n")
    stale = tmp_path / "stale.txt"
    stale.write_text("kernel_source_sha256_16: 0000000000000000\n"
                     "dram_bytes_per_launch_full_workload: 123\n")
    monkeypatch.setattr(bench, "PROFILE_SUMMARY", str(good))
    assert bench.profiled_traffic("long_8192_causal") == 123.0
    assert bench.profiled_traffic("decoder_2048_causal") is None
    monkeypatch.setattr(bench, "PROFILE_SUMMARY", str(stale))
    assert bench.profiled_traffic("long_8192_causal") is None
    monkeypatch.setattr(bench, "PROFILE_SUMMARY", str(tmp_path / "missing.txt"))
    assert bench.profiled_traffic("long_8192_causal") is None


def test_source_hash_follows_code_not_comments(tmp_path):
    src = tmp_path / "k.cu"
    src.write_text("// header\nint f(int x) {  /* doubled */\n  return 2 * x;  // twice\n}\n")
    h0 = bench.source_hash([str(src)])
    src.write_text("// another header\n\nint f(int x) {\n  return 2 * x;\n}\n/* trailing\n   note */\n")
    assert bench.source_hash([str(src)]) == h0  # comments and blank lines only
    src.write_text("int f(int x) {\n  return 3 * x;\n}\n")
    assert bench.source_hash([str(src)]) != h0  # a code edit


def test_bench_arguments_parse():
    a = bench.parse_args(["--gpus", "2", "--steps", "3", "--warmup", "4", "--no-naive",
                          "--no-kv", "--no-ext", "--no-chain", "--no-fp8"])
    assert (a.gpus, a.steps, a.warmup, a.impl) == (2, 3, 4, "ours")
    assert a.no_naive and a.no_kv and a.no_ext and a.no_chain and a.no_fp8
    assert bench.parse_args(["--impl", "reference"]).impl == "reference"


def test_clock_sampler_reads_nvml_inside_the_region(monkeypatch):
    # a fake NVML: the SM clock drops and the power-cap reason appears after
    # a few reads, as under a long load on a 1 kW part
    import sys
    import types
    calls = {"n": 0}
    fake = types.SimpleNamespace(
        NVML_CLOCK_SM=0,
        nvmlClocksEventReasonHwSlowdown=0x8, nvmlClocksEventReasonHwThermalSlowdown=0x40,
        nvmlClocksEventReasonSwThermalSlowdown=0x20, nvmlClocksEventReasonSwPowerCap=0x4,
        nvmlInit=lambda: None,
        nvmlDeviceGetHandleByUUID=lambda uuid: "h",
        nvmlDeviceGetHandleByIndex=lambda i: "h",
        nvmlDeviceGetMaxClockInfo=lambda h, c: 1965)

    def clock(h, c):
        calls["n"] += 1
        return 1965 if calls["n"] < 4 else 1560

    fake.nvmlDeviceGetClockInfo = clock
    fake.nvmlDeviceGetCurrentClocksEventReasons = lambda h: 0x0 if calls["n"] < 4 else 0x4
    fake.nvmlDeviceGetPowerUsage = lambda h: 990000
    monkeypatch.setitem(sys.modules, "pynvml", fake)
    import time
    sampler = bench.ClockSampler(0)
    with sampler:
        time.sleep(0.05)
    s = sampler.summary()
    assert s["samples"] >= 2 and s["source"].startswith("nvml")
    assert s["sm_max_mhz"] == 1965.0 and s["sm_mhz_min"] == 1560.0
    assert "sw_power_cap" in s["reasons"] and "hw_slowdown" not in s["reasons"]
    assert s["power_w_median"] == 990.0
