"""Throughput of the fused exact-attention forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

A step is one attn_fwd over the whole workload: B=8, H=32, N=8192, d=128,
causal, bf16 Q/K/V drawn N(0,1) from a fixed seed (the batch/head/length of
the score-matrix memory example on the anylearn.cc page "Attention Is
Memory-Bound, and Nobody Noticed for Five Years"). Metric: TFLOP/s with
4*B*H*N^2*d FLOPs per step, halved for causal.

With N > 1 (torchrun, one process per GPU) each rank runs its own copy of the
workload: the (batch, head) units are independent, so there is no
data-path collective ("weak" scaling); the barrier and the max-over-ranks of
the device time are measurement only.

Prints one JSON line on rank 0. `--impl reference` times the fp64 CPU oracle
on a bounded sample of the same workload instead (CPU only).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import re
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

WORKLOAD = "long_8192_causal"
METRIC = "attn fwd TFLOP/s (causal-adjusted) and % of B200 dense BF16 peak"
PROFILE_SUMMARY = os.path.join(ROOT, "profiles", "fused_attn_fwd_long_8192_causal.txt")
KV_PROFILE_SUMMARY = os.path.join(ROOT, "profiles", "fused_attn_fwd_kv_decode.txt")
# the sources that define the fused kernel; the ncu summary records their hash
KERNEL_SOURCES = [os.path.join(ROOT, "exact_attention_125_b200", "csrc", f)
                  for f in ("fused_fwd.cu", "sm100.cuh", "tmem_io.cuh", "watchdog.cuh",
                            "exp2_poly.cuh", "fp8.cuh")]
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
HBM_DATASHEET_GBS = 7700.0  # B200 HBM3e, HGX figure (context for fractions above the copy peak)


def parse_args(argv=None):
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=20)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--workload", default=WORKLOAD)
    p.add_argument("--e2e-steps", type=int, default=6)
    p.add_argument("--no-naive", action="store_true", help="skip the unfused traffic line")
    p.add_argument("--no-kv", action="store_true", help="skip the split-KV inference lines")
    p.add_argument("--no-ext", action="store_true", help="skip the window / distance-bias lines")
    p.add_argument("--no-chain", action="store_true", help="skip the elementwise-chain line")
    p.add_argument("--no-fp8", action="store_true", help="skip the FP8 line")
    p.add_argument("--traffic-sweep", action="store_true",
                   help="one fused and one unfused launch per sequence length (B*H*N fixed, "
                        "inputs above L2) for an ncu DRAM-bytes capture; prints the algorithmic "
                        "bytes of each kernel")
    p.add_argument("--profile-case", default=None, metavar="WORKLOAD",
                   help="run attn_fwd on this square workload --warmup + --steps times and "
                        "exit (a profiler capture target; prints nothing timed)")
    p.add_argument("--no-square", action="store_true",
                   help="skip the other square workloads and the host-overhead line")
    p.add_argument("--kv-only", default=None, metavar="WORKLOAD",
                   help="run only the split-KV line of this inference workload (one GPU)")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--cpu-seconds", type=float, default=15.0,
                   help="target CPU time of the oracle sample")
    return p.parse_args(argv)


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def _code_only(text: str) -> str:
    """C++ source without its comments and trailing blanks: what the compiler
    turns into code (string literals in these sources hold no comment
    markers)."""
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    text = re.sub(r"//[^\n]*", "", text)
    return "\n".join(line.rstrip() for line in text.splitlines() if line.strip())


def source_hash(paths=None) -> str:
    """Hash of the kernel sources' code (comments left out), which gates the
    committed ncu traffic figures: a comment edit leaves them valid, any code
    edit voids them."""
    h = hashlib.sha256()
    for path in (paths or KERNEL_SOURCES):
        with open(path, encoding="utf-8") as f:
            h.update(_code_only(f.read()).encode())
    return h.hexdigest()[:16]


def _summary_fields(path):
    """key: value lines of a committed ncu summary, or None when it is missing
    or was taken on another kernel source."""
    if not os.path.exists(path):
        return None
    fields = {}
    for line in open(path):
        if ":" in line and not line.startswith("#"):
            k, v = line.split(":", 1)
            fields[k.strip()] = v.strip()
    if fields.get("kernel_source_sha256_16") != source_hash():
        return None
    return fields


def profiled_traffic(workload: str = WORKLOAD):
    """DRAM bytes per launch of the fused kernel from the committed ncu summary
    (taken on long_8192_causal; None for any other workload)."""
    fields = _summary_fields(PROFILE_SUMMARY)
    if not fields or fields.get("workload", WORKLOAD) != workload:
        return None
    try:
        return float(fields["dram_bytes_per_launch_full_workload"])
    except (KeyError, ValueError):
        return None


def profiled_kv_traffic(w):
    """DRAM bytes per launch of the split-KV kernel on a decode workload: the
    capture's reads scaled by the key count (every K/V byte is read once, so
    reads grow with Nk), plus its writes. None for other shapes."""
    fields = _summary_fields(KV_PROFILE_SUMMARY)
    if not fields or w.Nq != 1 or w.causal:
        return None
    from exact_attention_125_b200.inputs import KV_WORKLOADS
    base = KV_WORKLOADS.get(fields.get("workload", ""))
    if base is None or (base.B, base.H, base.Nq, base.d) != (w.B, w.H, w.Nq, w.d):
        return None
    try:
        reads = float(fields["dram_bytes_read_per_launch"])
        writes = float(fields["dram_bytes_write_per_launch"])
    except (KeyError, ValueError):
        return None
    return reads * w.Nk / base.Nk + writes


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """SM clock, power and clock-event reasons sampled every 5 ms by an NVML
    thread while the timed region runs (a 20-step region lasts ~70 ms, too
    short for nvidia-smi's 200 ms loop). Falls back to nvidia-smi at its
    shortest interval when NVML cannot be loaded. Reads settings only."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    PERIOD_S = 0.005

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None
        self.thread = None
        self.rows = []
        self.source = None

    def _nvml_handle(self):
        import pynvml
        pynvml.nvmlInit()
        try:
            import torch
            uuid = str(torch.cuda.get_device_properties(self.gpu).uuid)
            return pynvml, pynvml.nvmlDeviceGetHandleByUUID(
                uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
        except Exception:  # noqa: BLE001 - any lookup failure: fall back to the index
            return pynvml, pynvml.nvmlDeviceGetHandleByIndex(self.gpu)

    def _nvml_sample(self):
        nv, h = self.nv, self.handle
        bits = [nv.nvmlClocksEventReasonHwSlowdown, nv.nvmlClocksEventReasonHwThermalSlowdown,
                nv.nvmlClocksEventReasonSwThermalSlowdown, nv.nvmlClocksEventReasonSwPowerCap]
        try:
            sm = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
            r = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
        except Exception:  # noqa: BLE001 - a failed read is skipped
            return
        try:
            watts = f"{nv.nvmlDeviceGetPowerUsage(h) / 1000:.1f}"
        except Exception:  # noqa: BLE001 - power is optional
            watts = "n/a"
        self.rows.append([str(self.gpu), str(sm), str(self.sm_max), watts, hex(r)]
                         + ["Active" if r & b else "Not Active" for b in bits])

    def _nvml_loop(self, stop):
        while not stop.wait(self.PERIOD_S):
            self._nvml_sample()

    def __enter__(self):
        import threading
        try:
            self.nv, self.handle = self._nvml_handle()
            self.sm_max = self.nv.nvmlDeviceGetMaxClockInfo(self.handle, self.nv.NVML_CLOCK_SM)
            self._nvml_sample()  # one sample as the timed region starts, whatever the thread does
            self.stop = threading.Event()
            self.thread = threading.Thread(target=self._nvml_loop, args=(self.stop,), daemon=True)
            self.thread.start()
            self.source = f"nvml every {self.PERIOD_S * 1e3:.0f} ms"
            return self
        except Exception:  # noqa: BLE001 - no NVML: nvidia-smi below
            self.thread = None
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "20"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
            self.source = "nvidia-smi every 20 ms"
        except (OSError, FileNotFoundError):
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        if self.thread is not None:
            self.stop.set()
            self.thread.join(timeout=5)
            self._nvml_sample()  # and one as it ends
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        rows = list(self.rows)
        if self.path and os.path.exists(self.path):
            for line in open(self.path):
                parts = [x.strip() for x in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
            os.unlink(self.path)
        out = summarize_clocks(rows)
        out["source"] = self.source
        return out


def summarize_clocks(rows):
    if not rows:
        return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
    def num(x):
        try:
            return float(x)
        except ValueError:
            return None
    sm = [num(r[1]) for r in rows if num(r[1]) is not None]
    mx = [num(r[2]) for r in rows if num(r[2]) is not None]
    names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
    reasons = set()
    for r in rows:
        for name, val in zip(names, r[5:9]):
            if val.strip().lower() == "active":
                reasons.add(name)
    watts = [num(r[3]) for r in rows if num(r[3]) is not None]
    masks = sorted({r[4] for r in rows if r[4].startswith("0x")})
    return {"sm_mhz": statistics.median(sm) if sm else None,
            "sm_max_mhz": max(mx) if mx else None,
            "sm_mhz_min": min(sm) if sm else None,
            "power_w_median": statistics.median(watts) if watts else None,
            "reason_masks": masks,
            "reasons": sorted(reasons), "samples": len(rows)}


# ------------------------------------------------------------- distributed
def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def init_dist(world, backend):
    import datetime

    import torch.distributed as dist
    if world > 1 and not dist.is_initialized():
        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return dist if world > 1 else None


def max_over_ranks(x: float, dist, device) -> float:
    if dist is None:
        return x
    import torch
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_tflops(flops_per_rank_step: float, world: int, steps: int, ms_max: float) -> float:
    """Whole-job throughput: every rank processes its own copy of the workload
    each step (weak scaling), timed as the slowest rank's device time."""
    return flops_per_rank_step * world * steps / (ms_max * 1e-3) / 1e12


def barrier(dist):
    if dist is not None:
        dist.barrier()


# ------------------------------------------------------------ oracle (CPU)
def cpu_oracle_sample(w, target_seconds: float):
    """Times the fp64 oracle on a bounded, seeded sample of the workload's rows.
    Returns (tflops, seconds, rows, cores, sample description)."""
    import numpy as np

    import oracle
    from exact_attention_125_b200.inputs import make_qkv

    # the oracle needs only the sampled heads: draw a 16-head slice with the
    # workload's distribution (same per-row work as any head of the workload)
    heads = 16
    q, k, v = make_qkv(1, heads, w.N, w.d, w.seed, w.dist)
    cores = oracle.default_threads()
    rng = np.random.default_rng(w.seed)

    def rows_for(n):
        flat = np.sort(rng.choice(heads * w.N, size=n, replace=False))
        return np.stack([flat // w.N, flat % w.N], 1).astype(np.int64)

    def flops(rows):
        keys = (rows[:, 1] + 1) if w.causal else np.full(len(rows), w.N)
        return float(4.0 * w.d * keys.sum())

    # two-point calibration: the difference removes the fixed per-call cost
    def timed(n):
        t0 = time.perf_counter()
        oracle.attention(q, k, v, w.scale, w.causal, rows=rows_for(n))
        return time.perf_counter() - t0
    n0 = max(cores, 16)
    t1, t2 = timed(n0), timed(2 * n0)
    per_row = max((t2 - t1) / n0, t2 / (2 * n0) * 0.25, 1e-9)
    n = int(min(heads * w.N, max(2 * n0, target_seconds / per_row)))
    rows = rows_for(n)
    t0 = time.perf_counter()
    oracle.attention(q, k, v, w.scale, w.causal, rows=rows)
    secs = time.perf_counter() - t0
    desc = (f"{n} seeded query rows of {w.name} (B=1 slice of {heads} heads, same N, d, "
            f"causal={w.causal}, distribution {w.dist}); FLOPs counted 4*d*|allowed keys| per row")
    return flops(rows) / secs / 1e12, secs, n, cores, desc


def run_reference(args):
    world, rank, _ = dist_env()
    if rank != 0:
        return 0
    from exact_attention_125_b200.inputs import WORKLOADS
    w = WORKLOADS[args.workload]
    per_step = []
    total_rows = 0
    cores = 0
    desc = ""
    for _ in range(args.warmup):
        cpu_oracle_sample(w, 1.0)
    for _ in range(args.steps):
        tf, secs, n, cores, desc = cpu_oracle_sample(w, max(1.0, args.cpu_seconds / max(args.steps, 1)))
        per_step.append((tf, secs))
        total_rows += n
    tflops = statistics.median(t for t, _ in per_step)
    ms = statistics.median(s for _, s in per_step) * 1e3
    line = {
        "impl": "reference", "metric": METRIC, "value": tflops, "unit": "TFLOP/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": w.name, "B": w.B, "H": w.H, "N": w.N, "d": w.d,
                   "causal": w.causal, "sample": "bounded row sample per step"},
        "cpu_baseline": {"value": tflops, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                         "sample": desc},
        "e2e": {"value": tflops, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }
    print(json.dumps(line), flush=True)
    return 0


# -------------------------------------------------------------- GPU bench
SWEEP_N = (1024, 2048, 4096, 8192)
SWEEP_BHN = 65536  # B*H*N of every sweep case: Q, K, V, O = 67 MB; the naive workspace
                   # 4 B*H*N^2 bytes is 2.1 GB at N = 8192
SWEEP_FLUSH_BYTES = 256 << 20  # written before each measured launch: twice the 126 MB L2


def run_traffic_sweep(args):
    """For each N in SWEEP_N: one attn_fwd and one attn_fwd_naive launch (the
    latter's three kernels) on (B=1, H=SWEEP_BHN/N, N, d=128, causal=False),
    in that order, after one warm-up of each on a separate small input, with
    L2 flushed (a 256 MB buffer written) before each of the two calls so the
    inputs come from HBM. An ncu capture of this run (DRAM bytes per launch)
    shows how each path's traffic grows with N; this prints the algorithmic
    bytes to compare with."""
    import torch

    import exact_attention_125_b200 as ea
    from exact_attention_125_b200 import costs
    device = torch.device("cuda", 0)
    torch.cuda.set_device(device)
    d = 128
    wq = torch.randn((1, 1, 256, d), device=device, dtype=torch.bfloat16)
    ea.attn_fwd(wq, wq, wq)
    ea.attn_fwd_naive(wq, wq, wq)
    flush = torch.empty((SWEEP_FLUSH_BYTES,), dtype=torch.uint8, device=device)
    torch.cuda.synchronize(device)
    rows = []
    for N in SWEEP_N:
        H = SWEEP_BHN // N
        g = torch.Generator(device=device).manual_seed(N)
        q, k, v = (torch.randn((1, H, N, d), device=device, generator=g).to(torch.bfloat16)
                   for _ in range(3))
        ws = torch.empty((ea.naive_workspace_bytes(1, H, N),), dtype=torch.uint8, device=device)
        flush.fill_(1)
        ea.attn_fwd(q, k, v, scale=1.0 / math.sqrt(d), causal=False)
        flush.fill_(2)
        ea.attn_fwd_naive(q, k, v, scale=1.0 / math.sqrt(d), causal=False, workspace=ws)
        torch.cuda.synchronize(device)
        if ea.last_device_error() != 0:
            raise SystemExit(f"device watchdog fired in the sweep at N={N}")
        rows.append({"N": N, "H": H, "fused_bytes": costs.fused_bytes(1, H, N, d),
                     "naive_kernel_bytes": costs.naive_kernel_bytes(1, H, N, d),
                     "naive_bytes": costs.naive_bytes(1, H, N, d)})
        del q, k, v, ws
        torch.cuda.empty_cache()
    # the BERT-base-shaped workload (1, 12, 1024, 64): its S and P (25 MB each)
    # fit in L2, so the unfused path's intermediates need not reach HBM at all
    from exact_attention_125_b200.inputs import WORKLOADS, make_workload
    w = WORKLOADS["bert_base_1024"]
    q, k, v = (t.to(device) for t in make_workload(w))
    ws = torch.empty((ea.naive_workspace_bytes(w.B, w.H, w.N),), dtype=torch.uint8, device=device)
    flush.fill_(3)
    ea.attn_fwd(q, k, v, scale=w.scale, causal=w.causal)
    flush.fill_(4)
    ea.attn_fwd_naive(q, k, v, scale=w.scale, causal=w.causal, workspace=ws)
    torch.cuda.synchronize(device)
    bert = {"workload": w.name, "B": w.B, "H": w.H, "N": w.N, "d": w.d,
            "fused_bytes": costs.fused_bytes(w.B, w.H, w.N, w.d),
            "naive_kernel_bytes": costs.naive_kernel_bytes(w.B, w.H, w.N, w.d),
            "naive_bytes": costs.naive_bytes(w.B, w.H, w.N, w.d)}
    print(json.dumps({"traffic_sweep": rows, "d": d, "causal": False, "bert_base": bert,
                      "launch_order": "per N: fused_attn_fwd_kernel, then the three naive kernels; "
                                      "then the same for bert_base_1024"}),
          flush=True)
    return 0


def run_profile_case(args):
    """attn_fwd on one square workload, warmup + steps launches, for ncu."""
    import torch

    import exact_attention_125_b200 as ea
    from exact_attention_125_b200.inputs import WORKLOADS, make_workload
    w = WORKLOADS[args.profile_case]
    device = torch.device("cuda", 0)
    torch.cuda.set_device(device)
    q, k, v = (t.to(device) for t in make_workload(w))
    o = torch.empty_like(q)
    lse = torch.empty((w.B, w.H, w.N), dtype=torch.float32, device=device)
    for _ in range(args.warmup + args.steps):
        ea.attn_fwd(q, k, v, o, lse, scale=w.scale, causal=w.causal)
    torch.cuda.synchronize(device)
    if ea.last_device_error() != 0:
        raise SystemExit("device watchdog fired")
    print(json.dumps({"profile_case": w.name, "launches": args.warmup + args.steps}), flush=True)
    return 0


def run_ours(args):
    import torch

    import exact_attention_125_b200 as ea
    from exact_attention_125_b200 import costs
    from exact_attention_125_b200.inputs import WORKLOADS, make_workload

    world, rank, local = dist_env()
    if args.traffic_sweep:
        return run_traffic_sweep(args)
    if args.profile_case:
        return run_profile_case(args)
    if args.kv_only:
        torch.cuda.set_device(local)
        peaks, _ = load_peaks()
        line = split_kv_line(args.kv_only, torch.device("cuda", local), peaks,
                             steps=args.steps, warmup=args.warmup)
        print(json.dumps({"split_kv": line}), flush=True)
        return 0
    if world != args.gpus:
        if not (world == 1 and args.gpus == 1):
            raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}; launch with torchrun")
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    dist = init_dist(world, "nccl")
    w = WORKLOADS[args.workload]
    peaks, peaks_kind = load_peaks()

    # seeded inputs (per-rank seed offset: each rank owns a different batch)
    qh, kh, vh = make_workload(w) if rank == 0 else _rank_inputs(w, rank)
    q, k, v = (t.to(device) for t in (qh, kh, vh))
    o = torch.empty_like(q)
    lse = torch.empty((w.B, w.H, w.N), dtype=torch.float32, device=device)
    stream = torch.cuda.current_stream(device)
    flops = costs.attn_flops(w.B, w.H, w.N, w.d, w.causal)

    def step():
        ea.attn_fwd(q, k, v, o, lse, scale=w.scale, causal=w.causal, stream=stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(device)
    if ea.last_device_error() != 0:
        raise SystemExit("device watchdog fired during warm-up")

    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clocks:
        barrier(dist)
        torch.cuda.synchronize(device)
        marks = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps - 1)]
        start.record(stream)
        for i in range(args.steps):
            step()
            if i + 1 < args.steps:
                marks[i].record(stream)
        end.record(stream)
        torch.cuda.synchronize(device)
        barrier(dist)
    ms_local = start.elapsed_time(end)
    bounds = [start, *marks, end]
    in_order = [a.elapsed_time(b) for a, b in zip(bounds[:-1], bounds[1:])]
    per_step = sorted(in_order)
    ms_total = max_over_ranks(ms_local, dist, device)
    if ea.last_device_error() != 0:
        raise SystemExit("device watchdog fired in the timed region")
    ms_step = ms_total / args.steps
    value = aggregate_tflops(flops, world, args.steps, ms_total)
    launch_tflops = flops / (ms_local / args.steps * 1e-3) / 1e12
    clock_info = clocks.summary()

    e2e = (e2e_through_abi(args, w, qh, kh, vh, device, dist, flops, world)
           if args.e2e_steps > 0 else None)
    naive = None if args.no_naive else naive_line(w, device, peaks)
    split_kv = None if args.no_kv else [split_kv_line(name, device, peaks)
                                       for name in KV_BENCH_WORKLOADS]
    ext = None if args.no_ext else [ext_line(spec, device, peaks) for spec in EXT_BENCH]
    chain = None if args.no_chain else chain_line(device, peaks)
    fp8 = None if args.no_fp8 else fp8_line(w, device, peaks)
    square = None if args.no_square else [square_line(name, device, peaks)
                                          for name in SQUARE_BENCH_WORKLOADS]
    host = None if args.no_square else host_overhead_line(device)

    peak = float(peaks["bf16_tflops"])
    line = {
        "metric": METRIC,
        "value": value,
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms_step,
        "ms_per_step_median_rank0": statistics.median(per_step),
        "ms_per_step_best_rank0": per_step[0],
        "ms_per_step_in_order_rank0": [round(t, 4) for t in in_order],
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": w.name, "B": w.B, "H": w.H, "N": w.N, "d": w.d,
                   "causal": w.causal, "per_rank": "one full copy of the workload",
                   "l2": "inputs larger than L2 (Q, K, V 1.5 GiB per step)",
                   "parallelism": f"replicas x{world}"},
        "pct_of_peak": {
            f"of_{peaks_kind}_burst_{peak:g}": 100.0 * launch_tflops / peak,
            f"of_{peaks_kind}_sustained_{float(peaks['bf16_tflops_sustained']):g}":
                100.0 * launch_tflops / float(peaks["bf16_tflops_sustained"]),
            "of_spec_2250": 100.0 * launch_tflops / 2250.0,
        },
        "roofline": {
            "bound": "tensor",
            "achieved": launch_tflops,
            "peak": peak,
            "unit": "TFLOP/s",
            "frac": launch_tflops / peak,
            "peak_source": f"MEASURED_PEAKS.json bf16_tflops ({peaks_kind}, burst)",
            "traffic": profiled_traffic(w.name),
            "algorithmic_bytes": costs.fused_bytes(w.B, w.H, w.N, w.d),
            "kernel": "fused_attn_fwd_kernel<128, false, false, false, false>",
        },
        "clocks": {k: clock_info.get(k) for k in ("sm_mhz", "sm_max_mhz", "reasons", "sm_mhz_min",
                                                  "power_w_median", "reason_masks", "samples",
                                                  "source")},
        "e2e": e2e,
        "gpu_launches": args.steps,
    }
    if square is not None:
        line["square_workloads"] = square
        line["host_overhead_per_call"] = host
    if naive is not None:
        line["naive"] = naive
    if split_kv is not None:
        line["split_kv"] = split_kv
    if ext is not None:
        line["masks_and_bias"] = ext
    if chain is not None:
        line["elementwise_chain"] = chain
    if fp8 is not None:
        fp8["speedup_over_bf16_line"] = ms_step / fp8["ms_per_step"]
        line["fp8"] = fp8
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        tf, secs, n, cores, desc = cpu_oracle_sample(w, args.cpu_seconds)
        line["cpu_baseline"] = {"value": tf, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                                "sample": desc, "seconds": secs, "rows_per_s": n / secs,
                                "extrapolated_full_workload_s": flops / (tf * 1e12),
                                "extrapolated": True}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.destroy_process_group()
    return 0


def _rank_inputs(w, rank):
    from exact_attention_125_b200.inputs import make_qkv
    return make_qkv(w.B, w.H, w.N, w.d, w.seed + 7919 * rank, w.dist)


def e2e_through_abi(args, w, qh, kh, vh, device, dist, flops, world):
    """Same metric through the C ABI with host buffers: every step copies Q, K, V
    from pinned host memory, runs attn_fwd, and copies O and lse back to pinned
    host memory. Steps are pipelined over two device buffer sets and three
    streams, so one step's upload overlaps the previous step's kernel and
    download (PCIe carries both directions at once); every step still moves
    all of its own inputs and results."""
    import torch

    import exact_attention_125_b200 as ea
    q_h, k_h, v_h = (t.pin_memory() for t in (qh, kh, vh))
    outs_h = [(torch.empty(qh.shape, dtype=torch.bfloat16).pin_memory(),
               torch.empty((w.B, w.H, w.N), dtype=torch.float32).pin_memory()) for _ in range(2)]
    bufs = []
    for _ in range(2):
        q, k, v = (torch.empty_like(t, device=device) for t in (q_h, k_h, v_h))
        bufs.append((q, k, v, torch.empty_like(q),
                     torch.empty((w.B, w.H, w.N), dtype=torch.float32, device=device)))
    s_in, s_run, s_out = (torch.cuda.Stream(device) for _ in range(3))
    ev = lambda: torch.cuda.Event()  # noqa: E731
    uploaded, computed, downloaded = ([ev(), ev()] for _ in range(3))
    started = [False, False]

    def step(i):
        b = i % 2
        q, k, v, o, lse = bufs[b]
        with torch.cuda.stream(s_in):
            if started[b]:
                s_in.wait_event(computed[b])  # the kernel that read this buffer set is done
            for dst, src in ((q, q_h), (k, k_h), (v, v_h)):
                dst.copy_(src, non_blocking=True)
            uploaded[b].record(s_in)
        s_run.wait_event(uploaded[b])
        if started[b]:
            s_run.wait_event(downloaded[b])  # its previous results have left the device
        st = ea.abi.attn_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                             lse.data_ptr(), w.B, w.H, w.N, w.d, w.scale, int(w.causal),
                             s_run.cuda_stream)
        if st != 0:
            raise ea.AttnError(st, "attn_fwd")
        computed[b].record(s_run)
        with torch.cuda.stream(s_out):
            s_out.wait_event(computed[b])
            outs_h[b][0].copy_(o, non_blocking=True)
            outs_h[b][1].copy_(lse, non_blocking=True)
            downloaded[b].record(s_out)
        started[b] = True

    for i in range(2):
        step(i)
    torch.cuda.synchronize(device)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(dist)
    start.record(s_in)
    for i in range(args.e2e_steps):
        step(i)
    for e in downloaded:
        s_out.wait_event(e)
    end.record(s_out)
    torch.cuda.synchronize(device)
    ms = max_over_ranks(start.elapsed_time(end), dist, device)
    h2d = sum(t.numel() * t.element_size() for t in (q_h, k_h, v_h))
    d2h = sum(t.numel() * t.element_size() for t in outs_h[0])
    return {"value": flops * world * args.e2e_steps / (ms * 1e-3) / 1e12, "unit": "TFLOP/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "ms_per_step": ms / args.e2e_steps, "steps": args.e2e_steps,
            "path": "pinned host -> device copy, attn_fwd via the C ABI, device -> pinned host; "
                    "steps pipelined over two buffer sets and three streams"}


def naive_line(w, device, peaks, steps=2):
    """The unfused path on the same workload, heads in groups so the S/P
    workspace stays bounded; reported as achieved HBM GB/s of its algorithmic
    traffic (four crossings of S and P plus Q, K, V, O, lse)."""
    import torch

    import exact_attention_125_b200 as ea
    from exact_attention_125_b200 import costs
    BH = w.B * w.H
    per_head_ws = ea.naive_workspace_bytes(1, 1, w.N)
    free, _ = torch.cuda.mem_get_info(device)
    group = max(1, min(BH, int(min(free * 0.6, 40e9) // per_head_ws)))
    while BH % group:
        group -= 1
    q = torch.randn((BH, w.N, w.d), device=device, dtype=torch.bfloat16)
    k, v = torch.randn_like(q), torch.randn_like(q)
    o = torch.empty_like(q)
    lse = torch.empty((BH, w.N), dtype=torch.float32, device=device)
    ws = torch.empty((per_head_ws * group,), dtype=torch.uint8, device=device)
    stream = torch.cuda.current_stream(device)

    def step():
        for g0 in range(0, BH, group):
            ea.attn_fwd_naive(q[g0:g0 + group].unsqueeze(0), k[g0:g0 + group].unsqueeze(0),
                              v[g0:g0 + group].unsqueeze(0), o[g0:g0 + group].unsqueeze(0),
                              lse[g0:g0 + group].unsqueeze(0), scale=w.scale, causal=w.causal,
                              workspace=ws, stream=stream)

    step()
    torch.cuda.synchronize(device)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record(stream)
    for _ in range(steps):
        step()
    end.record(stream)
    torch.cuda.synchronize(device)
    ms = start.elapsed_time(end) / steps
    nbytes = costs.naive_bytes(w.B, w.H, w.N, w.d)
    gbs = nbytes / (ms * 1e-3) / 1e9
    del ws
    torch.cuda.empty_cache()
    return {"ms_per_step": ms, "algorithmic_bytes": nbytes, "achieved_gbs": gbs,
            "hbm_peak_gbs": float(peaks["hbm_gbs"]), "frac": gbs / float(peaks["hbm_gbs"]),
            "tflops": costs.attn_flops(w.B, w.H, w.N, w.d, w.causal) / (ms * 1e-3) / 1e12,
            "head_group": group, "launches_per_step": 3 * (BH // group)}


# the other square workloads (the parity tests' configurations), each timed by
# itself in a sub-line of the JSON line
SQUARE_BENCH_WORKLOADS = ("single_head_128", "bert_base_1024", "decoder_2048_causal",
                          "stress_65536_causal")


def square_line(name, device, peaks):
    """attn_fwd on one square workload: median and best device time of single
    launches (CUDA events around each), TFLOP/s and the fraction of the bf16
    peak. Small workloads sit in L2 and are launch-latency bound; their step
    count is raised so the timed region spans ~50 ms."""
    import torch

    import exact_attention_125_b200 as ea
    from exact_attention_125_b200 import costs
    from exact_attention_125_b200.inputs import WORKLOADS, make_workload
    w = WORKLOADS[name]
    q, k, v = (t.to(device) for t in make_workload(w))
    o = torch.empty_like(q)
    lse = torch.empty((w.B, w.H, w.N), dtype=torch.float32, device=device)
    stream = torch.cuda.current_stream(device)
    flops = costs.attn_flops(w.B, w.H, w.N, w.d, w.causal)

    def step():
        ea.attn_fwd(q, k, v, o, lse, scale=w.scale, causal=w.causal, stream=stream)

    for _ in range(3):
        step()
    torch.cuda.synchronize(device)
    t0 = time.perf_counter()
    step()
    torch.cuda.synchronize(device)
    est = max(time.perf_counter() - t0, 1e-6)
    steps = int(min(200, max(5, 0.05 / est)))
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(steps + 1)]
    ev[0].record(stream)
    for i in range(steps):
        step()
        ev[i + 1].record(stream)
    torch.cuda.synchronize(device)
    if ea.last_device_error() != 0:
        raise SystemExit(f"device watchdog fired on {name}")
    ts = sorted(a.elapsed_time(b) for a, b in zip(ev[:-1], ev[1:]))
    med = statistics.median(ts)
    peak = float(peaks["bf16_tflops"])
    qkv_bytes = 3 * q.numel() * q.element_size()
    return {"workload": name, "B": w.B, "H": w.H, "N": w.N, "d": w.d, "causal": w.causal,
            "steps": steps, "ms_median": med, "ms_best": ts[0],
            "tflops": flops / (med * 1e-3) / 1e12, "tflops_best": flops / (ts[0] * 1e-3) / 1e12,
            "frac": flops / (med * 1e-3) / 1e12 / peak, "bound": "tensor",
            "l2": "inputs larger than L2" if qkv_bytes > 126e6 else "inputs fit in L2",
            "launches_per_step": 1}


def host_overhead_line(device, n_calls=2000):
    """Host time of one attn_fwd call through the C ABI (argument checks,
    tensor-map encoding, launch), on the smallest workload with the stream
    left to run: the median over calls of the CPU time each call takes."""
    import torch

    import exact_attention_125_b200 as ea
    from exact_attention_125_b200.inputs import WORKLOADS, make_workload
    w = WORKLOADS["single_head_128"]
    q, k, v = (t.to(device) for t in make_workload(w))
    o = torch.empty_like(q)
    lse = torch.empty((w.B, w.H, w.N), dtype=torch.float32, device=device)
    s = torch.cuda.current_stream(device).cuda_stream
    args = (q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), w.B, w.H,
            w.N, w.d, w.scale, int(w.causal), s)
    f = ea.abi.attn_fwd
    for _ in range(20):
        f(*args)
    torch.cuda.synchronize(device)
    ts = []
    for i in range(n_calls):
        t0 = time.perf_counter_ns()
        f(*args)
        ts.append(time.perf_counter_ns() - t0)
        if i % 100 == 99:
            torch.cuda.synchronize(device)
    torch.cuda.synchronize(device)
    ts.sort()
    return {"workload": w.name, "calls": n_calls, "us_median": ts[len(ts) // 2] / 1e3,
            "us_p10": ts[len(ts) // 10] / 1e3, "us_p90": ts[9 * len(ts) // 10] / 1e3,
            "includes": "Python ctypes call, validation, four tensor-map encodings, launch"}


KV_BENCH_WORKLOADS = ("decode_131072", "chunk_128x32768_causal")


def split_kv_line(name, device, peaks, steps=10, warmup=3):
    """attn_fwd_kv on an inference workload with the library's automatic split
    count (inputs larger than L2); reported as achieved HBM GB/s of its
    algorithmic traffic (Q, K, V read once, O and lse written once) and as
    TFLOP/s of the visible (query, key) pairs."""
    import torch

    import exact_attention_125_b200 as ea
    from exact_attention_125_b200 import costs
    from exact_attention_125_b200.inputs import KV_WORKLOADS
    w = KV_WORKLOADS[name]
    g = torch.Generator(device=device).manual_seed(w.seed)
    q = torch.randn((w.B, w.H, w.Nq, w.d), device=device, generator=g).to(torch.bfloat16)
    k = torch.randn((w.B, w.H, w.Nk, w.d), device=device, generator=g).to(torch.bfloat16)
    v = torch.randn((w.B, w.H, w.Nk, w.d), device=device, generator=g).to(torch.bfloat16)
    o = torch.empty_like(q)
    lse = torch.empty((w.B, w.H, w.Nq), dtype=torch.float32, device=device)
    splits = ea.kv_num_splits(w.B, w.H, w.Nq, w.Nk, w.d)
    ws_bytes = ea.kv_workspace_bytes(w.B, w.H, w.Nq, w.Nk, w.d, splits)
    ws = torch.empty((max(ws_bytes, 256),), dtype=torch.uint8, device=device)
    stream = torch.cuda.current_stream(device)

    def step():
        ea.attn_fwd_kv(q, k, v, o, lse, scale=w.scale, causal=w.causal, num_splits=splits,
                       workspace=ws, stream=stream)

    for _ in range(warmup):
        step()
    torch.cuda.synchronize(device)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record(stream)
    for _ in range(steps):
        step()
    end.record(stream)
    torch.cuda.synchronize(device)
    if ea.last_device_error() != 0:
        raise SystemExit(f"device watchdog fired in the split-KV line {name}")
    ms = start.elapsed_time(end) / steps
    nbytes = costs.kv_bytes(w.B, w.H, w.Nq, w.Nk, w.d)
    gbs = nbytes / (ms * 1e-3) / 1e9
    flops = costs.kv_flops(w.B, w.H, w.Nq, w.Nk, w.d, w.causal)
    del q, k, v, ws
    torch.cuda.empty_cache()
    return {"workload": w.name, "B": w.B, "H": w.H, "Nq": w.Nq, "Nk": w.Nk, "d": w.d,
            "causal": w.causal, "num_splits": splits, "ms_per_step": ms, "steps": steps,
            "algorithmic_bytes": nbytes, "achieved_gbs": gbs,
            "hbm_peak_gbs": float(peaks["hbm_gbs"]), "frac": gbs / float(peaks["hbm_gbs"]),
            # the measured peak is a copy (read + write); a read-only stream can
            # beat it, so the fraction is also given against the 7.7 TB/s datasheet
            "frac_of_datasheet_7700": gbs / HBM_DATASHEET_GBS,
            "above_measured_copy_peak": gbs > float(peaks["hbm_gbs"]),
            "bound": "hbm", "traffic": profiled_kv_traffic(w),
            "kernel": "fused_attn_fwd_kernel<128, true, false, true, false>" + (
                " + lse_combine_kernel<128>" if splits > 1 else ""),
            "tflops": flops / (ms * 1e-3) / 1e12,
            "launches_per_step": 2 if splits > 1 else 1,
            "l2": "inputs larger than L2"}


# (name, B, H, Nq, Nk, d, causal, window_left, window_right, distance bias)
EXT_BENCH = (
    ("window_4096_of_32768_causal", 2, 32, 32768, 32768, 128, True, 4095, -1, False),
    ("alibi_8192_causal", 8, 32, 8192, 8192, 128, True, -1, -1, True),
)


def ext_line(spec, device, peaks, steps=5, warmup=3):
    """attn_fwd_ext on a sliding-window or distance-biased shape: TFLOP/s of
    the allowed (query, key) pairs (4 d FLOP each) against the tensor peak."""
    import torch

    import exact_attention_125_b200 as ea
    from exact_attention_125_b200 import costs
    name, B, H, Nq, Nk, d, causal, wl, wr, bias = spec
    g = torch.Generator(device=device).manual_seed(4242)
    q = torch.randn((B, H, Nq, d), device=device, generator=g).to(torch.bfloat16)
    k = torch.randn((B, H, Nk, d), device=device, generator=g).to(torch.bfloat16)
    v = torch.randn((B, H, Nk, d), device=device, generator=g).to(torch.bfloat16)
    o = torch.empty_like(q)
    lse = torch.empty((B, H, Nq), dtype=torch.float32, device=device)
    slopes = (torch.tensor([2.0 ** (-8.0 * (h + 1) / H) for h in range(H)], dtype=torch.float32,
                           device=device) if bias else None)
    splits = ea.ext_num_splits(B, H, Nq, Nk, d, wl)
    ws_bytes = ea.ext_workspace_bytes(B, H, Nq, Nk, d, wl, splits)
    ws = torch.empty((max(ws_bytes, 256),), dtype=torch.uint8, device=device)
    stream = torch.cuda.current_stream(device)

    def step(sl=slopes):
        ea.attn_fwd_ext(q, k, v, o, lse, scale=1.0 / math.sqrt(d), causal=causal, window_left=wl,
                        window_right=wr, alibi_slopes=sl, num_splits=splits, workspace=ws,
                        stream=stream)

    def timed(sl, n):
        start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        start.record(stream)
        for _ in range(n):
            step(sl)
        end.record(stream)
        torch.cuda.synchronize(device)
        return start.elapsed_time(end) / n

    for _ in range(warmup):
        step()
    torch.cuda.synchronize(device)
    ms = timed(slopes, steps)
    # With the bias: the same call without it, timed in alternating samples
    # with the biased call, each after a 1 s idle gap so that both run below
    # the power cap at the same clock; their ratio is the bias's cost.
    same_run = None
    if bias:
        step(None)
        torch.cuda.synchronize(device)

        def gapped(sl):
            time.sleep(1.0)
            return timed(sl, steps)

        pairs = [(gapped(slopes), gapped(None)) for _ in range(3)]
        with_b = statistics.median(a for a, _ in pairs)
        without = statistics.median(b for _, b in pairs)
        same_run = {"ms_with_bias": with_b, "ms_without_bias": without,
                    "with_over_without_throughput": without / with_b,
                    "samples": f"3 alternating pairs of {steps} launches, each after a 1 s idle gap"}
    if ea.last_device_error() != 0:
        raise SystemExit(f"device watchdog fired in the line {name}")
    flops = 4.0 * B * H * d * costs.ext_visible_pairs(Nq, Nk, causal, wl, wr)
    tf = flops / (ms * 1e-3) / 1e12
    del q, k, v, ws
    torch.cuda.empty_cache()
    line = {"workload": name, "B": B, "H": H, "Nq": Nq, "Nk": Nk, "d": d, "causal": causal,
            "window_left": wl, "window_right": wr, "distance_bias": bias, "num_splits": splits,
            "ms_per_step": ms, "steps": steps, "tflops": tf, "bound": "tensor",
            "peak_tflops": float(peaks["bf16_tflops"]), "frac": tf / float(peaks["bf16_tflops"]),
            "kernel": (f"fused_attn_fwd_kernel<128, false, false, {str(bool(bias)).lower()}, "
                       f"{str(wl >= 0 or wr >= 0).lower()}> (square problem, unsplit)"
                       if Nq == Nk and splits == 1
                       else "fused_attn_fwd_kernel<128, true, false, true, false>")}
    if same_run is not None:
        line["against_unbiased_same_run"] = same_run
    return line


def chain_line(device, peaks, rows=65536, cols=8192, steps=10, warmup=3):
    """y = gelu_tanh(0.5 x + b) over a [65536, 8192] bf16 tensor (1 GiB, above L2),
    one fused kernel against three: achieved GB/s of each path's own traffic
    (fused: x read, y written; unfused: three reads and three writes) and the
    time ratio the page predicts to be about 3."""
    import torch

    import exact_attention_125_b200 as ea
    g = torch.Generator(device=device).manual_seed(77)
    x = torch.randn((rows, cols), device=device, generator=g).to(torch.bfloat16)
    b = torch.randn((cols,), device=device, generator=g).to(torch.bfloat16)
    y = torch.empty_like(x)
    tmp = torch.empty_like(x)
    stream = torch.cuda.current_stream(device)
    out = {}
    for name, fn in (("fused", lambda: ea.chain_fused(x, b, y, 0.5, "gelu_tanh", stream)),
                     ("unfused", lambda: ea.chain_unfused(x, b, y, tmp, 0.5, "gelu_tanh", stream))):
        for _ in range(warmup):
            fn()
        torch.cuda.synchronize(device)
        start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        start.record(stream)
        for _ in range(steps):
            fn()
        end.record(stream)
        torch.cuda.synchronize(device)
        ms = start.elapsed_time(end) / steps
        nbytes = (2 if name == "fused" else 6) * rows * cols * 2 + cols * 2
        out[name] = {"ms_per_step": ms, "algorithmic_bytes": nbytes,
                     "achieved_gbs": nbytes / (ms * 1e-3) / 1e9,
                     "frac": nbytes / (ms * 1e-3) / 1e9 / float(peaks["hbm_gbs"]),
                     "launches_per_step": 1 if name == "fused" else 3}
    del x, y, tmp
    torch.cuda.empty_cache()
    return {"workload": f"gelu_tanh(0.5 x + b), x [{rows}, {cols}] bf16", "bound": "hbm",
            "hbm_peak_gbs": float(peaks["hbm_gbs"]), **out,
            "speedup_fused_over_unfused": out["unfused"]["ms_per_step"] / out["fused"]["ms_per_step"],
            "kernel": "chain_pass_kernel"}


def fp8_line(w, device, peaks, steps=10, warmup=3):
    """attn_fwd_fp8 on the headline shape: N(0,1) Q, K, V quantised per tensor
    to E4M3 on the device; TFLOP/s against the FP8 dense peak, taken as the
    measured bf16 burst figure times the nominal FP8 / bf16 ratio of 2."""
    import torch

    import exact_attention_125_b200 as ea
    from exact_attention_125_b200 import costs
    from exact_attention_125_b200.inputs import quantize_e4m3
    g = torch.Generator(device=device).manual_seed(w.seed)
    qkv = [quantize_e4m3(torch.randn(w.shape, device=device, generator=g)) for _ in range(3)]
    (q8, qd), (k8, kd), (v8, vd) = qkv
    o = torch.empty(w.shape, dtype=torch.bfloat16, device=device)
    lse = torch.empty((w.B, w.H, w.N), dtype=torch.float32, device=device)
    stream = torch.cuda.current_stream(device)

    def step():
        ea.attn_fwd_fp8(q8, k8, v8, qd, kd, vd, o, lse, scale=w.scale, causal=w.causal,
                        stream=stream)

    for _ in range(warmup):
        step()
    torch.cuda.synchronize(device)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record(stream)
    for _ in range(steps):
        step()
    end.record(stream)
    torch.cuda.synchronize(device)
    if ea.last_device_error() != 0:
        raise SystemExit("device watchdog fired in the FP8 line")
    ms = start.elapsed_time(end) / steps
    tf = costs.attn_flops(w.B, w.H, w.N, w.d, w.causal) / (ms * 1e-3) / 1e12
    peak = 2.0 * float(peaks["bf16_tflops"])

    # The bf16 kernel on the same shape, alternated with the FP8 one in
    # samples that each follow a 1 s idle gap, so that both run below the
    # power cap at the same clock: the ratio of the two kernels as such.
    qb, kb, vb = (torch.randn(w.shape, device=device, generator=g).to(torch.bfloat16)
                  for _ in range(3))

    def step_bf16():
        ea.attn_fwd(qb, kb, vb, o, lse, scale=w.scale, causal=w.causal, stream=stream)

    def gapped(fn, n=5):
        time.sleep(1.0)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(n):
            fn()
        b.record(stream)
        torch.cuda.synchronize(device)
        return a.elapsed_time(b) / n

    step_bf16()
    pairs = [(gapped(step), gapped(step_bf16)) for _ in range(3)]
    if ea.last_device_error() != 0:
        raise SystemExit("device watchdog fired in the FP8 line")
    ms8 = statistics.median(x for x, _ in pairs)
    ms16 = statistics.median(y for _, y in pairs)
    del q8, k8, v8, qkv, qb, kb, vb
    torch.cuda.empty_cache()
    return {"workload": w.name + " (E4M3 Q, K, V)", "ms_per_step": ms, "steps": steps,
            "tflops": tf, "bound": "tensor", "peak_tflops": peak,
            "peak_source": "2 x MEASURED_PEAKS.json bf16_tflops (nominal FP8 / bf16 ratio)",
            "frac": tf / peak, "speedup_over_bf16_line": None,
            "against_bf16_same_run": {
                "ms_fp8": ms8, "ms_bf16": ms16, "fp8_over_bf16_throughput": ms16 / ms8,
                "samples": "3 alternating pairs of 5 launches, each after a 1 s idle gap"},
            "kernel": "fused_attn_fwd_kernel<128, false, true, false, false>"}


def main(argv=None):
    args = parse_args(argv)
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
