"""Builds libattn_b200.so in-tree with nvcc for sm_100a.

    python -m exact_attention_125_b200._build [--force]
"""
from __future__ import annotations

import glob
import os
import re
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIB = os.path.join(PKG, "libattn_b200.so")
HEADER = os.path.join(ROOT, "include", "attn.h")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-lineinfo", "-O3", "-std=c++17", "--use_fast_math",
    "-Xcompiler", "-fPIC", "-Xcompiler", "-Wall",
    "-shared",
]


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _inputs():
    return sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + \
        glob.glob(os.path.join(CSRC, "*.h")) + [HEADER, __file__]


def up_to_date() -> bool:
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    return all(os.path.getmtime(p) <= t for p in _inputs())


def nvcc() -> str:
    cand = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    return cand if os.path.exists(cand) else "nvcc"


# The fused kernels split the registers of their 384 threads between warp
# roles with setmaxnreg; the split adds up to exactly this launch allocation
# (kRegsAtLaunch in fused_fwd.cu), so a binary with any other count is rejected
# here rather than at run time.
FUSED_KERNEL_REGS = 168
_ENTRY = re.compile(r"Compiling entry function '([^']+)'")
_REGS = re.compile(r"Used (\d+) registers")


def register_counts(ptxas_log: str) -> dict:
    """{mangled kernel name: registers} from `-Xptxas -v` output."""
    counts, current = {}, None
    for line in ptxas_log.splitlines():
        m = _ENTRY.search(line)
        if m:
            current = m.group(1)
            continue
        m = _REGS.search(line)
        if m and current is not None:
            counts[current] = int(m.group(1))
            current = None
    return counts


def check_fused_registers(counts: dict) -> None:
    fused = {k: v for k, v in counts.items() if "fused_attn_fwd" in k}
    if not fused:
        raise RuntimeError("ptxas reported no fused attention kernel")
    bad = {k: v for k, v in fused.items() if v != FUSED_KERNEL_REGS}
    if bad:
        raise RuntimeError(
            f"fused kernels must be allocated exactly {FUSED_KERNEL_REGS} registers per thread "
            f"(their in-kernel register split depends on it); ptxas gave {bad}")


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and up_to_date():
        return LIB
    tmp = LIB + f".tmp{os.getpid()}"
    cmd = [nvcc(), *NVCC_FLAGS, "-Xptxas", "-v", *sources(), "-o", tmp]
    r = subprocess.run(cmd, cwd=CSRC, capture_output=True, text=True)
    log = r.stdout + r.stderr
    if verbose or r.returncode != 0:
        sys.stderr.write(log)
    if r.returncode != 0:
        raise subprocess.CalledProcessError(r.returncode, cmd, r.stdout, r.stderr)
    try:
        check_fused_registers(register_counts(log))
    except RuntimeError:
        os.remove(tmp)
        raise
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
