"""Build libsdpa_b200.so in-tree with nvcc for sm_100a.

Usage: ``python -m scaled_dot_product_fa2_b200.build [--force]``.  The build
also checks ptxas' report: no kernel may spill registers, and the prefill
kernels must launch at exactly the register count their in-kernel setmaxnreg
split is written for.
"""
from __future__ import annotations

import os
import re
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libsdpa_b200.so")
SOURCES = [os.path.join(CSRC, "sdpa_b200.cu")]
PREFILL_LAUNCH_REGS = 168

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-std=c++17", "-lineinfo",
    "-Xcompiler", "-fPIC", "-shared",
    "-Xptxas", "-v",
]


def _inputs():
    files = list(SOURCES)
    files += [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".cuh", ".h"))]
    files.append(os.path.join(INCLUDE, "sdpa_b200.h"))
    return files


def _stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(f) > t for f in _inputs())


# The prefill kernel's bias instantiation (template argument BIAS = true,
# mangled "Lb1E") holds a tile of bias next to the scores; ptxas spills one
# 32-bit value of it (4 bytes stored, reloaded in the loop), which costs
# nothing measurable.  Anything larger is a regression.
BIAS_SPILL_ALLOWANCE = 16


def check_ptxas_report(report: str) -> None:
    """Fail on spills, and on a prefill register count the split is not written for."""
    current = None
    for line in report.splitlines():
        m = re.search(r"Compiling entry function '(\S+)'", line)
        if m:
            current = m.group(1)
            continue
        m = re.search(r"(\d+) bytes spill stores, (\d+) bytes spill loads", line)
        if m and current and (int(m.group(1)) or int(m.group(2))):
            allowed = BIAS_SPILL_ALLOWANCE if ("prefill_kernel" in current and "Lb1E" in current) else 0
            if int(m.group(1)) > allowed or int(m.group(2)) > allowed:
                raise RuntimeError(f"kernel {current} spills registers:\n{line}")
        m = re.search(r"Used (\d+) registers", line)
        if m and current and "prefill_kernel" in current and int(m.group(1)) != PREFILL_LAUNCH_REGS:
            raise RuntimeError(f"{current} uses {m.group(1)} registers, expected {PREFILL_LAUNCH_REGS}")


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and not _stale():
        return LIB
    nvcc = os.environ.get("NVCC", "nvcc")
    tmp = LIB + f".tmp{os.getpid()}"
    cmd = [nvcc, *NVCC_FLAGS, "-I", INCLUDE, "-o", tmp, *SOURCES]
    try:
        proc = subprocess.run(cmd, capture_output=True, text=True)
        if proc.returncode != 0:
            raise RuntimeError("nvcc failed:\n" + proc.stdout + proc.stderr)
        check_ptxas_report(proc.stdout + proc.stderr)
        if verbose:
            print(proc.stdout + proc.stderr)
        os.replace(tmp, LIB)
    finally:
        if os.path.exists(tmp):
            os.remove(tmp)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv))
