"""Build step for ``libfa_sm100.so`` (nvcc, sm_100a only, in-tree)."""
from __future__ import annotations

import os
import shutil
import subprocess

PKG = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(PKG, "csrc")
ROOT = os.path.dirname(PKG)
LIB = os.path.join(PKG, "libfa_sm100.so")
SOURCES = ["fa_api.cu"]


def headers():
    """Every header under csrc/: a change to any of them rebuilds the library."""
    return sorted(f for f in os.listdir(CSRC) if f.endswith((".cuh", ".h")))
NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-lineinfo", "-O3", "-std=c++17",
    "-Xcompiler", "-fPIC", "-shared",
    "-Xptxas", "-v",
]


def nvcc_path() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _inputs():
    files = [os.path.join(CSRC, f) for f in SOURCES + headers()]
    files.append(os.path.join(ROOT, "include", "fa.h"))
    return files


def up_to_date() -> bool:
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    return all(os.path.getmtime(f) <= t for f in _inputs())


def build(force: bool = False, verbose: bool = False) -> str:
    """Compile the library next to the package; returns its path."""
    if not force and up_to_date():
        return LIB
    tmp = LIB + f".tmp{os.getpid()}"
    cmd = [nvcc_path(), *NVCC_FLAGS, "-I", os.path.join(ROOT, "include"),
           "-o", tmp, *[os.path.join(CSRC, s) for s in SOURCES]]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + res.stdout + res.stderr)
    if verbose:
        print(res.stderr)
    check_register_split(res.stdout + res.stderr)
    os.replace(tmp, LIB)
    return LIB


# The two-Q-tile kernels run 640 threads (96 registers each at launch) and
# redistribute them with setmaxnreg: 4 * 128 * 104 + 128 * 64 = 61440.
SPLIT_THREADS = 640
SPLIT_REQUEST = 4 * 128 * 104 + 128 * 64


def check_register_split(ptxas_log: str) -> None:
    """Refuse a build whose setmaxnreg requests exceed the registers the
    640-thread kernels are launched with: such a request would never be
    granted and the kernel would wait for it forever."""
    import re
    entry, seen = None, 0
    for line in ptxas_log.splitlines():
        m = re.search(r"Compiling entry function '(\S+)'", line)
        if m:
            entry = m.group(1)
            continue
        m = re.search(r"Used (\d+) registers", line)
        if m and entry and re.search(r"fa_fwd_kernelILi\d+ELi2E", entry):
            regs = int(m.group(1))
            if regs * SPLIT_THREADS < SPLIT_REQUEST:
                raise RuntimeError(f"{entry}: {regs} registers x {SPLIT_THREADS} threads < "
                                   f"setmaxnreg requests {SPLIT_REQUEST}")
            seen += 1
    if seen == 0:
        raise RuntimeError("ptxas register report for the two-Q-tile kernels not found")


if __name__ == "__main__":
    print(build(force=True, verbose=True))
