"""Build the CUDA library libsvdq.so in-tree with nvcc (sm_100a).

    python -m w4a4_rank_absorbed_b200.build [--verbose]

The library is one translation unit (csrc/svdq.cu) holding the three kernels
and the C ABI of include/svdq.h.  It is linked against the static CUDA
runtime; the driver's tensor-map encoder is resolved at run time, so the
build needs no GPU and no libcuda.
"""
from __future__ import annotations

import os
import re
import shutil
import subprocess
import sys

PKG_DIR = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG_DIR)
SRC = os.path.join(PKG_DIR, "csrc", "svdq.cu")
OUT = os.path.join(PKG_DIR, "libsvdq.so")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
# k_linear moves registers between their warpgroups with setmaxnreg; the split adds up to
# 512 threads x 128 registers, so the kernel must be launched with exactly 128 a thread
# (fewer at launch and a warpgroup's setmaxnreg.inc would wait for registers forever).
LINEAR_ENTRY_REGS = 128


def nvcc_path() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def sources():
    csrc = os.path.join(PKG_DIR, "csrc")
    files = [os.path.join(csrc, f) for f in sorted(os.listdir(csrc)) if f.endswith((".cu", ".cuh"))]
    return files + [os.path.join(ROOT, "include", "svdq.h")]


OUT_CHECK = os.path.join(PKG_DIR, "libsvdq_check.so")


def up_to_date(out: str = OUT) -> bool:
    if not os.path.exists(out):
        return False
    t = os.path.getmtime(out)
    return all(os.path.getmtime(f) <= t for f in sources())


def _compile(out: str, extra, verbose: bool) -> str:
    cmd = [nvcc_path(), *ARCH, "-O3", "-std=c++17", "-lineinfo", "-shared", "-Xcompiler", "-fPIC",
           "-Xcompiler", "-fvisibility=hidden", "-Xptxas=-v", *extra, "-o", out + ".tmp", SRC]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + res.stdout + res.stderr)
    if verbose:
        sys.stdout.write(res.stdout + res.stderr)
    for kernel in ("8k_linearILb0E", "8k_linearILb1E"):
        regs = entry_registers(res.stdout + res.stderr, kernel)
        if regs != LINEAR_ENTRY_REGS:
            os.remove(out + ".tmp")
            raise RuntimeError(f"{kernel} compiled to {regs} registers per thread at entry, expected "
                               f"{LINEAR_ENTRY_REGS}: its setmaxnreg split would not add up")
    os.replace(out + ".tmp", out)
    return out


def build(verbose: bool = False, force: bool = False, check: bool = False) -> str:
    """Build libsvdq.so (check=True: the debug build libsvdq_check.so, every copy checked)."""
    out = OUT_CHECK if check else OUT
    if not force and up_to_date(out):
        return out
    return _compile(out, ["-DSVDQ_CHECK"] if check else [], verbose)


def entry_registers(ptxas_log: str, kernel: str) -> int | None:
    """Registers per thread that ptxas reports for the entry function whose name holds `kernel`."""
    lines = ptxas_log.splitlines()
    for i, line in enumerate(lines):
        if "Compiling entry function" in line and kernel in line:
            for nxt in lines[i + 1:i + 6]:
                m = re.search(r"Used (\d+) registers", nxt)
                if m:
                    return int(m.group(1))
    return None


if __name__ == "__main__":
    print(build(verbose="--verbose" in sys.argv, force=True, check="--check" in sys.argv))
