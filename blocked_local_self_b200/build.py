"""Build libhalo.so (the C-ABI CUDA library) in-tree for sm_100a.

Usage: python -m blocked_local_self_b200.build [--force]
"""
from __future__ import annotations

import os
import re
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libhalo.so")
SOURCES = [os.path.join(CSRC, "halo_api.cu")]
DEPS = SOURCES + [os.path.join(CSRC, f) for f in ("halo_tc.cuh", "halo_tc2.cuh", "halo_tc3.cuh", "halo_tc4.cuh", "halo_simt.cuh", "halo_bwd.cuh", "halo_bwd_tc.cuh", "halo_win.cuh", "halo_fused.cuh", "sm100.cuh")] + [
    os.path.join(ROOT, "include", "halo.h")]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-shared", "-cudart", "static",
         "-Xptxas", "-v"]


def _nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if cand and (os.path.sep not in cand or os.path.exists(cand)):
            return cand
    return "nvcc"


def needs_build() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(f) > t for f in DEPS)


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and not needs_build():
        return LIB
    tmp = LIB + ".tmp"
    cmd = [_nvcc(), *ARCH, *FLAGS, "-o", tmp, *SOURCES]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        sys.stderr.write(res.stdout + res.stderr)
        raise RuntimeError("nvcc failed building libhalo.so")
    log = res.stdout + res.stderr
    # The tensor-core kernel must not spill (a few bytes are tolerated), and must launch with the register
    # count its setmaxnreg split assumes (checked again at launch time).
    checked = 0
    for m in re.finditer(r"Compiling entry function '(\w+)'(.*?)Used (\d+) registers", log, re.S):
        name, spill, regs = m.group(1), m.group(2), int(m.group(3))
        if "halo_fwd_tc" in name or "halo_fused_tc" in name:  # the forward tensor-core kernels (setmaxnreg split)
            sp = re.search(r"(\d+) bytes spill stores", spill)
            if sp and int(sp.group(1)) > 32:
                raise RuntimeError(f"{name} spills registers: {spill.strip()}")
            if regs != 168:
                raise RuntimeError(f"{name} launches with {regs} registers, expected 168")
            checked += 1
    if checked == 0:
        raise RuntimeError("no tensor-core kernel found in the ptxas report")
    if verbose:
        sys.stdout.write(log)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose="-v" in sys.argv)
    print(LIB)
