"""Build libdt.so (the C-ABI library) in-tree with nvcc for sm_100a.

Usage: ``python -m partitioned_attention_state_b200.build [--verbose]``.
Cross-compiles without a GPU.  The output sits next to this file so that it
travels with the source tree.
"""

from __future__ import annotations

import os
import re
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libdt.so")
SOURCES = ["plan.cpp", "api.cu", "attn_fused_sm100.cu", "state_ops.cu"]
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
         "--expt-relaxed-constexpr"]


def _check_launch_registers(ptxas_log: str) -> None:
    """The fused kernel splits its launch register pool between warpgroups
    with setmaxnreg; the split is sized for exactly kLaunchRegs registers per
    thread at launch.  A smaller pool would make setmaxnreg.inc wait forever,
    so refuse to build if ptxas chose another count."""
    src = open(os.path.join(CSRC, "attn_fused_sm100.cu")).read()
    want = int(re.search(r"constexpr int kLaunchRegs = (\d+);", src).group(1))
    found = []
    cur = None
    for line in ptxas_log.splitlines():
        m = re.search(r"Compiling entry function '(\S+)'", line)
        if m:
            cur = m.group(1)
        m = re.search(r"Used (\d+) registers", line)
        if m and cur and "attn_partial_fused_kernel" in cur:
            found.append(int(m.group(1)))
    if not found or any(n != want for n in found):
        raise RuntimeError(f"fused kernel launch registers {found} != {want}: setmaxnreg split would not fit")


def _newer(out: str, deps) -> bool:
    if not os.path.exists(out):
        return False
    t = os.path.getmtime(out)
    return all(os.path.getmtime(d) <= t for d in deps)


def build(verbose: bool = False, force: bool = False) -> str:
    deps = [os.path.join(CSRC, f) for f in os.listdir(CSRC)]
    deps.append(os.path.join(HERE, "..", "include", "dt.h"))
    if not force and _newer(LIB, deps):
        return LIB
    objdir = os.path.join(HERE, "_build")
    os.makedirs(objdir, exist_ok=True)
    objs = []
    for src in SOURCES:
        obj = os.path.join(objdir, os.path.splitext(src)[0] + ".o")
        cmd = [NVCC, *ARCH, *FLAGS, "-Xptxas=-v", "-c", os.path.join(CSRC, src), "-o", obj]
        if verbose:
            print(" ".join(cmd), flush=True)
        res = subprocess.run(cmd, check=True, capture_output=True, text=True)
        if verbose:
            sys.stderr.write(res.stderr)
        if src == "attn_fused_sm100.cu":
            _check_launch_registers(res.stderr)
        objs.append(obj)
    cmd = [NVCC, *ARCH, "-shared", "-Xcompiler", "-fPIC", "-o", LIB + ".tmp", *objs]
    if verbose:
        print(" ".join(cmd), flush=True)
    subprocess.run(cmd, check=True)
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    build(verbose="--verbose" in sys.argv, force="--force" in sys.argv)
    print(LIB)
