"""Builds libgdn.so (the C-ABI CUDA library) in-tree for sm_100a with nvcc.

    python -m looped_linear_attention_b200.build [--force] [--verbose]

The library links the CUDA runtime statically and looks up the driver entry
point it needs (cuTensorMapEncodeTiled) at run time, so it loads on a host
without a GPU (the kernels then simply cannot run).
"""
from __future__ import annotations

import argparse
import glob
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB_PATH = os.path.join(PKG, "libgdn.so")

ARCH_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a"]


def _nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: set NVCC or put CUDA's bin directory on PATH")


def sources():
    return sorted(glob.glob(os.path.join(CSRC, "*.cu")))


def _stale(out: str, deps) -> bool:
    if not os.path.exists(out):
        return True
    t = os.path.getmtime(out)
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose: bool = False, ptxas_info: bool = False) -> str:
    deps = (sources() + glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h"))
            + glob.glob(os.path.join(INCLUDE, "*.h")))
    if not force and not _stale(LIB_PATH, deps):
        return LIB_PATH
    tmp = LIB_PATH + f".tmp{os.getpid()}"
    cmd = [_nvcc(), "-O3", "-std=c++17", *ARCH_FLAGS, "-lineinfo", "-Xcompiler", "-fPIC",
           "-shared", "-cudart", "static", "-Xptxas=-v", "-I", INCLUDE, "-I", CSRC, "-o", tmp,
           *sources()]
    if verbose:
        print(" ".join(cmd), file=sys.stderr)
    r = subprocess.run(cmd, capture_output=True, text=True)
    if ptxas_info or r.returncode != 0:
        sys.stderr.write(r.stdout + r.stderr)
    if r.returncode != 0:
        raise RuntimeError("nvcc failed")
    spills = check_no_spills(r.stdout + r.stderr)
    if spills:
        os.remove(tmp)
        raise RuntimeError("register spills in " + ", ".join(spills) +
                           " (the tensor-core kernels are kept spill-free)")
    os.replace(tmp, LIB_PATH)
    return LIB_PATH


# Kernels that drive tcgen05 / tensor memory must not spill registers: spills
# around asynchronously written tensor-memory load registers were the one
# difference between faulting and clean builds of the prefill kernel.
SPILL_FREE_KERNELS = ("gdn_prefill_tc_kernel", "gdn_segment_correct_kernel", "swa_fwd_kernel")


def check_no_spills(ptxas_log: str):
    """Names of the tensor-core kernels for which ptxas reports spill stores or loads."""
    bad, current = [], None
    for line in ptxas_log.splitlines():
        if "Compiling entry function" in line:
            current = line.split("'")[1] if "'" in line else line
        elif "spill stores" in line and current:
            nums = [int(t) for t in line.replace(",", " ").split() if t.isdigit()]
            if len(nums) >= 3 and (nums[1] or nums[2]) and any(
                    k in current for k in SPILL_FREE_KERNELS):
                bad.append(current)
    return bad


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", action="store_true")
    ap.add_argument("--ptxas-info", action="store_true")
    a = ap.parse_args()
    print(build(force=a.force, verbose=a.verbose, ptxas_info=a.ptxas_info))


if __name__ == "__main__":
    main()
