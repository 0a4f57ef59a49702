"""Build the BSFA C-ABI library (libbsfa.so) for sm_100a with nvcc, in-tree.

The translation units compile in parallel; the library links the CUDA runtime
statically and reaches the driver's tensor-map encoder at run time, so it needs
no -lcuda.
"""
from __future__ import annotations

import concurrent.futures as cf
import os
import re
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
BUILD = os.path.join(PKG, "_build")
LIB = os.path.join(PKG, "libbsfa.so")
SOURCES = ["bsfa_api.cu", "bsfa_fwd_d64.cu", "bsfa_fwd_d128.cu"]
HEADERS = ["ptx.cuh", "bsfa_fwd_kernel.cuh", "bsfa_launch.cuh"]

# The forward kernel re-balances registers between its warpgroups
# (setmaxnreg); the split is sized for exactly this launch budget per thread, so
# the build refuses a kernel compiled with any other count.
FWD_KERNEL_REGS = 168

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-std=c++17", "-lineinfo",
    "-Xcompiler", "-fPIC",
    "--expt-relaxed-constexpr",
    "-I", INCLUDE, "-I", CSRC,
    "-Xptxas", "-v",
]


def check_registers(ptxas_log: str) -> None:
    """Every bsfa_fwd_kernel variant must be compiled with FWD_KERNEL_REGS registers."""
    entry = None
    for line in ptxas_log.splitlines():
        m = re.search(r"Compiling entry function '([^']+)'", line)
        if m:
            entry = m.group(1)
            continue
        m = re.search(r"Used (\d+) registers", line)
        if m and entry and "bsfa_fwd_kernel" in entry:
            if int(m.group(1)) != FWD_KERNEL_REGS:
                raise RuntimeError(f"{entry}: {m.group(1)} registers, expected {FWD_KERNEL_REGS}")
            entry = None


def nvcc() -> str:
    cand = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(cand):
        raise RuntimeError("nvcc not found")
    return cand


def _stale(target: str, deps: list[str]) -> bool:
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(d) > t for d in deps)


TRACE_BUILD = os.path.join(PKG, "_build_trace")
TRACE_LIB = os.path.join(PKG, "libbsfa_trace.so")


def build(force: bool = False, verbose: bool = False, extra_flags: list[str] | None = None,
          trace: bool = False) -> str:
    """Compile every translation unit and link libbsfa.so; returns the library path.

    trace=True builds the profiling variant instead, libbsfa_trace.so (kernels
    compiled with BSFA_TRACE, which stamp the SM clock at fixed points of each
    role; include/bsfa_trace.h), in its own build folder.
    """
    build_dir, lib = (TRACE_BUILD, TRACE_LIB) if trace else (BUILD, LIB)
    os.makedirs(build_dir, exist_ok=True)
    flags = NVCC_FLAGS + (["-DBSFA_TRACE"] if trace else []) + list(extra_flags or [])
    headers = [os.path.join(CSRC, h) for h in HEADERS] + [os.path.join(INCLUDE, h)
                                                         for h in ("bsfa.h", "bsfa_trace.h")]
    objs, jobs = [], []
    for src in SOURCES:
        s = os.path.join(CSRC, src)
        o = os.path.join(build_dir, src.replace(".cu", ".o"))
        objs.append(o)
        if force or _stale(o, [s] + headers + [__file__]):
            jobs.append([nvcc(), *flags, "-c", s, "-o", o])

    def run(cmd):
        r = subprocess.run(cmd, capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError(f"nvcc failed: {' '.join(cmd)}\n{r.stdout}\n{r.stderr}")
        if verbose and (r.stdout or r.stderr):
            print(r.stdout, r.stderr, file=sys.stderr)
        check_registers(r.stdout + r.stderr)
        return r

    with cf.ThreadPoolExecutor(max_workers=len(jobs) or 1) as ex:
        list(ex.map(run, jobs))
    if jobs or _stale(lib, objs):
        run([nvcc(), "-gencode", "arch=compute_100a,code=sm_100a", "-shared", "-Xcompiler", "-fPIC",
             "-o", lib, *objs])
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="--verbose" in sys.argv, trace="--trace" in sys.argv))
