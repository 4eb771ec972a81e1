"""Build the sm_100a shared library ``libqlora_nf4.so`` in place with nvcc.

Usage: ``python -m bit_nf4_quantized_blk_b200.build [--checks]`` (or
``build()``, ``build(checks=True)`` for the debug library with the index and
alignment tests compiled in).
Every kernel is compiled for ``sm_100a`` only; the CUDA runtime is linked
statically and the driver entry point for TMA descriptors is resolved at run
time, so the library loads on a machine without a GPU driver (its calls then
return QLORA_ERR_CUDA / QLORA_ERR_UNSUPPORTED).
"""

from __future__ import annotations

import concurrent.futures
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
BUILD = os.path.join(HERE, "_build")
LIB = os.path.join(HERE, "libqlora_nf4.so")

SOURCES = ["api.cu", "quantize.cu", "dequant.cu", "gemv.cu", "lora_side.cu", "gemm_tc.cu", "gemm_nf4.cu", "merge.cu", "vdb_tc.cu", "selftest.cu"]

NVCC_FLAGS = [
    "-O3",
    "-std=c++17",
    "-gencode",
    "arch=compute_100a,code=sm_100a",
    "-lineinfo",
    "-Xcompiler",
    "-fPIC",
    "-Xcompiler",
    "-ffp-contract=off",
    "-Xcompiler",
    "-fno-fast-math",
    "-cudart",
    "static",
]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _stale(obj: str, deps) -> bool:
    if not os.path.exists(obj):
        return True
    t = os.path.getmtime(obj)
    return any(os.path.getmtime(d) > t for d in deps)


CHECKS_BUILD = os.path.join(HERE, "_build_checks")
CHECKS_LIB = os.path.join(HERE, "libqlora_nf4_checks.so")


def build(verbose: bool = False, ptxas_info: bool = False, checks: bool = False) -> str:
    """Compile the sources (in parallel, only those older than their inputs)
    and link the library.  checks=True builds libqlora_nf4_checks.so with
    -DQLORA_CHECKS: the same kernels with their index and alignment tests
    compiled in (a failed test records QLORA_ERR_CHECK and skips the access)."""
    build_dir, lib = (CHECKS_BUILD, CHECKS_LIB) if checks else (BUILD, LIB)
    os.makedirs(build_dir, exist_ok=True)
    headers = [os.path.join(CSRC, h) for h in os.listdir(CSRC) if h.endswith((".cuh", ".h"))]
    headers.append(os.path.join(HERE, "..", "include", "qlora_nf4.h"))
    objs, jobs = [], []
    for src in SOURCES:
        path = os.path.join(CSRC, src)
        obj = os.path.join(build_dir, src.replace(".cu", ".o"))
        objs.append(obj)
        if not _stale(obj, [path, *headers]) and not ptxas_info:
            continue
        cmd = [nvcc(), *NVCC_FLAGS, *(["-DQLORA_CHECKS"] if checks else []), "-c", path, "-o", obj]
        if ptxas_info:
            cmd += ["-Xptxas", "-v"]
        jobs.append(cmd)
    if jobs:
        workers = max(1, min(len(jobs), os.cpu_count() or 1))
        with concurrent.futures.ThreadPoolExecutor(workers) as pool:
            for cmd in jobs:
                if verbose:
                    print(" ".join(cmd))
            for _ in pool.map(lambda c: subprocess.run(c, check=True), jobs):
                pass
    if _stale(lib, objs):
        cmd = [nvcc(), "-shared", "-gencode", "arch=compute_100a,code=sm_100a", "-cudart", "static", "-o", lib, *objs]
        if verbose:
            print(" ".join(cmd))
        subprocess.run(cmd, check=True)
    return lib


if __name__ == "__main__":
    print(build(verbose=True, ptxas_info="-v" in sys.argv, checks="--checks" in sys.argv))
