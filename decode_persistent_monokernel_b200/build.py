"""Builds libkie.so (the C-ABI decode library), its profiling twin and the
micro-benchmark library libkie_ubench.so in-tree with nvcc for sm_100a."""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
SOURCES = ["kie_api.cu", "monokernel.cu", "prefill_gemm.cu", "prefill.cu"]
HEADERS = ["kie_internal.h", "prefill_internal.h", os.path.join("..", "..", "include", "kie.h")]
LIB = os.path.join(HERE, "libkie.so")
PROF_LIB = os.path.join(HERE, "libkie_prof.so")  # activity counters compiled in
UBENCH_LIB = os.path.join(HERE, "libkie_ubench.so")  # micro-benchmarks (kie_ubench.h)
UBENCH_SOURCES = ["ubench.cu"]
UBENCH_HEADERS = [os.path.join("..", "..", "include", "kie_ubench.h")]

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-shared",
    "-Xptxas", "-v",
]


def nvcc() -> str:
    for c in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if c and (os.path.sep not in c or os.path.exists(c)):
            return c
    return "nvcc"


def _stale(lib: str, sources, headers) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    deps = [os.path.join(CSRC, s) for s in sources + headers]
    return any(os.path.getmtime(p) > t for p in deps)


def _build_one(lib: str, extra, force: bool, verbose: bool, sources=None, headers=None) -> str:
    sources = SOURCES if sources is None else sources
    headers = HEADERS if headers is None else headers
    if not force and not _stale(lib, sources, headers):
        return lib
    tmp = lib + f".tmp{os.getpid()}"
    cmd = [nvcc(), *NVCC_FLAGS, *extra, "-I", os.path.join(ROOT, "include"),
           *[os.path.join(CSRC, s) for s in sources], "-o", tmp]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + res.stdout + res.stderr)
    if verbose:
        sys.stderr.write(res.stderr)
    os.replace(tmp, lib)
    if lib == LIB:
        with open(os.path.join(HERE, "ptxas_info.txt"), "w") as f:
            f.write(res.stderr)
    return lib


def build(force: bool = False, verbose: bool = False, profile: bool = True) -> str:
    """Builds libkie.so and (unless profile=False) the profiling libkie_prof.so."""
    _build_one(LIB, [], force, verbose)
    if profile:
        _build_one(PROF_LIB, ["-DKIE_PROFILE"], force, False)
    _build_one(UBENCH_LIB, [], force, False, UBENCH_SOURCES, UBENCH_HEADERS)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose=True)
    print(LIB)
