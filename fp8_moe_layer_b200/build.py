"""Builds the CUDA library ``libfp8moe.so`` in place (sm_100a only) with nvcc.

The library links the CUDA runtime dynamically (``-cudart shared``) so that, inside a process that
already imported torch, it shares torch's runtime: the same current device, streams and events.
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libfp8moe.so")
# The wait-test build: the same sources with every in-kernel wait bounded at 2 ms and a host
# switch that withholds one GEMM signal (include/moe_testing.h), for the tests of the
# device-timeout path. Nothing but those tests loads it.
LIB_WAITTEST = os.path.join(HERE, "libfp8moe_waittest.so")
# The role-counter build: the grouped GEMMs add up the cycles each warp role waits
# (include/moe_testing.h; fp8_moe_layer_b200/role_counters.py reads them).
LIB_ROLES = os.path.join(HERE, "libfp8moe_roles.so")
VARIANTS = {LIB: [], LIB_WAITTEST: ["-DMOE_WAIT_TEST"], LIB_ROLES: ["-DMOE_ROLE_COUNTERS"]}
SOURCES = ["moe_api.cu", "route.cu", "router_mma.cu", "permute.cu", "gemm.cu", "combine.cu",
           "noalloc.cu", "dispatch.cu"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc_path() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the FP8 MoE library needs the CUDA 12.9 toolkit")


def sources():
    return [os.path.join(CSRC, s) for s in SOURCES]


def needs_build(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    deps = sources() + [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith(".cuh")]
    inc = os.path.join(os.path.dirname(HERE), "include")
    deps += [os.path.join(inc, f) for f in os.listdir(inc) if f.endswith(".h")]
    return any(os.path.getmtime(p) > t for p in deps)


def build(force: bool = False, verbose: bool = False, ptxas_info: bool = False,
          lib: str = LIB) -> str:
    """Compile `lib` (the library, or its wait-test build) if any source is newer than it;
    returns its path."""
    if not force and not needs_build(lib):
        return lib
    cmd = [nvcc_path(), "-O3", "-std=c++17", *ARCH, "-lineinfo", "-shared", "-cudart", "shared",
           "-Xcompiler", "-fPIC", "-Xcompiler", "-Wall", *VARIANTS[lib], "-o", lib + ".tmp",
           *sources()]
    if ptxas_info:
        cmd.insert(1, "-Xptxas=-v")
    if verbose:
        print(" ".join(cmd), file=sys.stderr)
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError(f"nvcc failed ({res.returncode}):\n{res.stdout}\n{res.stderr}")
    if verbose or ptxas_info:
        print(res.stdout + res.stderr, file=sys.stderr)
    os.replace(lib + ".tmp", lib)
    return lib


if __name__ == "__main__":
    for target in ([LIB, LIB_WAITTEST, LIB_ROLES] if "--all" in sys.argv else [LIB]):
        build(force="--force" in sys.argv, verbose=True, ptxas_info="--ptxas-info" in sys.argv,
              lib=target)
        print(target)
