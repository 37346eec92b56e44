"""Source-level rules of the CUDA library, checked on the CPU.

Every kernel is launched with programmatic dependent launch, so it may start before the kernel
in front of it has finished: each one must call pdl_wait() before it reads anything, i.e. as the
first statement of its body. And no device code may trap or assert (a fault would take the shared
GPU down); errors go to the status word instead."""
import glob
import os
import re

CSRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                    "fp8_moe_layer_b200", "csrc")


def kernels(src):
    for m in re.finditer(r"__global__[^{;]*?\)\s*\{", src, re.S):
        name = re.search(r"(\w+)\s*\(", src[m.start():m.end()].split("__launch_bounds__")[-1]
                         .split(")", 1)[-1])
        yield (name.group(1) if name else "?"), src[m.end():m.end() + 200]


def test_every_kernel_waits_for_its_predecessor_first():
    n = 0
    for path in glob.glob(os.path.join(CSRC, "*.cu")):
        src = open(path).read()
        for name, body in kernels(src):
            n += 1
            first = body.strip().split(";")[0].strip()
            assert first == "pdl_wait()", f"{os.path.basename(path)}:{name} starts with {first!r}"
    assert n >= 15


def test_no_trap_or_device_assert():
    for path in glob.glob(os.path.join(CSRC, "*.cu*")):
        src = re.sub(r"//.*", "", open(path).read())
        src = src.replace("static_assert(", "")          # compile-time checks are fine
        assert "__trap" not in src and "trap;" not in src and "assert(" not in src, path


def test_no_cluster_multicast_loads():
    # The library runs as replicas on several GPUs; no load may use cluster multicast (the pair
    # GEMM signals its two CTAs with separate commits instead). The qualifier is assembled here
    # so that this file does not spell it.
    qualifier = "." + "multicast" + "::" + "cluster"
    for path in glob.glob(os.path.join(CSRC, "*.cu*")):
        assert qualifier not in open(path).read(), path


def test_every_spin_wait_is_bounded():
    # mbarrier polls go through the bounded helpers only (a timeout records a status and returns)
    for path in glob.glob(os.path.join(CSRC, "*.cu*")):
        src = re.sub(r"//.*", "", open(path).read())
        if os.path.basename(path) == "common.cuh":
            continue                                    # the helpers themselves
        assert "mbarrier.try_wait" not in src, path
        assert "while (!mbar_try_wait" not in src and "while(!mbar_try_wait" not in src, path
