"""The C-ABI library loads on a machine without a GPU, exports every entry point that
include/moe.h declares, and rejects bad arguments on the host before touching the device."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(moe_[a-z0-9_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def ops():
    from fp8_moe_layer_b200 import build
    build.build()
    from fp8_moe_layer_b200 import ops
    return ops


def test_header_declares_the_entry_points():
    names = declared_functions()
    for n in ("moe_route_topk", "moe_permute", "moe_grouped_ffn_fp8", "moe_combine",
              "moe_forward", "moe_workspace_bytes", "moe_device_status", "moe_status_string",
              "moe_clear_status"):
        assert n in names


def test_library_exports_every_declared_symbol(ops):
    lib = ctypes.CDLL(ops.LIB_PATH)
    for name in declared_functions():
        assert hasattr(lib, name), name


def test_status_strings(ops):
    for code in range(0, -7, -1):
        assert ops.status_string(code) not in ("", "unknown status")
    assert ops.status_string(42) == "unknown status"


def test_workspace_bytes_is_pure_and_rejects_bad_dims(ops):
    from fp8_moe_layer_b200.inputs import WORKLOADS
    for s in WORKLOADS.values():
        n = ops.workspace_bytes(ops.dims(s.T, s.d, s.E, s.F, s.k_max, s.F_shared))
        assert n > 0 and n % 256 == 0
    assert ops.workspace_bytes(ops.dims(4, 100, 8, 64, 2)) == 0       # d not a multiple of 16
    assert ops.workspace_bytes(ops.dims(4, 128, 0, 64, 2)) == 0       # no experts
    assert ops.workspace_bytes(ops.dims(4, 128, 8, 64, 33)) == 0      # k_max > 32
    assert ops.workspace_bytes(ops.dims(4, 128, 2000, 64, 2)) == 0    # E > 1024
    assert ops.workspace_bytes(ops.dims(4, 128, 8, 64, 2, 32)) == 0   # F_shared != F


def test_host_validation_without_gpu(ops):
    L = ops.LIB
    dm = ops.dims(4, 128, 8, 256, 2)
    bad = ops.dims(4, 100, 8, 256, 2)
    # invalid shape: rejected before any CUDA call
    assert L.moe_forward(ctypes.byref(bad), *([None] * 3), 2, *([None] * 11), 0, None,
                         None) == ops.MOE_ERR_INVALID_ARG
    # missing pointers
    assert L.moe_forward(ctypes.byref(dm), *([None] * 3), 2, *([None] * 11), 0, None,
                         None) == ops.MOE_ERR_INVALID_ARG
    assert L.moe_route_topk(ctypes.byref(dm), None, None, None, 2, None, None, None, None, 0,
                            None) == ops.MOE_ERR_INVALID_ARG
    assert L.moe_combine(None, None, None, None, None, None, None, None) == ops.MOE_ERR_INVALID_ARG
    # k out of range and a too small workspace are host-side errors too
    fake = ctypes.c_void_p(1 << 20)   # aligned, never dereferenced by the host checks
    args = [fake] * 3
    assert L.moe_route_topk(ctypes.byref(dm), fake, fake, None, 9, None, fake, fake, fake, 1 << 30,
                            None) == ops.MOE_ERR_INVALID_ARG
    assert L.moe_route_topk(ctypes.byref(dm), fake, fake, None, 2, None, fake, fake, fake, 16,
                            None) == ops.MOE_ERR_WORKSPACE
    # T == 0 is a valid no-op
    zero = ops.dims(0, 128, 8, 256, 2)
    assert L.moe_forward(ctypes.byref(zero), *([None] * 3), 2, *([None] * 11), 0, None,
                         None) == ops.MOE_OK
