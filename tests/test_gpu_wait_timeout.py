"""The device-timeout path, exercised without faulting, trapping or hanging the GPU.

Every spin-wait inside the library's kernels is bounded; when one expires, the kernel records
MOE_ERR_DEVICE_TIMEOUT (with a where-code) in the workspace status word, lets its in-flight copies
and MMAs land, frees its tensor memory and returns. These tests load the library's wait-test
build (include/moe_testing.h: every wait bounded at 2 ms, and a switch that makes the gate/up
GEMM withhold one "accumulator ready" signal), so a wait that nothing satisfies runs out. They
check that the status is reported, and that the same process and CUDA context then run the layer
normally, in the wait-test build and in the production library, with outputs equal to the
oracle's.
"""
import ctypes

import pytest
import torch

from fp8_moe_layer_b200 import inputs as I
from tests import helpers as H

pytestmark = pytest.mark.gpu

WHERE_GEMM1 = 4          # where-code of the gate/up GEMM in the status word


@pytest.fixture(scope="module")
def libs():
    from fp8_moe_layer_b200 import build, ops
    lib = ops.load_library(build.build(lib=build.LIB_WAITTEST))
    lib.moe_test_withhold_gemm_commit.argtypes = [ctypes.c_int]
    lib.moe_test_withhold_gemm_commit.restype = None
    yield ops, lib
    lib.moe_test_withhold_gemm_commit(0)


def _forward(ops, d, s, ws, lib=None):
    return ops.moe_forward(d["hidden"], d["router_w"], d["router_bias"], s.k, d["k_per_token"],
                           d["w13"], d["w13_scale"], d["w2"], d["w2_scale"], s.k_max,
                           shared=d["shared"], ws=ws, lib=lib)


@pytest.mark.parametrize("shape", [
    I.WORKLOADS["tiny_T16"],
    # 16 experts x 32 weight tiles = 512 tiles on 148 SMs: after the expired wait a CTA's MMA
    # issuer also runs out of its own bounded wait for a free accumulator (third tile)
    I.MoEShape("timeout_many_tiles", 64, 256, 16, 2048, 2, 2),
], ids=lambda s: s.name)
def test_expired_wait_is_reported_and_the_context_stays_usable(libs, shape):
    ops, lib = libs
    inp = H.make_inputs(shape, seed=0)
    d = H.to_cuda(inp)
    dm = ops.dims(shape.T, shape.d, shape.E, shape.F, shape.k_max, shape.F_shared)
    ref = H.run_oracle(inp)

    ws = ops.alloc_workspace(dm)
    lib.moe_test_withhold_gemm_commit(1)
    try:
        _forward(ops, d, shape, ws, lib=lib)              # the launches themselves succeed
        torch.cuda.synchronize()
    finally:
        lib.moe_test_withhold_gemm_commit(0)
    assert ops.device_status(ws) == ops.MOE_ERR_DEVICE_TIMEOUT
    assert int(ws[4:8].view(torch.int32).item()) == WHERE_GEMM1

    # the same context: the wait-test build on a fresh workspace, then the production library
    ws2 = ops.alloc_workspace(dm)
    y2 = _forward(ops, d, shape, ws2, lib=lib)
    assert ops.device_status(ws2) == ops.MOE_OK
    H.check_output(y2, None, ref["y64"], f"{shape.name} after a timeout (wait-test build)")
    ws3 = ops.alloc_workspace(dm)
    y3 = _forward(ops, d, shape, ws3)
    assert ops.device_status(ws3) == ops.MOE_OK
    H.check_output(y3, None, ref["y64"], f"{shape.name} after a timeout (library)")
