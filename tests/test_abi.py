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
    # expert-parallel dispatch: the rank count must divide E and lie in [1, 32]
    ep = lambda dm_, n, k, ws_bytes, cnt=fake: L.moe_ep_dispatch(
        ctypes.byref(dm_), n, fake, fake, fake, k, None, fake, fake, fake, cnt, fake, fake, fake,
        ws_bytes, None)
    assert ep(dm, 3, 2, 1 << 30) == ops.MOE_ERR_INVALID_ARG
    assert ep(dm, 0, 2, 1 << 30) == ops.MOE_ERR_INVALID_ARG
    assert ep(ops.dims(4, 128, 64, 256, 2), 64, 2, 1 << 30) == ops.MOE_ERR_INVALID_ARG
    assert ep(dm, 4, 2, 1 << 30, cnt=None) == ops.MOE_ERR_INVALID_ARG
    assert ep(dm, 4, 3, 1 << 30) == ops.MOE_ERR_INVALID_ARG          # k > k_max
    assert ep(dm, 4, 2, 16) == ops.MOE_ERR_WORKSPACE
    assert ep(bad, 4, 2, 1 << 30) == ops.MOE_ERR_INVALID_ARG
    assert L.moe_ep_dispatch(ctypes.byref(dm), 4, ctypes.c_void_p((1 << 20) + 8), fake, fake, 2,
                             None, fake, fake, fake, fake, fake, fake, fake, 1 << 30,
                             None) == ops.MOE_ERR_INVALID_ARG              # hidden misaligned
    # T == 0 is a valid no-op
    zero = ops.dims(0, 128, 8, 256, 2)
    assert L.moe_forward(ctypes.byref(zero), *([None] * 3), 2, *([None] * 11), 0, None,
                         None) == ops.MOE_OK


# The final C signatures, written out: a C file assigns every entry point to a pointer of exactly
# this type, and gcc rejects any difference (-Werror). The Python binding's argument counts must
# match too. (Departures from the boundary first sketched are listed in the design notes.)
SIGNATURES = {
    "moe_workspace_bytes": "size_t (*)(const moe_dims*)",
    "moe_status_string": "const char* (*)(int)",
    "moe_kernel_launch_count": "uint64_t (*)(void)",
    "moe_clear_status": "int (*)(void*, void*)",
    "moe_device_status": "int (*)(const void*, void*, int32_t*)",
    "moe_route_topk": "int (*)(const moe_dims*, const uint16_t*, const float*, const float*, "
                      "int32_t, const int32_t*, int32_t*, float*, void*, size_t, void*)",
    "moe_permute": "int (*)(const moe_dims*, const int32_t*, int32_t, const int32_t*, int32_t*, "
                   "int32_t*, int32_t*, void*, size_t, void*)",
    "moe_grouped_ffn_fp8": "int (*)(const moe_dims*, const uint16_t*, const uint8_t*, "
                           "const float*, const uint8_t*, const float*, const int32_t*, "
                           "const int32_t*, float*, float*, void*, size_t, void*)",
    "moe_combine": "int (*)(const moe_dims*, const float*, const float*, const int32_t*, "
                   "const float*, uint16_t*, float*, void*)",
    "moe_forward": "int (*)(const moe_dims*, const uint16_t*, const float*, const float*, int32_t, "
                   "const int32_t*, const uint8_t*, const float*, const uint8_t*, const float*, "
                   "const uint8_t*, const float*, const uint8_t*, const float*, uint16_t*, void*, "
                   "size_t, void*, const moe_debug_out*)",
    "moe_route_topk_noalloc": "int (*)(const moe_dims*, const uint16_t*, const float*, "
                              "const float*, int32_t, const int32_t*, int32_t*, float*, void*)",
    "moe_ep_dispatch": "int (*)(const moe_dims*, int32_t, const uint16_t*, const int32_t*, "
                       "const float*, int32_t, const int32_t*, uint16_t*, int32_t*, float*, "
                       "int32_t*, int32_t*, float*, void*, size_t, void*)",
}


def _nargs(sig: str) -> int:
    inner = sig.split("(*)(", 1)[1].rsplit(")", 1)[0].strip()
    return 0 if inner == "void" else inner.count(",") + 1


def test_header_signatures_are_the_final_ones(tmp_path):
    import shutil
    import subprocess
    assert sorted(SIGNATURES) == declared_functions()
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no C compiler")
    lines = ['#include "moe.h"']
    for i, (name, sig) in enumerate(SIGNATURES.items()):
        ptr = sig.replace("(*)", f"(*p{i})", 1)
        lines.append(f"{ptr} = {name};")
    src = tmp_path / "sig.c"
    src.write_text("\n".join(lines) + "\n")
    res = subprocess.run([gcc, "-std=c11", "-Wall", "-Werror", "-c", str(src), "-o",
                          str(tmp_path / "sig.o"), f"-I{os.path.dirname(HEADER)}"],
                         capture_output=True, text=True)
    assert res.returncode == 0, res.stderr


def test_binding_argument_counts_match_the_header(ops):
    for name, sig in SIGNATURES.items():
        fn = getattr(ops.LIB, name)
        assert len(fn.argtypes) == _nargs(sig), name


def test_test_builds_export_their_entry_points_and_the_library_does_not():
    from fp8_moe_layer_b200 import build
    path = build.build(lib=build.LIB_WAITTEST)
    text = re.sub(r"/\*.*?\*/", "", open(os.path.join(ROOT, "include", "moe_testing.h")).read(),
                  flags=re.S)
    names = sorted(set(re.findall(r"\b(moe_[a-z0-9_]+)\s*\(", text)))
    assert names == ["moe_role_counters_read", "moe_role_counters_reset",
                     "moe_test_withhold_gemm_commit"]
    test_lib = ctypes.CDLL(path)
    roles_lib = ctypes.CDLL(build.build(lib=build.LIB_ROLES))
    prod = ctypes.CDLL(os.path.join(ROOT, "fp8_moe_layer_b200", "libfp8moe.so"))
    assert hasattr(test_lib, "moe_test_withhold_gemm_commit")
    assert hasattr(roles_lib, "moe_role_counters_read")
    assert hasattr(roles_lib, "moe_role_counters_reset")
    for n in names:
        assert not hasattr(prod, n)
    for n in declared_functions():
        assert hasattr(test_lib, n), n
        assert hasattr(roles_lib, n), n
