"""The workspace-free router entry point, for callers that cannot allocate device memory.

moe_route_topk_noalloc keeps its scratch in a fixed device array inside the library instead of
a caller-provided workspace. These tests call it through the C ABI, twice in a row on the same
inputs (the array keeps the previous call's contents), and check each result against the
workspace entry point moe_route_topk with the tolerances the other routing tests use. This file
is named so that pytest collects it after every other test file.
"""
import ctypes

import numpy as np
import pytest
import torch

from fp8_moe_layer_b200 import inputs as I
from oracle import moe_oracle as O
from tests import helpers as H

pytestmark = pytest.mark.gpu

SHAPES = [
    I.WORKLOADS["tiny_T16"],                                # E <= 32: no scratch needed
    I.MoEShape("scratch_E64_T37", 37, 256, 64, 64, 6, 6, zipf_s=0.8),
    I.WORKLOADS["qwen3_T64"],                               # E = 128, Zipf router bias
    I.WORKLOADS["prism_T64"],                               # E = 512, per-token k
    # shapes where the workspace router takes another algorithm than this entry point's
    # CUDA-core logits: the one-kernel decode router (T <= 8, E > 32) and the tensor-core router
    # with fp64 refinement (T * E * d >= 2^29)
    I.WORKLOADS["qwen3_T1"],
    I.WORKLOADS["qwen3_T4096"],
]


def _noalloc(ops, shape, hidden, rw, rb, kpt):
    dm = ops.dims(shape.T, shape.d, shape.E, 16, shape.k_max)
    ids = torch.full((shape.T, shape.k_max), -7, dtype=torch.int32, device="cuda")
    w = torch.full((shape.T, shape.k_max), float("nan"), dtype=torch.float32, device="cuda")
    p = lambda t: None if t is None else t.data_ptr()
    rc = ops.LIB.moe_route_topk_noalloc(
        ctypes.byref(dm), p(hidden.view(torch.int16)), p(rw), p(rb), shape.k, p(kpt), p(ids),
        p(w), torch.cuda.current_stream().cuda_stream)
    assert rc == ops.MOE_OK, ops.status_string(rc)
    torch.cuda.synchronize()
    return H.np_(ids), H.np_(w)


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: s.name)
def test_noalloc_router_matches_workspace_router(shape):
    from fp8_moe_layer_b200 import ops
    hidden = I.make_hidden(shape, 0).cuda()
    rw, rb = I.make_router(shape, 0)
    rw, rb = rw.cuda(), None if rb is None else rb.cuda()
    kpt = I.make_k_per_token(shape, 0)
    kpt = None if kpt is None else kpt.cuda()
    ref_ids, ref_w = ops.moe_route_topk(hidden, rw, rb, shape.k, kpt, shape.k_max)
    ref_ids, ref_w = H.np_(ref_ids), H.np_(ref_w)
    # both entry points decide in fp64; only an exact fp64 tie may order experts differently
    x = O.bf16_bits_to_f64(H.hidden_bits(hidden.cpu()))
    logits = O.router_logits(x, H.np_(rw), H.np_(rb))
    k_t = O.token_k(shape.T, shape.k, H.np_(kpt))
    exact = set(H.exact_tie_tokens(logits, k_t).tolist())
    for call in range(2):
        ids, w = _noalloc(ops, shape, hidden, rw, rb, kpt)
        for t in range(shape.T):
            kt = int(k_t[t])
            assert np.all(ids[t, kt:] == -1) and np.all(w[t, kt:] == 0), (call, t)
            if t in exact:
                assert set(ids[t, :kt].tolist()) <= set(np.argsort(-logits[t])[:kt + 4].tolist())
                continue
            assert np.array_equal(ids[t], ref_ids[t]), (call, t, ids[t], ref_ids[t])
            assert np.abs(w[t] - ref_w[t]).max() <= H.WEIGHT_ATOL, (call, t, w[t], ref_w[t])


def test_noalloc_router_rejects_shapes_beyond_its_scratch():
    from fp8_moe_layer_b200 import ops
    # 65536 tokens x 512 experts of fp32 partial logits is 128 MiB > the 16 MiB array
    dm = ops.dims(65536, 2048, 512, 16, 8)
    fake = ctypes.c_void_p(1 << 20)          # never dereferenced: the size check comes first
    rc = ops.LIB.moe_route_topk_noalloc(ctypes.byref(dm), fake, fake, None, 8, None, fake, fake,
                                        None)
    assert rc == ops.MOE_ERR_UNSUPPORTED
