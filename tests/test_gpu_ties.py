"""Exact ties in the routing decision on the GPU: router weights whose rows come in identical
pairs (experts 2j and 2j+1 score exactly the same for every token), through every router path
and both selection methods (k_t rounds of a warp selection, or a block-wide sort for k_t > 8).
The rule: equal logits go to the lower expert id, in the selected set and in the slot order."""
import numpy as np
import pytest
import torch

from fp8_moe_layer_b200 import inputs as I
from oracle import moe_oracle as O
from tests import helpers as H

pytestmark = pytest.mark.gpu

TIE_SHAPES = [
    I.MoEShape("ties_gemv_T5_k16", 5, 256, 96, 64, 16, 16),                 # one-kernel decode router
    I.MoEShape("ties_cuda_core_T64_k4", 64, 256, 128, 64, 4, 4),           # warp selection
    I.MoEShape("ties_cuda_core_T64_k16", 64, 256, 128, 64, 16, 16),        # block sort
    I.MoEShape("ties_elastic_T64_E512", 64, 256, 512, 64, 2, 32, k_choices=(2, 8, 16, 32)),
    I.MoEShape("ties_mma_T4096_k16", 4096, 512, 256, 64, 16, 16),          # tensor-core router
]


@pytest.fixture(scope="module")
def ops():
    from fp8_moe_layer_b200 import ops
    return ops


@pytest.mark.parametrize("shape", TIE_SHAPES, ids=lambda s: s.name)
def test_duplicate_router_rows_go_to_lower_id(ops, shape):
    hidden = I.make_hidden(shape, 0)
    rw, rb = I.make_router(shape, 0)
    rw = rw.clone()
    rw[1::2] = rw[0::2]                        # experts 2j and 2j+1: identical rows
    kpt = I.make_k_per_token(shape, 0)
    x = O.bf16_bits_to_f64(H.hidden_bits(hidden))
    logits = O.router_logits(x, rw.numpy(), None)
    k_t = O.token_k(shape.T, shape.k, None if kpt is None else kpt.numpy())
    ids_ref = O.select_topk(logits, k_t, shape.k_max)
    ref = dict(logits=logits, topk_ids=ids_ref, topk_w=O.routing_weights(logits, ids_ref), k_t=k_t)
    c = lambda t: None if t is None else t.cuda()
    ids, w = ops.moe_route_topk(c(hidden), c(rw), None, shape.k, c(kpt), shape.k_max)
    ids, w = H.np_(ids), H.np_(w)
    # the oracle comparison (ids exact except within EXACT_TIE, where any valid top-k passes)
    H.check_routing(ids, w, ref)
    # the tie rule itself: the odd twin is never chosen without its even twin, which comes first
    ties = 0
    for t in range(shape.T):
        sel = [int(e) for e in ids[t, :k_t[t]]]
        pos = {e: j for j, e in enumerate(sel)}
        for e in sel:
            if e % 2 == 1:
                assert e - 1 in pos, (t, sel)
                assert pos[e - 1] < pos[e], (t, sel)
                ties += 1
        # twins of equal weight
        for e in sel:
            if e % 2 == 1:
                assert w[t, pos[e]] == w[t, pos[e - 1]], (t, sel)
    assert ties > 0
