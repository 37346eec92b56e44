"""CUDA-graph executor of the layer (one graph per token bucket and k profile): a replay matches
the oracle on the real tokens within the output tolerance, equals the eager moe_forward of the
padded batch bit for bit, and matches the unpadded eager call; inputs change between replays."""
import numpy as np
import pytest
import torch

from fp8_moe_layer_b200 import inputs as I
from tests import helpers as H

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ops():
    from fp8_moe_layer_b200 import ops
    return ops


def _pad(hidden, T_b):
    return torch.cat([hidden, hidden[:1].expand(T_b - hidden.shape[0], -1)])


@pytest.mark.parametrize("shape,T", [
    (I.MoEShape("graph_small", 64, 256, 16, 128, 4, 4, zipf_s=1.0), 5),
    (I.MoEShape("graph_shared", 64, 256, 8, 128, 2, 2, F_shared=128), 17),
    (I.MoEShape("graph_elastic", 64, 256, 32, 64, 2, 8, k_choices=(1, 2, 4, 8)), 23),
    (I.WORKLOADS["qwen3_T64"], 1),
], ids=lambda v: getattr(v, "name", str(v)))
def test_graph_replay_matches_eager(ops, shape, T):
    from fp8_moe_layer_b200.graphs import MoEGraphExecutor
    inp = H.make_inputs(shape, seed=7)
    layer = ops.MoELayerFP8(inp)
    ex = MoEGraphExecutor(layer, buckets=(1, 8, 32, 64))
    T_b = ex.bucket(T)
    kpt_full = inp.k_per_token.cuda() if inp.k_per_token is not None else None
    for rep, shift in enumerate((0, 3)):           # two replays with different tokens
        h = inp.hidden[shift:shift + T].cuda()
        kpt = kpt_full[shift:shift + T] if kpt_full is not None else None
        y_graph = ex(h, kpt).clone()
        torch.cuda.synchronize()
        assert ex.device_status() == ops.MOE_OK
        # the oracle on the same real tokens
        ref = H.run_oracle_on(inp, h, kpt)
        H.check_output(y_graph, None, ref["y64"], f"{shape.name} graph replay {rep}")
        # the same padded batch through the eager call: identical bits
        hp = _pad(h, T_b)
        kp = None
        if kpt is not None:
            kp = torch.cat([kpt, torch.ones(T_b - T, dtype=torch.int32, device="cuda")])
        lay_b = ops.MoELayerFP8(inp, max_T=T_b)
        y_eager_padded = lay_b(hp, kp)[:T]
        assert torch.equal(y_graph.view(torch.int16), y_eager_padded.view(torch.int16)), rep
        # the unpadded eager call: same outputs within the tolerance
        y_eager = layer(h, kpt)
        diff = (y_graph.float() - y_eager.float()).abs().max().item()
        assert diff <= H.Y_ATOL + 0.5 ** 8 * y_eager.float().abs().max().item(), (rep, diff)
    assert len(ex.graphs) == 1
