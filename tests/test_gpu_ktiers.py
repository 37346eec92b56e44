"""k-aware batching on the GPU: the tiered fixed-k calls (eager and graph-replayed) match the
oracle on every token, and the output of the one-call elastic layer, within the output
tolerance."""
import pytest
import torch

from fp8_moe_layer_b200 import inputs as I
from tests import helpers as H

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("shape", [
    I.MoEShape("tiers_small", 96, 256, 32, 64, 2, 8, k_choices=(1, 2, 4, 8)),
    I.WORKLOADS["prism_T64"],
], ids=lambda s: s.name)
@pytest.mark.parametrize("graphs", [False, True])
def test_tiered_equals_elastic(shape, graphs):
    from fp8_moe_layer_b200 import ops
    from fp8_moe_layer_b200.ktiers import KTieredLayer, k_tiers
    inp = H.make_inputs(shape, seed=3)
    layer = ops.MoELayerFP8(inp)
    h = inp.hidden.cuda()
    kpt_host = inp.k_per_token
    y_e = layer(h, kpt_host.cuda()).float()
    tiered = KTieredLayer(layer, graphs=graphs, buckets=(8, 16, 32, 64, 128))
    y_t = tiered(h, kpt_host).float()
    torch.cuda.synchronize()
    assert len(k_tiers(kpt_host)) > 1
    assert ops.device_status(layer.ws) == ops.MOE_OK
    diff = (y_t - y_e).abs().max().item()
    assert diff <= H.Y_ATOL + 0.5 ** 8 * y_e.abs().max().item(), diff
    ref = H.run_oracle(inp)
    H.check_output(y_t.to(torch.bfloat16), None, ref["y64"], f"{shape.name} tiered")
