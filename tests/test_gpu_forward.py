"""GPU parity of the fused layer (moe_forward through the C ABI) against the oracle: every
token on small layers and edge cases, sampled tokens on the full-size workloads (routing and
grouping always checked on every token)."""
import numpy as np
import pytest
import torch

from fp8_moe_layer_b200 import inputs as I
from oracle import moe_oracle as O
from tests import helpers as H

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ops():
    from fp8_moe_layer_b200 import ops
    return ops


def forward_and_check(ops, inp, sample=None, seed=0):
    """moe_forward through the C ABI against the oracle. Routing and grouping are checked on
    every token (bit-exact). Outputs: every token, or -- when ``sample`` is given -- the tokens of
    every active expert's first and last routed rows (so every group's first tile and ragged tail
    tile is compared) plus ``sample`` tokens at random."""
    s = inp.shape
    d = H.to_cuda(inp)
    dm = ops.dims(s.T, s.d, s.E, s.F, s.k_max, s.F_shared)
    ws = ops.alloc_workspace(dm)
    y, dbg = ops.moe_forward(d["hidden"], d["router_w"], d["router_bias"], s.k, d["k_per_token"],
                             d["w13"], d["w13_scale"], d["w2"], d["w2_scale"], s.k_max,
                             shared=d["shared"], ws=ws, debug=True)
    assert ops.device_status(ws) == ops.MOE_OK
    gpu = {k: H.np_(v) for k, v in dbg.items()}

    # routing on every token, grouping bit-exact against the oracle's sort of the GPU's own ids
    # (and against the oracle's own grouping when the ids are identical)
    x = O.bf16_bits_to_f64(H.hidden_bits(inp.hidden))
    logits = O.router_logits(x, H.np_(inp.router_w), H.np_(inp.router_bias))
    k_t = O.token_k(s.T, s.k, H.np_(inp.k_per_token))
    ids = O.select_topk(logits, k_t, s.k_max)
    route_ref = dict(logits=logits, topk_ids=ids, topk_w=O.routing_weights(logits, ids), k_t=k_t)
    n_near, differed, n_exact = H.check_routing(gpu["topk_ids"], gpu["topk_w"], route_ref)
    same_grouping = H.check_grouping(gpu["expert_offsets"], gpu["perm_token"], gpu["inv_row"],
                                     gpu["topk_ids"], k_t, s.E, ref_ids=ids)

    # outputs: every token whose routing equals the oracle's (all but exact fp64 ties)
    agree = np.all(gpu["topk_ids"] == ids, axis=1)
    if sample is None:
        tokens = np.arange(s.T)
    else:
        tokens = H.coverage_tokens(gpu["expert_offsets"], gpu["perm_token"], s.E, s.T, sample,
                                   seed=seed, shared=bool(s.F_shared))
    tokens = tokens[agree[tokens]]
    ref = H.run_oracle(inp, tokens=tokens)
    stats = H.check_output(y[tokens], torch.from_numpy(gpu["y_f32"][tokens]), ref["y64"], s.name)
    print(f"{s.name}: tokens checked {len(tokens)}/{s.T}, near ties (<{H.NEAR_TIE:g}) {n_near} "
          f"(differing {differed}), exact ties (<{H.EXACT_TIE:g}) {n_exact}, grouping equal to "
          f"the oracle's {same_grouping}, {stats}")
    return y, dbg, stats


SMALL = [
    I.WORKLOADS["tiny_T16"],
    I.MoEShape("ragged_T37", 37, 256, 6, 64, 2, 2),
    I.MoEShape("elastic_small", 50, 128, 16, 64, 1, 8, k_choices=(1, 2, 4, 8)),
    I.MoEShape("shared_zipf", 33, 128, 8, 128, 3, 3, F_shared=128, zipf_s=1.2),
    I.MoEShape("k_equals_E", 19, 128, 5, 64, 5, 5),
    I.MoEShape("single_expert", 45, 128, 1, 128, 1, 1),
    I.MoEShape("ragged_K_F", 29, 192, 5, 96, 2, 2),
    I.MoEShape("small_d", 12, 64, 4, 32, 2, 2),
    # decode batches with E > 32 (the one-kernel GEMV router)
    I.MoEShape("decode_gemv_T3", 3, 256, 96, 128, 6, 6, zipf_s=1.0),
    I.MoEShape("decode_gemv_T8_shared", 8, 256, 40, 128, 4, 4, F_shared=128),
    # one to four tokens: groups of one to four rows in 16-column token tiles, the shared
    # expert's group, per-token k, K-split gate/up partials, E <= 32 with the fused router
    I.MoEShape("decode_T1", 1, 256, 64, 128, 8, 8),
    I.MoEShape("decode_T2_shared", 2, 256, 40, 128, 4, 4, F_shared=128),
    I.MoEShape("decode_T4_elastic", 4, 128, 48, 64, 2, 8, k_choices=(1, 2, 4, 8)),
    I.MoEShape("decode_T3_small_E", 3, 512, 8, 1024, 2, 2),
    I.MoEShape("decode_T4_long_F", 4, 128, 4, 4096, 2, 2, F_shared=4096),
    # token tiles >= 192 rows run the gate/up GEMM on 2-SM pairs, and the down GEMM too when
    # F >= 2048: odd weight m-tile counts (F = 192 -> 3 gate/up tiles, d = 384 -> 3 down tiles;
    # the pair's second half falls off the matrix), ragged tails, a shared-expert group
    I.MoEShape("pair_odd_m", 260, 384, 4, 192, 2, 2, zipf_s=0.5),
    I.MoEShape("pair_shared", 280, 256, 4, 128, 2, 2, F_shared=128),
    I.MoEShape("pair_down_odd_m", 160, 384, 2, 2048, 2, 2),
]


@pytest.mark.parametrize("shape", SMALL, ids=lambda s: s.name)
def test_forward_small_every_token(ops, shape):
    forward_and_check(ops, H.make_inputs(shape, seed=1))


def test_forward_skew_all_tokens_one_expert(ops):
    """Every token picks expert 2 first: one group with many token tiles."""
    shape = I.MoEShape("skew", 300, 256, 8, 128, 2, 2)
    inp = H.make_inputs(shape, seed=2)
    inp.router_bias = torch.zeros(shape.E)
    inp.router_bias[2] = 30.0
    forward_and_check(ops, inp)


def test_forward_zero_token_row_and_empty_batch(ops):
    shape = I.MoEShape("zero_row", 20, 128, 4, 64, 2, 2)
    inp = H.make_inputs(shape, seed=4)
    inp.hidden[7].zero_()
    y, _, _ = forward_and_check(ops, inp)
    # T = 0: a valid call that launches nothing
    d = H.to_cuda(inp)
    empty = torch.empty(0, shape.d, dtype=torch.bfloat16, device="cuda")
    y0 = ops.moe_forward(empty, d["router_w"], None, 2, None, d["w13"], d["w13_scale"], d["w2"],
                         d["w2_scale"], 2)
    assert y0.shape == (0, shape.d)


def test_forward_is_deterministic(ops):
    shape = I.WORKLOADS["qwen3_T64"]
    inp = H.make_inputs(shape, seed=0)
    layer = ops.MoELayerFP8(inp)
    h = inp.hidden.cuda()
    y1 = layer(h).clone()
    y2 = layer(h).clone()
    assert torch.equal(y1.view(torch.int16), y2.view(torch.int16))


# (workload, random tokens beside every expert's first- and last-row tokens; None = every token)
FULL = [("mixtral_T1", None), ("mixtral_T32", None), ("mixtral_T512", 128), ("qwen3_T1", None),
        ("qwen3_T64", None), ("qwen3_T4096", 128), ("prism_T64", None), ("prism_T2048", 128),
        ("deepseek_T128", None)]


@pytest.mark.parametrize("name,sample", FULL, ids=[f[0] for f in FULL])
def test_forward_full_size_workloads(ops, name, sample):
    forward_and_check(ops, H.make_inputs(I.WORKLOADS[name], seed=0), sample=sample)


def test_forward_deepseek_prefill(ops):
    forward_and_check(ops, H.make_inputs(I.WORKLOADS["deepseek_T8192"], seed=0), sample=64)
