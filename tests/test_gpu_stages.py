"""GPU parity of each stage entry point (router/top-k, permutation, grouped FP8 FFN, combine)
against the oracle, through the C ABI."""
import numpy as np
import pytest
import torch

from fp8_moe_layer_b200 import inputs as I
from oracle import moe_oracle as O
from tests import helpers as H

pytestmark = pytest.mark.gpu

ROUTE_SHAPES = [
    I.WORKLOADS["tiny_T16"],
    I.MoEShape("cuda_core_router", 37, 256, 64, 64, 6, 6, zipf_s=0.8),     # E > 32, small T·E·d
    # decode batches (T <= 8, E > 32): the one-kernel GEMV router
    I.MoEShape("gemv_router_T5", 5, 256, 96, 64, 6, 6, zipf_s=1.0),
    I.MoEShape("gemv_router_T1_E1000", 1, 512, 1000, 64, 8, 8),
    I.MoEShape("gemv_router_elastic_T7", 7, 256, 64, 64, 2, 8, k_choices=(1, 2, 4, 8)),
    # the tensor-core router (T·E·d >= 2^29): E % 128 != 0 and T % 64 != 0, and E = 33
    I.MoEShape("mma_router_ragged_E", 1000, 1056, 520, 64, 4, 4),
    I.MoEShape("mma_router_E33", 8200, 2048, 33, 64, 3, 3),
    I.MoEShape("ragged", 37, 256, 6, 64, 2, 2),
    I.MoEShape("k_equals_E", 19, 128, 5, 64, 5, 5),
    I.WORKLOADS["qwen3_T64"],
    I.WORKLOADS["prism_T64"],
    I.WORKLOADS["mixtral_T32"],
    I.WORKLOADS["deepseek_T128"],
    I.WORKLOADS["prism_T2048"],
    I.WORKLOADS["qwen3_T4096"],
]


@pytest.fixture(scope="module")
def ops():
    from fp8_moe_layer_b200 import ops
    return ops


def _router_only(shape, seed=0):
    hidden = I.make_hidden(shape, seed)
    rw, rb = I.make_router(shape, seed)
    kpt = I.make_k_per_token(shape, seed)
    return hidden, rw, rb, kpt


def _oracle_route(shape, hidden, rw, rb, kpt):
    x = O.bf16_bits_to_f64(H.hidden_bits(hidden))
    logits = O.router_logits(x, rw.numpy(), None if rb is None else rb.numpy())
    k_t = O.token_k(shape.T, shape.k, None if kpt is None else kpt.numpy())
    ids = O.select_topk(logits, k_t, shape.k_max)
    return dict(logits=logits, topk_ids=ids, topk_w=O.routing_weights(logits, ids), k_t=k_t)


@pytest.mark.parametrize("shape", ROUTE_SHAPES, ids=lambda s: s.name)
def test_route_topk_matches_oracle(ops, shape):
    hidden, rw, rb, kpt = _router_only(shape)
    ref = _oracle_route(shape, hidden, rw, rb, kpt)
    c = lambda t: None if t is None else t.cuda()
    ids, w = ops.moe_route_topk(c(hidden), c(rw), c(rb), shape.k, c(kpt), shape.k_max)
    n_near, differed, n_exact = H.check_routing(H.np_(ids), H.np_(w), ref)
    print(f"{shape.name}: near-tie tokens (<{H.NEAR_TIE:g}) {n_near}, differing among them "
          f"{differed}, exact ties (<{H.EXACT_TIE:g}) {n_exact}")


def _random_ids(T, E, k_max, k_t, rng, skew=None):
    ids = np.full((T, k_max), -1, dtype=np.int32)
    p = None
    if skew is not None:
        p = np.arange(1, E + 1, dtype=np.float64) ** -skew
        p /= p.sum()
    for t in range(T):
        ids[t, :k_t[t]] = rng.choice(E, size=int(k_t[t]), replace=False, p=p)
    return ids


@pytest.mark.parametrize("T,E,k_max,elastic,skew", [
    (1, 8, 2, False, None), (16, 8, 2, False, None), (37, 6, 3, False, 2.0),
    (2048, 512, 32, True, None), (8192, 256, 8, False, 1.2), (4096, 128, 8, False, 3.0),
    (333, 1, 1, False, None), (1000, 1024, 4, True, 0.5)])
def test_permute_matches_oracle_bit_exact(ops, T, E, k_max, elastic, skew):
    rng = np.random.default_rng(T * 7 + E)
    k_t = rng.integers(1, k_max + 1, size=T) if elastic else np.full(T, k_max)
    ids = _random_ids(T, E, k_max, k_t, rng, skew)
    kpt = torch.from_numpy(k_t.astype(np.int32)).cuda() if elastic else None
    offsets, perm, inv = ops.moe_permute(torch.from_numpy(ids).cuda(), k_max, kpt, E)
    H.check_grouping(H.np_(offsets), H.np_(perm), H.np_(inv), ids, k_t, E)


def test_permute_flags_out_of_range_expert_ids(ops):
    T, E, k_max = 10, 4, 2
    ids = np.tile(np.array([[0, 1]], dtype=np.int32), (T, 1))
    ids[3, 1] = 7                                    # not an expert
    dm = ops.dims(T, 16, E, 16, k_max)
    ws = ops.alloc_workspace(dm)
    offsets, perm, inv = ops.moe_permute(torch.from_numpy(ids).cuda(), k_max, None, E, ws=ws)
    assert ops.device_status(ws) == ops.MOE_ERR_DEVICE_CHECK
    assert H.np_(offsets)[E] == 2 * T - 1 and H.np_(inv)[3, 1] == -1


def test_permute_skips_unused_slots_without_a_report(ops):
    """-1 inside a token's k_t slots is an unused slot (the expert-parallel receiver's padding):
    skipped, not reported."""
    T, E, k_max = 10, 4, 3
    ids = np.tile(np.array([[2, 0, -1]], dtype=np.int32), (T, 1))
    ids[4] = [-1, -1, 3]
    dm = ops.dims(T, 16, E, 16, k_max)
    ws = ops.alloc_workspace(dm)
    offsets, perm, inv = ops.moe_permute(torch.from_numpy(ids).cuda(), k_max, None, E, ws=ws)
    assert ops.device_status(ws) == ops.MOE_OK
    pairs = sorted((int(ids[t, j]), t, j) for t in range(T) for j in range(k_max) if ids[t, j] >= 0)
    assert H.np_(offsets).tolist() == [sum(1 for p in pairs if p[0] < e) for e in range(E + 1)]
    assert H.np_(perm)[:len(pairs)].tolist() == [t for _, t, _ in pairs]
    inv = H.np_(inv)
    assert all(inv[t, j] == r for r, (_, t, j) in enumerate(pairs))
    assert (inv[ids < 0] == -1).all()


FFN_SHAPES = [
    I.WORKLOADS["tiny_T16"],
    I.MoEShape("ragged_K", 29, 192, 5, 96, 2, 2),        # K = 192, F = 96: partial tiles
    I.MoEShape("many_ntiles", 300, 256, 2, 128, 1, 1),   # 150 rows per expert
    I.MoEShape("wide", 24, 1024, 4, 512, 2, 2),
]


@pytest.mark.parametrize("shape", FFN_SHAPES, ids=lambda s: s.name)
def test_grouped_ffn_matches_oracle(ops, shape):
    inp = H.make_inputs(shape, seed=3)
    ref = H.run_oracle(inp)
    d = H.to_cuda(inp)
    offsets = torch.from_numpy(ref["offsets"].astype(np.int32)).cuda()
    perm = torch.full((shape.T * shape.k_max,), 0, dtype=torch.int32)
    perm[:len(ref["perm_token"])] = torch.from_numpy(ref["perm_token"])
    out, xs = ops.moe_grouped_ffn_fp8(d["hidden"], d["w13"], d["w13_scale"], d["w2"],
                                      d["w2_scale"], offsets, perm.cuda(), shape.k_max,
                                      want_act_scale=True)
    assert np.array_equal(H.np_(xs), ref["x_scale"])             # fp32 decisions: bit-exact
    R = int(ref["offsets"][-1])
    o = H.np_(out)[:R].astype(np.float64)
    o_ref = np.stack([ref["o_rows"][r] for r in range(R)])
    err = np.abs(o - o_ref)
    scale = max(1.0, np.abs(o_ref).max())
    rel = np.linalg.norm(o - o_ref) / np.linalg.norm(o_ref)
    print(f"{shape.name}: expert_out max|err| {err.max():.3e} (max|o| {np.abs(o_ref).max():.3e})"
          f" relL2 {rel:.3e}")
    assert err.max() <= H.Y_ATOL * scale and rel <= H.Y_REL_L2


def test_combine_matches_oracle(ops):
    shape = I.MoEShape("combine", 41, 128, 6, 64, 3, 3, F_shared=64)
    inp = H.make_inputs(shape, seed=5)
    ref = H.run_oracle(inp)
    R = int(ref["offsets"][-1])
    o = np.zeros((shape.T * shape.k_max, shape.d), dtype=np.float32)
    o[:R] = np.stack([ref["o_rows"][r] for r in range(R)]).astype(np.float32)
    so = ref["shared_out"].astype(np.float32)
    y, yf = ops.moe_combine(torch.from_numpy(o).cuda(),
                            torch.from_numpy(ref["topk_w"].astype(np.float32)).cuda(),
                            torch.from_numpy(ref["inv_row"]).cuda(),
                            torch.from_numpy(so).cuda(), want_f32=True)
    stats = H.check_output(y, yf, ref["y64"], "combine")
    assert stats["max_abs_f32"] <= 1e-5 * max(1.0, stats["max_abs_y"])
