"""Expert parallelism on one GPU: the dispatch kernel against the reference send plan (bit-exact),
and the whole expert-parallel layer -- n ranks, each with its own batch and E/n of the experts,
run in one process with the all-to-alls done as device copies -- against the oracle on every
rank's tokens."""
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


@pytest.fixture(scope="module")
def EP():
    from fp8_moe_layer_b200 import expert_parallel
    return expert_parallel


# (shape, ranks): T > 1024 crosses the plan kernel's token chunks; E / n < k_max gives fewer
# slots per row than k_max; n = 1 sends everything to one rank; n = 32 is the largest
PLAN_CASES = [
    (I.MoEShape("plan_T37_E16_k4", 37, 128, 16, 64, 4, 4), 4),
    (I.MoEShape("plan_T3000_E64_k8", 3000, 256, 64, 64, 8, 8), 8),
    (I.MoEShape("plan_elastic_T500", 500, 128, 64, 64, 2, 8, k_choices=(1, 2, 4, 8)), 4),
    (I.MoEShape("plan_E8_k2_n8", 129, 128, 8, 64, 2, 2), 8),
    (I.MoEShape("plan_n1", 50, 128, 16, 64, 4, 4), 1),
    (I.MoEShape("plan_n32", 300, 128, 64, 64, 8, 8), 32),
]


@pytest.mark.parametrize("shape,n", PLAN_CASES, ids=lambda c: getattr(c, "name", str(c)))
def test_dispatch_plan_bit_exact(ops, shape, n):
    hidden = I.make_hidden(shape, 3).cuda()
    rw, rb = I.make_router(shape, 3)
    kpt = I.make_k_per_token(shape, 3)
    kpt = None if kpt is None else kpt.cuda()
    ids, w = ops.moe_route_topk(hidden, rw.cuda(), None if rb is None else rb.cuda(), shape.k,
                                kpt, shape.k_max)
    ws = ops.alloc_workspace(ops.dims(shape.T, shape.d, shape.E, 16, shape.k_max))
    out = ops.moe_ep_dispatch(hidden, ids, w, shape.k, kpt, shape.E, n, ws=ws)
    assert ops.device_status(ws) == ops.MOE_OK
    k_t = O.token_k(shape.T, shape.k, None if kpt is None else H.np_(kpt))
    ref = H.ep_dispatch_reference(H.np_(ids), H.np_(w), k_t, shape.E, n)
    rows = len(ref["tokens"])
    assert np.array_equal(H.np_(out["send_counts"]), ref["counts"])
    assert np.array_equal(H.np_(out["slot_of"]), ref["slot_of"])
    assert np.array_equal(H.np_(out["slot_w"]), ref["slot_w"])
    assert np.array_equal(H.np_(out["send_ids"])[:rows], ref["send_ids"])
    assert np.array_equal(H.np_(out["send_w"])[:rows].view(np.uint32),
                          ref["send_w"].view(np.uint32))
    sent = out["send_hidden"][:rows].view(torch.int16).cpu()
    assert torch.equal(sent, hidden.view(torch.int16).cpu()[torch.from_numpy(ref["tokens"])])


def test_dispatch_flags_bad_routing_data(ops):
    """An expert id >= E and an expert selected twice are reported (MOE_ERR_DEVICE_CHECK) and
    left out of the plan; nothing is written out of bounds."""
    T, d, E, k_max, n = 8, 128, 8, 4, 4
    hidden = torch.randn(T, d, device="cuda").to(torch.bfloat16)
    ids = torch.tensor([[0, 2, 4, 6]] * T, dtype=torch.int32)
    ids[3, 1] = E + 3                 # out of range
    ids[5] = torch.tensor([1, 1, 1, 7])   # expert 1 (rank 0, E/n = 2 slots) three times
    w = torch.full((T, k_max), 0.25)
    ws = ops.alloc_workspace(ops.dims(T, d, E, 16, k_max))
    out = ops.moe_ep_dispatch(hidden, ids.cuda(), w.cuda(), k_max, None, E, n, ws=ws)
    assert ops.device_status(ws) == ops.MOE_ERR_DEVICE_CHECK
    slot_of = H.np_(out["slot_of"])
    # ranks hold experts {0,1} {2,3} {4,5} {6,7}; token 3 routes to 0, 4, 6 once id E+3 is dropped
    assert (slot_of[3] >= 0).tolist() == [True, False, True, True]
    # token 5: one row on rank 0 with its first two (of three) copies of expert 1, one on rank 3
    assert (slot_of[5] >= 0).tolist() == [True, False, False, True]
    assert H.np_(out["send_ids"])[slot_of[5, 0]].tolist() == [1, 1]
    for t in (0, 1, 2, 4, 6, 7):
        assert (slot_of[t] >= 0).all()
    assert H.np_(out["send_counts"]).sum() == (slot_of >= 0).sum()


def _ranks(EP, inp, n):
    s = inp.shape
    d = H.to_cuda(inp)
    El = s.E // n
    sl = lambda t, r: t[r * El:(r + 1) * El]
    return [EP.ExpertParallelRank(r, n, d["router_w"], d["router_bias"], s.k, s.k_max,
                                  sl(d["w13"], r), sl(d["w13_scale"], r), sl(d["w2"], r),
                                  sl(d["w2_scale"], r), shared=d["shared"])
            for r in range(n)]


# (shape, ranks, tokens per rank, idle): `idle` biases the router away from the last rank's
# experts, so that rank receives no rows
EP_CASES = [
    (I.MoEShape("ep2_E8_k2", 0, 256, 8, 128, 2, 2), 2, (40, 23), False),
    (I.MoEShape("ep4_shared_elastic", 0, 128, 16, 64, 2, 4, F_shared=64, k_choices=(1, 2, 4)),
     4, (31, 8, 50, 1), False),
    (I.MoEShape("ep8_E8_one_expert_per_rank", 0, 256, 8, 128, 2, 2), 8,
     (16, 9, 3, 20, 1, 5, 12, 7), False),
    (I.MoEShape("ep4_idle_rank_empty_batch", 0, 128, 16, 64, 3, 3), 4, (20, 0, 33, 5), True),
    (I.MoEShape("ep2_E64_k8_T300", 0, 256, 64, 128, 8, 8, zipf_s=1.0), 2, (300, 260), False),
]


@pytest.mark.parametrize("case", EP_CASES, ids=lambda c: c[0].name)
def test_expert_parallel_layer_matches_oracle(EP, case):
    shape, n, Ts, idle = case
    inp = H.make_inputs(shape, 0)
    if idle:
        bias = torch.zeros(shape.E)
        bias[(n - 1) * (shape.E // n):] = -30.0
        inp.router_bias = bias
    ranks = _ranks(EP, inp, n)
    hiddens, kpts = [], []
    for r, T in enumerate(Ts):
        sh = shape.with_T(T)
        hiddens.append(I.make_hidden(sh, 100 + r).cuda())
        kp = I.make_k_per_token(sh, 100 + r)
        kpts.append(None if kp is None else kp.cuda())
    ys = EP.loopback_forward(ranks, hiddens, kpts)
    for r, (y, T) in enumerate(zip(ys, Ts)):
        assert y.shape == (T, shape.d) and y.dtype == torch.bfloat16
        if T == 0:
            continue
        ref = H.run_oracle_on(inp, hiddens[r], kpts[r])
        H.check_output(y, None, ref["y64"], f"{shape.name} rank {r}")
