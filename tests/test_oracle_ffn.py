"""Pins of the oracle's quantisation, expert FFN and combine: brute-force dense evaluation of
every expert per token (torch float64, torch's FP8 casts), closed-form special cases and
invariants of the whole layer."""
import numpy as np
import pytest
import torch

from fp8_moe_layer_b200 import inputs as I
from oracle import moe_oracle as O


def _np(t):
    return None if t is None else t.numpy()


def run_oracle(inp: I.MoEInputs, tokens=None):
    s = inp.shape
    shared = None
    if s.F_shared:
        shared = (inp.w13_shared.numpy(), inp.w13s_scale.numpy(), inp.w2_shared.numpy(),
                  inp.w2s_scale.numpy())
    return O.moe_forward(inp.hidden.view(torch.int16).numpy().view(np.uint16),
                         inp.router_w.numpy(), _np(inp.router_bias), s.k, _np(inp.k_per_token),
                         inp.w13.numpy(), inp.w13_scale.numpy(), inp.w2.numpy(),
                         inp.w2_scale.numpy(), shared=shared, tokens=tokens, k_max=s.k_max)


# ---------------------------------------------------------------- independent dense reference
def _t_dq(codes):
    return torch.from_numpy(np.ascontiguousarray(codes)).view(torch.float8_e4m3fn).to(
        torch.float64)


def _t_quant_rows(a32: torch.Tensor):
    amax = a32.abs().amax(dim=-1)
    s = torch.where(amax > 0, amax / 448.0, torch.ones_like(amax))
    return (a32 / s[:, None]).to(torch.float8_e4m3fn).to(torch.float64), s.to(torch.float64)


def dense_expert(x32, w13, s13, w2, s2w):
    """One expert on every given token, torch float64 (library casts for FP8)."""
    xq, xs = _t_quant_rows(x32)
    F = w2.shape[1]
    h = (xq @ _t_dq(w13).T) * xs[:, None] * torch.from_numpy(s13).double()[None, :]
    g, u = h[:, :F], h[:, F:]
    act = g * torch.sigmoid(g) * u
    aq, s2 = _t_quant_rows(act.float())
    return (aq @ _t_dq(w2).T) * s2[:, None] * torch.from_numpy(s2w).double()[None, :]


def brute_force_layer(inp: I.MoEInputs):
    """Evaluate EVERY expert on every token densely, then mask to the chosen top-k."""
    s = inp.shape
    x32 = inp.hidden.float()
    logits = x32.double() @ inp.router_w.double().T
    if inp.router_bias is not None:
        logits = logits + inp.router_bias.double()[None, :]
    probs = torch.softmax(logits, dim=1)
    k_t = [s.k] * s.T if inp.k_per_token is None else inp.k_per_token.tolist()
    dense = [dense_expert(x32, inp.w13[e].numpy(), inp.w13_scale[e].numpy(), inp.w2[e].numpy(),
                          inp.w2_scale[e].numpy()) for e in range(s.E)]
    y = torch.zeros(s.T, s.d, dtype=torch.float64)
    for t in range(s.T):
        order = sorted(range(s.E), key=lambda e: (-logits[t, e].item(), e))[:k_t[t]]
        p = probs[t, order]
        w = p / p.sum()
        for wj, e in zip(w, order):
            y[t] += wj * dense[e][t]
    if s.F_shared:
        y += dense_expert(x32, inp.w13_shared.numpy(), inp.w13s_scale.numpy(),
                          inp.w2_shared.numpy(), inp.w2s_scale.numpy())
    return y.numpy()


SMALL = [
    I.MoEShape("small_uniform", 24, 64, 6, 96, 2, 2),
    I.MoEShape("small_zipf_shared", 20, 48, 5, 32, 3, 3, F_shared=32, zipf_s=1.2),
    I.MoEShape("small_elastic", 18, 32, 8, 48, 2, 8, k_choices=(1, 2, 4, 8)),
    I.WORKLOADS["tiny_T16"],
]


@pytest.mark.parametrize("shape", SMALL, ids=lambda s: s.name)
def test_permuted_path_equals_dense_brute_force(shape):
    inp = I.make_inputs(shape, seed=11)
    out = run_oracle(inp)
    ref = brute_force_layer(inp)
    err = np.abs(out["y64"] - ref).max()
    assert err <= 1e-12 * max(1.0, np.abs(ref).max()), err


def test_single_expert_is_dense_quantised_swiglu():
    shape = I.MoEShape("one_expert", 10, 64, 1, 128, 1, 1)
    inp = I.make_inputs(shape, seed=3)
    out = run_oracle(inp)
    ref = dense_expert(inp.hidden.float(), inp.w13[0].numpy(), inp.w13_scale[0].numpy(),
                       inp.w2[0].numpy(), inp.w2_scale[0].numpy()).numpy()
    assert np.allclose(out["topk_w"][:, 0], 1.0)
    assert np.abs(out["y64"] - ref).max() <= 1e-12 * np.abs(ref).max()


def test_zero_down_weights_and_zero_tokens_give_zero():
    shape = I.MoEShape("zeros", 8, 32, 4, 32, 2, 2)
    inp = I.make_inputs(shape, seed=5)
    inp.w2.zero_()
    assert np.all(run_oracle(inp)["y64"] == 0)
    inp = I.make_inputs(shape, seed=5)
    inp.hidden[3].zero_()
    out = run_oracle(inp)
    assert out["x_scale"][3] == 1.0 and np.all(out["xq"][3] == 0)
    assert np.all(out["y64"][3] == 0)


def test_activation_quant_hits_448_and_matches_torch_cast():
    rng = np.random.default_rng(9)
    a = (rng.normal(size=(50, 77)) * rng.uniform(0.01, 100, size=(50, 1))).astype(np.float32)
    a[7] = 0
    q, s = O.quantize_rows_fp32(a)
    assert s[7] == 1.0 and np.all(q[7] == 0)
    for r in range(50):
        if r == 7:
            continue
        i = np.argmax(np.abs(a[r]))
        assert q[r, i] in (0x7E, 0xFE)
    ref, sref = _t_quant_rows(torch.from_numpy(a))
    assert np.array_equal(s, sref.float().numpy())
    assert np.array_equal(O.e4m3_decode(q), ref.numpy())


def test_scale_placement():
    """Doubling the up-projection scales or the down scales doubles y exactly; the gate scales
    do not (silu is not linear) -- pins where each per-channel scale enters."""
    shape = I.MoEShape("scales", 12, 32, 4, 64, 2, 2)
    inp = I.make_inputs(shape, seed=8)
    y0 = run_oracle(inp)["y64"]
    up = I.make_inputs(shape, seed=8)
    up.w13_scale[:, shape.F:] *= 2
    assert np.allclose(run_oracle(up)["y64"], 2 * y0, rtol=1e-13, atol=0)
    dn = I.make_inputs(shape, seed=8)
    dn.w2_scale *= 2
    assert np.allclose(run_oracle(dn)["y64"], 2 * y0, rtol=1e-13, atol=0)
    one = I.make_inputs(shape, seed=8)
    one.w2_scale[:, 5] *= 2                       # one output channel of the down projection
    y1 = run_oracle(one)["y64"]
    assert np.allclose(y1[:, 5], 2 * y0[:, 5], rtol=1e-13, atol=0)
    assert np.array_equal(np.delete(y1, 5, axis=1), np.delete(y0, 5, axis=1))
    gt = I.make_inputs(shape, seed=8)
    gt.w13_scale[:, :shape.F] *= 2
    assert not np.allclose(run_oracle(gt)["y64"], 2 * y0, rtol=1e-3)


def test_token_order_is_restored():
    """Permuting the tokens permutes the outputs the same way (combine restores token order)."""
    shape = I.MoEShape("perm", 30, 32, 7, 32, 3, 3, zipf_s=1.0)
    inp = I.make_inputs(shape, seed=2)
    out = run_oracle(inp)
    perm = torch.randperm(shape.T, generator=torch.Generator().manual_seed(1))
    inp2 = I.make_inputs(shape, seed=2)
    inp2.hidden = inp.hidden[perm].contiguous()
    out2 = run_oracle(inp2)
    assert np.array_equal(out2["y_bf16"], out["y_bf16"][perm.numpy()])
    assert np.array_equal(out2["topk_ids"], out["topk_ids"][perm.numpy()])


def test_token_subset_matches_full_run():
    shape = I.MoEShape("subset", 25, 32, 6, 32, 2, 2, F_shared=32)
    inp = I.make_inputs(shape, seed=4)
    full = run_oracle(inp)
    sub = np.array([0, 3, 17, 24])
    part = run_oracle(inp, tokens=sub)
    assert np.array_equal(part["y64"], full["y64"][sub])


def test_shared_expert_adds_dense_ffn_with_weight_one():
    shape = I.MoEShape("shared", 12, 32, 4, 32, 2, 2, F_shared=32)
    inp = I.make_inputs(shape, seed=6)
    with_shared = run_oracle(inp)["y64"]
    inp_ns = I.make_inputs(shape, seed=6)
    inp_ns.shape = I.MoEShape("noshared", 12, 32, 4, 32, 2, 2)
    without = run_oracle(inp_ns)["y64"]
    dense = dense_expert(inp.hidden.float(), inp.w13_shared.numpy(), inp.w13s_scale.numpy(),
                         inp.w2_shared.numpy(), inp.w2s_scale.numpy()).numpy()
    assert np.abs(with_shared - without - dense).max() <= 1e-12 * np.abs(dense).max()
