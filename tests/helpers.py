"""Shared helpers of the tests: run the oracle on a seeded layer, move a layer to the GPU and
compare the CUDA path's outputs with the oracle's (tolerances stated here, once)."""
from __future__ import annotations

import numpy as np
import torch

from fp8_moe_layer_b200 import inputs as I
from oracle import moe_oracle as O

# ----------------------------------------------------------------------------- tolerances
# Routing weights: fp32 softmax of fp32 logits against the float64 oracle. |dw_j| <= 2 w_j
# max|dl|, and the rounding error of an fp32 dot product grows like sqrt(d): 2e-6 at d <= 512,
# scaled by sqrt(d / 512) above (7.5e-6 at d = 7168).
def weight_atol(d: int) -> float:
    return 2e-6 * max(1.0, (d / 512.0) ** 0.5)
# Output of the layer (bf16). The bar is max |err| <= 2e-2 and relative L2 <= 1e-2:
#  (i)   the fp32 sum before its bf16 rounding is within 2e-2 of the float64 result;
#  (ii)  the bf16 output is within 2e-2 + half a bf16 ulp of it (one more rounding of (i));
#  (iii) the relative L2 error of the bf16 output is <= 1e-2.
Y_ATOL = 2e-2
Y_REL_L2 = 1e-2
# Logit gap below which two experts count as a near tie (their order may legitimately differ
# between an fp32 and a float64 evaluation).
NEAR_TIE = 1e-4


def np_(t):
    return None if t is None else t.detach().cpu().numpy()


def hidden_bits(hidden: torch.Tensor) -> np.ndarray:
    return hidden.view(torch.int16).cpu().numpy().view(np.uint16)


def make_inputs(shape: I.MoEShape, seed: int = 0) -> I.MoEInputs:
    """Seeded layer; the FP8 weight cast runs on the GPU when there is one (same bytes)."""
    return I.make_inputs(shape, seed, quant_device="cuda" if torch.cuda.is_available() else None)


def run_oracle(inp: I.MoEInputs, tokens=None):
    s = inp.shape
    shared = None
    if s.F_shared:
        shared = (np_(inp.w13_shared), np_(inp.w13s_scale), np_(inp.w2_shared),
                  np_(inp.w2s_scale))
    return O.moe_forward(hidden_bits(inp.hidden), np_(inp.router_w), np_(inp.router_bias), s.k,
                         np_(inp.k_per_token), np_(inp.w13), np_(inp.w13_scale), np_(inp.w2),
                         np_(inp.w2_scale), shared=shared, tokens=tokens, k_max=s.k_max)


def to_cuda(inp: I.MoEInputs) -> dict:
    c = lambda t: None if t is None else t.cuda()
    out = dict(hidden=c(inp.hidden), router_w=c(inp.router_w), router_bias=c(inp.router_bias),
               k_per_token=c(inp.k_per_token), w13=c(inp.w13), w13_scale=c(inp.w13_scale),
               w2=c(inp.w2), w2_scale=c(inp.w2_scale), shared=None)
    if inp.shape.F_shared:
        out["shared"] = (c(inp.w13_shared), c(inp.w13s_scale), c(inp.w2_shared),
                         c(inp.w2s_scale))
    return out


def bf16_half_ulp(v: np.ndarray) -> np.ndarray:
    _, x = np.frexp(np.abs(v))
    return np.ldexp(1.0, np.maximum(x - 1, -126) - 8)


def order_tie_tokens(logits: np.ndarray, k_t: np.ndarray, gap: float = NEAR_TIE) -> np.ndarray:
    """Tokens with two of their k_t selected logits within ``gap`` of each other: the slot order
    of those two experts is not decided by fp32 vs float64 evaluation."""
    s = -np.sort(-logits, axis=-1)
    out = []
    for t in range(logits.shape[0]):
        kk = int(k_t[t])
        if kk > 1 and np.min(s[t, :kk - 1] - s[t, 1:kk]) < gap:
            out.append(t)
    return np.asarray(out, dtype=np.int64)


def check_routing(gpu_ids: np.ndarray, gpu_w: np.ndarray, ref: dict, d: int):
    """Routing parity.
    * Tokens without any near tie: ids bit-exact (set and slot order), weights within
      weight_atol(d).
    * Near tie at the k-th place (k-th and (k+1)-th oracle logits within NEAR_TIE): the GPU's
      choice must be a valid top-k -- k_t distinct experts, each within NEAR_TIE of the k-th.
    * Near tie inside the selection only: the SET is bit-exact, the GPU order is descending in
      the oracle logits up to NEAR_TIE, and each expert's weight matches.
    Returns (boundary near ties, how many of them chose differently, order-only near ties)."""
    logits, ids, w, k_t = ref["logits"], ref["topk_ids"], ref["topk_w"], ref["k_t"]
    atol = weight_atol(d)
    near = set(O.near_tie_tokens(logits, k_t, NEAR_TIE).tolist())
    order = set(order_tie_tokens(logits, k_t, NEAR_TIE).tolist()) - near
    differed = 0
    for t in range(ids.shape[0]):
        kt = int(k_t[t])
        assert np.all(gpu_ids[t, kt:] == -1) and np.all(gpu_w[t, kt:] == 0), t
        sel = gpu_ids[t, :kt]
        if t in near:
            if not np.array_equal(sel, ids[t, :kt]):
                differed += 1
                kth = np.sort(logits[t])[::-1][kt - 1]
                assert len(set(sel.tolist())) == kt
                assert np.all(logits[t, sel] >= kth - NEAR_TIE), t
            continue
        if t in order:
            assert set(sel.tolist()) == set(ids[t, :kt].tolist()), t
            assert np.all(np.diff(logits[t, sel]) <= NEAR_TIE), t
            ref_w = dict(zip(ids[t, :kt].tolist(), w[t, :kt].tolist()))
            assert max(abs(gpu_w[t, j] - ref_w[int(e)]) for j, e in enumerate(sel)) <= atol
            continue
        assert np.array_equal(sel, ids[t, :kt]), (t, gpu_ids[t], ids[t])
        assert np.abs(gpu_w[t, :kt] - w[t, :kt]).max() <= atol, (t, gpu_w[t], w[t])
    return len(near), differed, len(order)


def check_grouping(gpu_offsets, gpu_perm, gpu_inv, ids, k_t, E):
    """The GPU grouping must equal the oracle's counting sort of the SAME ids, bit for bit."""
    counts, offsets, perm, inv = O.group_by_expert(ids, k_t, E)
    R = int(offsets[-1])
    assert np.array_equal(gpu_offsets[:E + 1], offsets)
    assert np.array_equal(gpu_perm[:R], perm)
    assert np.array_equal(gpu_inv, inv)


def check_output(y_bf16: torch.Tensor, y_f32, y64: np.ndarray, what=""):
    """The layer-output bar (i)-(iii) above. Returns the measured errors."""
    yb = y_bf16.float().cpu().numpy().astype(np.float64)
    err_b = np.abs(yb - y64)
    stats = dict(max_abs_bf16=float(err_b.max()) if err_b.size else 0.0,
                 rel_l2=float(np.linalg.norm(yb - y64) / max(np.linalg.norm(y64), 1e-30)),
                 max_abs_y=float(np.abs(y64).max()) if y64.size else 0.0)
    if y_f32 is not None:
        yf = y_f32.cpu().numpy().astype(np.float64)
        stats["max_abs_f32"] = float(np.abs(yf - y64).max()) if yf.size else 0.0
        assert stats["max_abs_f32"] <= Y_ATOL, (what, stats)
    assert np.all(err_b <= Y_ATOL + bf16_half_ulp(y64)), (what, stats)
    assert stats["rel_l2"] <= Y_REL_L2, (what, stats)
    return stats
