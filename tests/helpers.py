"""Shared helpers of the tests: run the oracle on a seeded layer, move a layer to the GPU and
compare the CUDA path's outputs with the oracle's (tolerances stated here, once)."""
from __future__ import annotations

import numpy as np
import torch

from fp8_moe_layer_b200 import inputs as I
from oracle import moe_oracle as O

# ----------------------------------------------------------------------------- tolerances
# Routing decisions. Both sides take them in fp64: the kernels sum exact bf16 x fp32 products in
# fp64, the oracle uses numpy float64. Their logits then differ only by fp64 summation error, at
# most d * 2^-53 * sum|x w| (< 1e-10 for every workload here, ~3e-13 typical), so two logits closer
# than EXACT_TIE are the only ones whose order may legitimately differ. Every other token's ids
# must be bit-exact, set and slot order, including the tokens whose k-th and (k+1)-th logits lie
# within NEAR_TIE, which are only counted and reported separately.
EXACT_TIE = 1e-9
NEAR_TIE = 1e-4
# Routing weights: fp64 softmax over the selection of fp64 logits, rounded once to fp32 on the GPU,
# so |dw| <= 2^-24 w + 2 w max|dl| < 1e-7; the bar leaves a factor of 10.
WEIGHT_ATOL = 1e-6
# Output of the layer (bf16). The bar is max |err| <= 2e-2 and relative L2 <= 1e-2:
#  (i)   the fp32 sum before its bf16 rounding is within 2e-2 of the float64 result;
#  (ii)  the bf16 output is within 2e-2 + half a bf16 ulp of it (one more rounding of (i));
#  (iii) the relative L2 error of the bf16 output is <= 1e-2.
Y_ATOL = 2e-2
Y_REL_L2 = 1e-2


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


def run_oracle_on(inp: I.MoEInputs, hidden: torch.Tensor, k_per_token=None):
    """The oracle on other tokens of the same layer (hidden bf16 [n, d], k_per_token [n] or None):
    every step is per token, so a batch's outputs do not depend on the other tokens in it."""
    s = inp.shape
    shared = None
    if s.F_shared:
        shared = (np_(inp.w13_shared), np_(inp.w13s_scale), np_(inp.w2_shared),
                  np_(inp.w2s_scale))
    return O.moe_forward(hidden_bits(hidden.cpu()), np_(inp.router_w), np_(inp.router_bias), s.k,
                         np_(k_per_token), np_(inp.w13), np_(inp.w13_scale), np_(inp.w2),
                         np_(inp.w2_scale), shared=shared, k_max=s.k_max)


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


def exact_tie_tokens(logits: np.ndarray, k_t: np.ndarray, gap: float = EXACT_TIE) -> np.ndarray:
    """Tokens with two of their k_t + 1 largest logits within ``gap`` of each other: inside the
    selection (slot order) or at its boundary (the set). fp64 summation order decides those."""
    s = -np.sort(-logits, axis=-1)
    out = []
    for t in range(logits.shape[0]):
        kk = min(int(k_t[t]) + 1, logits.shape[1])
        if kk > 1 and np.min(s[t, :kk - 1] - s[t, 1:kk]) < gap:
            out.append(t)
    return np.asarray(out, dtype=np.int64)


def check_routing(gpu_ids: np.ndarray, gpu_w: np.ndarray, ref: dict, d: int = 0):
    """Routing parity against the oracle's fp64 decision.
    * Every token without an exact tie (EXACT_TIE): ids bit-exact, set and slot order, and
      weights within WEIGHT_ATOL. This includes the tokens whose k-th and (k+1)-th oracle logits
      differ by less than NEAR_TIE; they are counted and reported separately.
    * A token with an exact tie: the GPU's choice must be a valid top-k (k_t distinct experts,
      each within EXACT_TIE of the k-th logit, descending up to EXACT_TIE), and each selected
      expert's weight must match the oracle's weight of that expert when it selected it too.
    Unused slots hold id -1 and weight 0. Returns (near-tie tokens, how many of them chose
    differently from the oracle, exact-tie tokens)."""
    logits, ids, w, k_t = ref["logits"], ref["topk_ids"], ref["topk_w"], ref["k_t"]
    near = set(O.near_tie_tokens(logits, k_t, NEAR_TIE).tolist())
    exact = set(exact_tie_tokens(logits, k_t, EXACT_TIE).tolist())
    near_differed = 0
    for t in range(ids.shape[0]):
        kt = int(k_t[t])
        assert np.all(gpu_ids[t, kt:] == -1) and np.all(gpu_w[t, kt:] == 0), t
        sel = gpu_ids[t, :kt]
        same = np.array_equal(sel, ids[t, :kt])
        if t in near and not same:
            near_differed += 1
        if t in exact:
            kth = np.sort(logits[t])[::-1][kt - 1]
            assert len(set(sel.tolist())) == kt, t
            assert np.all(logits[t, sel] >= kth - EXACT_TIE), t
            assert np.all(np.diff(logits[t, sel]) <= EXACT_TIE), t
            ref_w = dict(zip(ids[t, :kt].tolist(), w[t, :kt].tolist()))
            for j, e in enumerate(sel.tolist()):
                if e in ref_w:
                    assert abs(gpu_w[t, j] - ref_w[e]) <= WEIGHT_ATOL * 10, (t, e)
            continue
        assert same, (t, gpu_ids[t], ids[t], logits[t, ids[t, :kt]])
        assert np.abs(gpu_w[t, :kt] - w[t, :kt]).max() <= WEIGHT_ATOL, (t, gpu_w[t], w[t])
    return len(near), near_differed, len(exact)


def check_grouping(gpu_offsets, gpu_perm, gpu_inv, ids, k_t, E, ref_ids=None):
    """The GPU grouping must equal the oracle's counting sort of the SAME ids, bit for bit; and,
    when the GPU's ids equal the oracle's own (``ref_ids``), the oracle's grouping itself."""
    counts, offsets, perm, inv = O.group_by_expert(ids, k_t, E)
    R = int(offsets[-1])
    assert np.array_equal(gpu_offsets[:E + 1], offsets)
    assert np.array_equal(gpu_perm[:R], perm)
    assert np.array_equal(gpu_inv, inv)
    assert R == int(np.sum(k_t))                        # expert counts sum to sum_t k_t
    if ref_ids is not None and np.array_equal(ids, ref_ids):
        _, o_off, o_perm, o_inv = O.group_by_expert(ref_ids, k_t, E)
        assert np.array_equal(gpu_offsets[:E + 1], o_off)
        assert np.array_equal(gpu_perm[:R], o_perm) and np.array_equal(gpu_inv, o_inv)
        return True
    return False


def coverage_tokens(offsets: np.ndarray, perm: np.ndarray, E: int, T: int, n_random: int,
                    seed: int = 0, shared: bool = False) -> np.ndarray:
    """A token sample for the full-size workloads that reaches every GEMM tile kind: for every
    active expert the tokens of its first and last routed rows (its first tile and its ragged
    tail tile), the last token (the shared expert's tail), and ``n_random`` tokens at random."""
    pick = set()
    for e in range(E):
        a, b = int(offsets[e]), int(offsets[e + 1])
        if b > a:
            pick.add(int(perm[a]))
            pick.add(int(perm[b - 1]))
    if shared:
        pick.add(T - 1)
    rest = np.setdiff1d(np.arange(T), np.fromiter(pick, dtype=np.int64, count=len(pick)))
    rng = np.random.default_rng(seed)
    if len(rest):
        pick.update(rng.choice(rest, size=min(n_random, len(rest)), replace=False).tolist())
    return np.array(sorted(pick), dtype=np.int64)


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


def ep_dispatch_reference(ids: np.ndarray, w: np.ndarray, k_t: np.ndarray, E: int, n_ranks: int):
    """The expert-parallel send plan written out with loops: one row per (rank, token) pair where
    the rank holds one of the token's selected experts, rows ordered by rank then token; a row's
    local ids (global id - rank * E/n) and weights in slot order, padded with -1 / 0 to
    kl = min(k_max, E/n) slots."""
    T, k_max = ids.shape
    El = E // n_ranks
    kl = min(k_max, El)
    tokens, rids, rw = [], [], []
    counts = np.zeros(n_ranks, dtype=np.int64)
    slot_of = np.full((T, n_ranks), -1, dtype=np.int32)
    for r in range(n_ranks):
        for t in range(T):
            sel = [j for j in range(int(k_t[t])) if r * El <= ids[t, j] < (r + 1) * El]
            if not sel:
                continue
            slot_of[t, r] = len(tokens)
            tokens.append(t)
            rids.append([int(ids[t, j]) - r * El for j in sel] + [-1] * (kl - len(sel)))
            rw.append([float(w[t, j]) for j in sel] + [0.0] * (kl - len(sel)))
            counts[r] += 1
    return dict(tokens=np.array(tokens, dtype=np.int64),
                send_ids=np.array(rids, dtype=np.int32).reshape(-1, kl),
                send_w=np.array(rw, dtype=np.float32).reshape(-1, kl),
                counts=counts, slot_of=slot_of,
                slot_w=(slot_of >= 0).astype(np.float32), kl=kl)
