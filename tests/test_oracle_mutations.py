"""The oracle's pins are strong enough: each plausible mistake planted in the oracle (a dropped
term, a wrong sign or index, a swapped operand, a wrong rounding rule) makes a pin fail."""
import numpy as np
import pytest

from oracle import moe_oracle as O
from tests import test_oracle_ffn as FFN
from tests import test_oracle_formats as FMT
from tests import test_oracle_routing as ROUTE

_orig = {name: getattr(O, name) for name in
         ("expert_ffn", "router_logits", "select_topk", "group_by_expert", "quantize_rows_fp32",
          "combine", "e4m3_encode", "routing_weights", "silu")}


def ffn_swapped_gate_up(xq, xs, w13, s13, w2, s2w, return_intermediate=False):
    F = w2.shape[1]
    w13 = np.concatenate([w13[F:], w13[:F]])
    s13 = np.concatenate([s13[F:], s13[:F]])
    return _orig["expert_ffn"](xq, xs, w13, s13, w2, s2w, return_intermediate)


def ffn_scale_on_wrong_axis(xq, xs, w13, s13, w2, s2w, return_intermediate=False):
    o = _orig["expert_ffn"](xq, xs, w13, s13, w2, np.ones_like(s2w))
    return o * np.resize(np.asarray(s2w, np.float64), o.shape[0])[:, None]


def logits_without_bias(x, W, b=None):
    return _orig["router_logits"](x, W, None)


def topk_ties_to_higher(l, k_t, k_max):
    E = l.shape[1]
    return np.where(_orig["select_topk"](l[:, ::-1], k_t, k_max) >= 0,
                    E - 1 - _orig["select_topk"](l[:, ::-1], k_t, k_max), -1).astype(np.int32)


def grouping_tokens_descending(ids, k_t, E):
    counts, offsets, perm, inv = _orig["group_by_expert"](ids[::-1], k_t[::-1], E)
    T = ids.shape[0]
    return counts, offsets, (T - 1 - perm).astype(np.int32), inv[::-1]


def quant_wrong_max(a):
    a = np.asarray(a, np.float32)
    amax = np.abs(a).max(axis=-1)
    s = np.where(amax == 0, 1, amax / np.float32(447)).astype(np.float32)
    return O.e4m3_encode((a / s[..., None]).astype(np.float64)), s


def combine_unweighted(o_rows, weights, inv_row, k_t, tokens, shared_out=None):
    w = np.where(weights > 0, 1.0 / np.maximum(k_t[:, None], 1), 0.0)
    return _orig["combine"](o_rows, w, inv_row, k_t, tokens, shared_out)


def encode_ties_away(v):
    v = np.asarray(v, np.float64)
    nudged = v + np.sign(v) * np.abs(v) * 1e-12
    return _orig["e4m3_encode"](nudged)


def weights_not_renormalised(l, ids):
    p = O.softmax(l)
    w = np.zeros(ids.shape)
    for t in range(ids.shape[0]):
        sel = ids[t][ids[t] >= 0]
        w[t, :len(sel)] = p[t, sel]
    return w


def silu_wrong_sign(g):
    return g / (1.0 + np.exp(g))


SMALL_ZIPF = FFN.SMALL[1]
SMALL_UNI = FFN.SMALL[0]

MUTATIONS = [
    ("expert_ffn", ffn_swapped_gate_up, lambda: FFN.test_permuted_path_equals_dense_brute_force(SMALL_UNI)),
    ("expert_ffn", ffn_scale_on_wrong_axis, FFN.test_scale_placement),
    ("router_logits", logits_without_bias, lambda: FFN.test_permuted_path_equals_dense_brute_force(SMALL_ZIPF)),
    ("select_topk", topk_ties_to_higher, ROUTE.test_topk_brute_force_with_ties),
    ("group_by_expert", grouping_tokens_descending, lambda: ROUTE.test_grouping_matches_stable_argsort_and_invariants(False)),
    ("quantize_rows_fp32", quant_wrong_max, FFN.test_activation_quant_hits_448_and_matches_torch_cast),
    ("combine", combine_unweighted, lambda: FFN.test_permuted_path_equals_dense_brute_force(SMALL_UNI)),
    ("e4m3_encode", encode_ties_away, FMT.test_encode_midpoints_ties_to_even),
    ("routing_weights", weights_not_renormalised, ROUTE.test_weights_sum_to_one_and_special_cases),
    ("silu", silu_wrong_sign, lambda: FFN.test_permuted_path_equals_dense_brute_force(SMALL_UNI)),
]


@pytest.mark.parametrize("name,mutant,pin", MUTATIONS, ids=[m[1].__name__ for m in MUTATIONS])
def test_planted_mistake_is_caught(monkeypatch, name, mutant, pin):
    monkeypatch.setattr(O, name, mutant)
    with pytest.raises(AssertionError):
        pin()
