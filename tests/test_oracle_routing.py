"""Pins of the oracle's router (logits, top-k with ties, renormalised weights) and grouping
(stable counting sort by expert) against exact sums, brute force, library routines and
invariants."""
import itertools
import math

import numpy as np
import pytest
from scipy.special import softmax as scipy_softmax

from oracle import moe_oracle as O


def test_logits_match_correctly_rounded_sums():
    rng = np.random.default_rng(0)
    T, E, d = 5, 7, 300
    x = rng.normal(size=(T, d)).astype(np.float32)
    W = (rng.normal(size=(E, d)) * 0.02).astype(np.float32)
    b = rng.normal(size=E).astype(np.float32)
    l = O.router_logits(x.astype(np.float64), W, b)
    for t in range(T):
        for e in range(E):
            exact = math.fsum([float(x[t, i]) * float(W[e, i]) for i in range(d)] + [float(b[e])])
            scale = math.fsum(abs(float(x[t, i]) * float(W[e, i])) for i in range(d))
            assert abs(l[t, e] - exact) <= 1e-14 * max(scale, 1.0)
    # no bias -> the bias term really is absent
    l0 = O.router_logits(x.astype(np.float64), W, None)
    assert np.allclose(l - l0, b[None, :].astype(np.float64), atol=1e-12)


def _brute_topk(lrow, k):
    """The unique k-subset S such that every member beats every non-member (ties: lower index
    wins), listed by descending logit, lower index first among equals."""
    E = len(lrow)

    def beats(a, b):
        return lrow[a] > lrow[b] or (lrow[a] == lrow[b] and a < b)

    found = [S for S in itertools.combinations(range(E), k)
             if all(beats(a, b) for a in S for b in range(E) if b not in S)]
    assert len(found) == 1
    S = list(found[0])
    # order: insertion order by "beats"
    return sorted(S, key=lambda a: sum(beats(b, a) for b in S))


def test_topk_brute_force_with_ties():
    rng = np.random.default_rng(3)
    for trial in range(200):
        E = int(rng.integers(2, 7))
        k = int(rng.integers(1, E + 1))
        lrow = rng.integers(-3, 3, size=E).astype(np.float64)   # many exact ties
        ids = O.select_topk(lrow[None, :], np.array([k]), k)
        assert list(ids[0]) == _brute_topk(lrow, k), (lrow, k)


def test_topk_duplicate_router_rows_tie_to_lower_index():
    rng = np.random.default_rng(4)
    d, E = 64, 6
    W = rng.normal(size=(E, d))
    W[4] = W[1]                      # experts 1 and 4 produce identical logits
    W[1] *= 10.0
    W[4] = W[1]
    x = rng.normal(size=(3, d))
    x[:, :] = np.abs(x) * np.sign(W[1])[None, :]   # make experts 1/4 the clear winners
    l = O.router_logits(x, W)
    ids = O.select_topk(l, np.array([2, 2, 2]), 2)
    assert np.all(ids[:, 0] == 1) and np.all(ids[:, 1] == 4)


def test_weights_sum_to_one_and_special_cases():
    rng = np.random.default_rng(5)
    T, E = 40, 9
    l = rng.normal(size=(T, E)) * 2
    for k in range(1, E + 1):
        k_t = np.full(T, k)
        ids = O.select_topk(l, k_t, k)
        w = O.routing_weights(l, ids)
        assert np.allclose(w.sum(axis=1), 1.0, atol=1e-12)
        assert np.all(np.diff(w, axis=1) <= 1e-15)           # descending with the logits
        if k == 1:
            assert np.all(w[:, 0] == 1.0)
        if k == E:
            # k = E: plain softmax (library), reordered by the selection
            ref = scipy_softmax(l, axis=1)
            assert np.allclose(w, np.take_along_axis(ref, ids.astype(np.int64), 1), atol=1e-14)
    # renormalisation: w_j is proportional to exp(l_j) over the selection
    ids = O.select_topk(l, np.full(T, 3), 3)
    w = O.routing_weights(l, ids)
    for t in range(T):
        sel = l[t, ids[t]]
        ref = np.exp(sel - sel.max()) / np.exp(sel - sel.max()).sum()
        assert np.allclose(w[t], ref, rtol=1e-13)


def test_elastic_k_pads_unused_slots():
    rng = np.random.default_rng(6)
    l = rng.normal(size=(5, 12))
    k_t = np.array([1, 3, 12, 2, 5])
    ids = O.select_topk(l, k_t, 12)
    w = O.routing_weights(l, ids)
    for t in range(5):
        assert np.all(ids[t, k_t[t]:] == -1) and np.all(w[t, k_t[t]:] == 0)
        assert np.all(ids[t, :k_t[t]] >= 0)
        assert abs(w[t].sum() - 1) < 1e-12


def test_near_tie_detection():
    l = np.array([[3.0, 2.0, 1.99995, 0.0], [3.0, 2.0, 1.0, 0.0]])
    assert list(O.near_tie_tokens(l, np.array([2, 2]))) == [0]
    assert list(O.near_tie_tokens(l, np.array([1, 1]))) == []


@pytest.mark.parametrize("elastic", [False, True])
def test_grouping_matches_stable_argsort_and_invariants(elastic):
    rng = np.random.default_rng(7)
    T, E, k_max = 300, 11, 5
    k_t = rng.integers(1, k_max + 1, size=T) if elastic else np.full(T, 3)
    ids = np.full((T, k_max), -1, dtype=np.int32)
    for t in range(T):
        ids[t, :k_t[t]] = rng.choice(E, size=k_t[t], replace=False)
    counts, offsets, perm_token, inv_row = O.group_by_expert(ids, k_t, E)
    # library: stable argsort of the key (expert, token)
    tt, jj = np.nonzero(ids >= 0)
    ee = ids[tt, jj]
    order = np.argsort(ee.astype(np.int64) * T + tt, kind="stable")
    assert np.array_equal(perm_token, tt[order])
    assert np.array_equal(counts, np.bincount(ee, minlength=E))
    assert counts.sum() == k_t.sum() and offsets[-1] == k_t.sum() and offsets[0] == 0
    for t in range(T):
        for j in range(k_max):
            r = inv_row[t, j]
            if j >= k_t[t]:
                assert r == -1
                continue
            assert perm_token[r] == t
            e = ids[t, j]
            assert offsets[e] <= r < offsets[e + 1]
    # permute then unpermute is the identity
    payload = rng.normal(size=(T, 4))
    permuted = payload[perm_token]
    back = np.zeros((T, k_max, 4))
    for t in range(T):
        for j in range(k_t[t]):
            back[t, j] = permuted[inv_row[t, j]]
    for t in range(T):
        assert np.array_equal(back[t, :k_t[t]], np.repeat(payload[t][None], k_t[t], 0))
