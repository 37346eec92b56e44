"""Host side of k-aware batching: the tiers partition the tokens by k, keep each tier's tokens in
their original order, and come in ascending k."""
import numpy as np
import pytest
import torch

from fp8_moe_layer_b200.ktiers import k_tiers


@pytest.mark.parametrize("seed", range(5))
def test_tiers_partition_tokens_by_k(seed):
    rng = np.random.default_rng(seed)
    T = int(rng.integers(1, 300))
    k = rng.choice([2, 4, 8, 16, 32], size=T).astype(np.int32)
    tiers = k_tiers(torch.from_numpy(k))
    seen = np.concatenate([idx for _, idx in tiers])
    assert sorted(seen.tolist()) == list(range(T))                    # every token exactly once
    assert [kk for kk, _ in tiers] == sorted(set(k.tolist()))          # one tier per distinct k
    for kk, idx in tiers:
        assert np.all(k[idx] == kk)
        assert np.all(np.diff(idx) > 0)                                # original order kept


def test_single_k_is_one_tier():
    tiers = k_tiers(np.full(7, 4, dtype=np.int32))
    assert len(tiers) == 1 and tiers[0][0] == 4 and tiers[0][1].tolist() == list(range(7))


def test_empty_batch_has_no_tiers():
    assert k_tiers(np.zeros(0, dtype=np.int32)) == []
