"""The measurement arithmetic behind every roofline fraction (CPU): algorithmic bytes and flops
of a step against the closed forms of the workloads, and the sweep's counting of distinct active
experts from a step's own grouping (the same as the bench's)."""
import numpy as np
import pytest

import bench
from fp8_moe_layer_b200 import inputs as I
from fp8_moe_layer_b200 import workload_sweep as WS


def _offsets(counts):
    return np.concatenate([[0], np.cumsum(counts)]).astype(np.int64)


@pytest.mark.parametrize("name,active,expect_mb", [
    # Mixtral-8x7B shape: 2 (T=1) or all 8 experts active; 3dF FP8 weight bytes + (2F + d) fp32
    # scales per expert, E d fp32 router weights, T d bf16 in and out
    ("mixtral_T1", 2, 352.7), ("mixtral_T32", 8, 1411.0), ("mixtral_T512", 8, 1419.0),
    ("qwen3_T1", 8, 38.9),
])
def test_step_bytes_match_the_closed_form(name, active, expect_mb):
    s = I.WORKLOADS[name]
    counts = np.zeros(s.E, dtype=np.int64)
    counts[:active] = s.T * s.k // active
    counts[0] += s.T * s.k - counts.sum()
    w = bench.algorithmic(s, _offsets(counts))
    assert w["active_experts"] == active and w["routed_rows"] == s.T * s.k
    assert abs(w["bytes"] / 1e6 - expect_mb) < 0.05 * expect_mb
    # exact closed form
    per_expert = 3 * s.d * s.F + (2 * s.F + s.d) * 4
    assert w["bytes"] == active * per_expert + s.E * s.d * 4 + 4 * s.T * s.d
    assert w["flops"] == 6 * s.d * s.F * s.T * s.k + 2 * s.T * s.E * s.d


def test_shared_expert_counts_as_one_more_active_expert_and_T_more_rows():
    s = I.WORKLOADS["deepseek_T128"]
    counts = np.zeros(s.E, dtype=np.int64)
    counts[:64] = s.T * s.k // 64
    w = bench.algorithmic(s, _offsets(counts))
    assert w["active_experts"] == 65
    assert w["flops"] == 6 * s.d * s.F * (s.T * s.k + s.T) + 2 * s.T * s.E * s.d


def test_sweep_and_bench_count_the_same_work():
    s = I.WORKLOADS["qwen3_T64"]
    rng = np.random.default_rng(0)
    counts = rng.multinomial(s.T * s.k, np.ones(s.E) / s.E)
    counts[:10] = 0                                   # some experts idle
    off = _offsets(counts)
    active, R, B, flops = WS.work(s, off)
    w = bench.algorithmic(s, off)
    assert (active, R, B, flops) == (w["active_experts"], w["routed_rows"], w["bytes"], w["flops"])
    assert active == int((counts > 0).sum())

