"""Layer latency against the number of distinct active experts, at a fixed batch.

ELDR ("ELDR : Microsoft et KAIST accelerent le decodage des MoE", first paragraph) reports that
on Qwen3-30B-A3B a decode step's MoE-layer latency grows 4.7x when the batch activates 128
instead of 16 distinct experts, because every distinct expert's weights are read from HBM. This
sweep measures the same curve for this library on the Qwen3-30B-A3B layer shape (d=2048, E=128,
F=768, top-8): the router bias confines each batch to exactly n experts (a large positive bias on
n experts drawn at random, the router weights then spread the tokens over them), and the layer
is timed with CUDA events, L2 flushed between steps.

    python -m fp8_moe_layer_b200.expert_sweep --T 128 --active 16 32 64 128

Prints one JSON line per n: distinct experts seen, microseconds per layer, HBM bytes the step
must read (the active experts' weights and scales, router, hidden in and out) and their rate.
"""
from __future__ import annotations

import argparse
import json

import numpy as np
import torch

from . import inputs as I
from . import ops


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--T", type=int, default=128)
    ap.add_argument("--active", type=int, nargs="+", default=[16, 32, 64, 128])
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--seed", type=int, default=0)
    args = ap.parse_args()
    base = I.WORKLOADS["qwen3_T64"]
    shape = I.MoEShape(f"qwen3_T{args.T}", args.T, base.d, base.E, base.F, base.k, base.k_max)
    inp = I.make_inputs(shape, seed=args.seed, quant_device="cuda")
    layer = ops.MoELayerFP8(inp)
    h = inp.hidden.cuda()
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    flush_rd = torch.ones((256 << 20) // 4, dtype=torch.float32, device="cuda")
    gen = torch.Generator().manual_seed(args.seed + 1)
    per_expert = 3 * shape.d * shape.F + (2 * shape.F + shape.d) * 4
    results = []
    for n in args.active:
        chosen = torch.randperm(shape.E, generator=gen)[:n]
        bias = torch.full((shape.E,), -30.0)
        bias[chosen] = 0.0
        layer.router_bias = bias.cuda()
        _, dbg = layer(h, debug=True)
        counts = np.diff(dbg["expert_offsets"].cpu().numpy())
        active = int((counts > 0).sum())
        for _ in range(args.warmup):
            layer(h)
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(args.steps)]
        for i in range(args.steps):
            flush.fill_(i & 0xFF)
            flush_rd.sum()
            torch.cuda._sleep(400_000)     # ~0.2 ms: the host enqueues the step meanwhile
            ev[i][0].record()
            layer(h)
            ev[i][1].record()
        torch.cuda.synchronize()
        us = float(np.mean([a.elapsed_time(b) for a, b in ev])) * 1e3
        hbm = active * per_expert + shape.E * shape.d * 4 + 2 * shape.T * shape.d * 2
        row = dict(T=shape.T, n_target=n, active_experts=active, us_per_layer=round(us, 2),
                   hbm_bytes=hbm, hbm_gbs=round(hbm / (us * 1e-6) / 1e9, 1))
        results.append(row)
        print(json.dumps(row), flush=True)
    if len(results) > 1:
        r0, r1 = results[0], results[-1]
        print(json.dumps(dict(latency_ratio=round(r1["us_per_layer"] / r0["us_per_layer"], 2),
                              bytes_ratio=round(r1["hbm_bytes"] / r0["hbm_bytes"], 2),
                              experts=[r0["active_experts"], r1["active_experts"]])), flush=True)


if __name__ == "__main__":
    main()
