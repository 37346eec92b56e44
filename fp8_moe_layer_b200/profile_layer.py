"""Runs the fused layer a few times on one seeded workload, for profilers (Nsight Compute).

    python -m fp8_moe_layer_b200.profile_layer --workload mixtral_T512 --iters 3
    python -m fp8_moe_layer_b200.profile_layer --workload deepseek_T8192 --E 32 --T 1024

Each iteration is one moe_forward (8 kernels, in stage order: router logits, top-k + quant,
permute, gather, gate/up GEMM, requant, down GEMM, combine). Prints the per-stage device times
of the last iteration (CUDA events; not a benchmark number when run under a profiler).
"""
from __future__ import annotations

import argparse
import json

import torch

from . import inputs as I
from . import ops


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--workload", default="mixtral_T512")
    ap.add_argument("--iters", type=int, default=3)
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--E", type=int, default=0, help="fewer experts (same layer shape otherwise)")
    ap.add_argument("--T", type=int, default=0, help="another token count")
    args = ap.parse_args()
    shape = I.WORKLOADS[args.workload]
    if args.E or args.T:
        # a smaller case of the same kernels (e.g. for an Nsight Compute capture): the workload's
        # d, F, k, shared expert, router skew and k distribution, with E experts and T tokens
        E = args.E or shape.E
        shape = I.MoEShape(f"{shape.name.rsplit('_T', 1)[0]}_E{E}_T{args.T or shape.T}",
                           args.T or shape.T, shape.d, E, shape.F, shape.k, shape.k_max,
                           shape.F_shared, shape.zipf_s, shape.k_choices)
    inp = I.make_inputs(shape, seed=args.seed, quant_device="cuda")
    layer = ops.MoELayerFP8(inp)
    h = inp.hidden.cuda()
    kpt = None if inp.k_per_token is None else inp.k_per_token.cuda()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(ops.NUM_STAGES + 1)]
    for _ in range(args.iters):
        layer(h, kpt, stage_events=ev)
    torch.cuda.synchronize()
    status = ops.device_status(layer.ws)
    stages = {n: round(ev[i].elapsed_time(ev[i + 1]) * 1e3, 2)
              for i, n in enumerate(ops.STAGE_NAMES)}
    print(json.dumps(dict(workload=shape.name, status=status, stage_us=stages)))
    if status != ops.MOE_OK:
        raise SystemExit(f"device status {status}")


if __name__ == "__main__":
    main()
