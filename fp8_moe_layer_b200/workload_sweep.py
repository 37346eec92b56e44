"""Every workload of the layer, timed on the device, against its roofline.

    python -m fp8_moe_layer_b200.workload_sweep [--workloads mixtral_T1 qwen3_T4096 ...]

For each workload: microseconds per layer (CUDA events around moe_forward, L2 flushed between
steps; for T <= 512 also replayed from a captured CUDA graph), tokens/s, the step's algorithmic HBM bytes (the distinct active experts' weights and
scales from the step's own routing, the router weights, bf16 hidden in and out) and FLOPs
(6 d F per routed row and shared-expert row, 2 T E d for the router), the roofline time
max(bytes / HBM, flops / FP8 peak) and the achieved fraction of it. HBM is the measured copy
bandwidth (MEASURED_PEAKS.json); the FP8 tensor-core peak is measured here with cuBLAS
(torch._scaled_mm, 8192^3 e4m3 -> bf16, best of 10). A second pass records per-kernel times.
"""
from __future__ import annotations

import argparse
import json
import os

import numpy as np
import torch

from . import inputs as I
from . import ops

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def fp8_peak_tflops(n: int = 8192, reps: int = 10) -> float:
    a = torch.randn(n, n, device="cuda").to(torch.float8_e4m3fn)
    b = torch.randn(n, n, device="cuda").to(torch.float8_e4m3fn)
    one = torch.tensor(1.0, device="cuda")
    best = float("inf")
    for _ in range(reps + 2):
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record()
        torch._scaled_mm(a, b.t(), scale_a=one, scale_b=one, out_dtype=torch.bfloat16)
        e.record()
        torch.cuda.synchronize()
        best = min(best, s.elapsed_time(e))
    return 2.0 * n ** 3 / (best * 1e-3) / 1e12


def hbm_gbs() -> float:
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        return float(json.load(open(path))["hbm_gbs"])
    return 6650.0


def work(shape, offsets):
    counts = np.diff(offsets[: shape.E + 1])
    active = int((counts > 0).sum()) + (1 if shape.F_shared else 0)
    R = int(offsets[shape.E])
    rows = R + (shape.T if shape.F_shared else 0)
    B = active * (3 * shape.d * shape.F + (2 * shape.F + shape.d) * 4) + shape.E * shape.d * 4 \
        + 2 * shape.T * shape.d * 2
    flops = 6 * shape.d * shape.F * rows + 2 * shape.T * shape.E * shape.d
    return active, R, B, flops


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--workloads", nargs="+", default=[n for n in I.WORKLOADS if n != "tiny_T16"])
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    args = ap.parse_args()
    peak_fp8 = fp8_peak_tflops()
    bw = hbm_gbs()
    print(json.dumps(dict(fp8_peak_tflops_cublas=round(peak_fp8, 1), hbm_gbs=bw)), flush=True)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    flush_rd = torch.ones((256 << 20) // 4, dtype=torch.float32, device="cuda")
    for name in args.workloads:
        shape = I.WORKLOADS[name]
        inp = I.make_inputs(shape, seed=0, quant_device="cuda")
        layer = ops.MoELayerFP8(inp)
        h = inp.hidden.cuda()
        kpt = None if inp.k_per_token is None else inp.k_per_token.cuda()
        _, dbg = layer(h, kpt, debug=True)
        active, R, B, flops = work(shape, dbg["expert_offsets"].cpu().numpy())
        for _ in range(args.warmup):
            layer(h, kpt)
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(args.steps)]
        for i in range(args.steps):
            flush.fill_(i & 0xFF)
            flush_rd.sum()
            torch.cuda._sleep(400_000)     # ~0.2 ms: the host enqueues the step meanwhile
            ev[i][0].record()
            layer(h, kpt)
            ev[i][1].record()
        torch.cuda.synchronize()
        us = float(np.median([a.elapsed_time(b) for a, b in ev])) * 1e3
        st = [[torch.cuda.Event(enable_timing=True) for _ in range(ops.NUM_STAGES + 1)]
              for _ in range(args.steps)]
        for i in range(args.steps):
            flush.fill_(i & 0xFF)
            flush_rd.sum()
            torch.cuda._sleep(400_000)     # ~0.2 ms: the host enqueues the step meanwhile
            layer(h, kpt, stage_events=st[i])
        torch.cuda.synchronize()
        stage = np.median(np.array([[st[i][j].elapsed_time(st[i][j + 1])
                                     for j in range(ops.NUM_STAGES)] for i in range(args.steps)]),
                          axis=0) * 1e3
        us_graph = None
        if shape.T <= 512:
            # the same step replayed from a captured CUDA graph (graphs.MoEGraphExecutor)
            from .graphs import MoEGraphExecutor
            ex = MoEGraphExecutor(layer, buckets=(shape.T,))
            for _ in range(args.warmup):
                ex(h, kpt)
            gev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                   for _ in range(args.steps)]
            for i in range(args.steps):
                flush.fill_(i & 0xFF)
                flush_rd.sum()
                torch.cuda._sleep(400_000)     # ~0.2 ms: the host enqueues the step meanwhile
                gev[i][0].record()
                ex(h, kpt)
                gev[i][1].record()
            torch.cuda.synchronize()
            us_graph = round(float(np.median([a.elapsed_time(b) for a, b in gev])) * 1e3, 2)
            del ex
        t_hbm = B / (bw * 1e9) * 1e6
        t_fp8 = flops / (peak_fp8 * 1e12) * 1e6
        t_roof = max(t_hbm, t_fp8)
        status = ops.device_status(layer.ws)
        print(json.dumps(dict(
            workload=name, T=shape.T, us_per_layer=round(us, 2), us_per_layer_graph=us_graph,
            tokens_per_s=round(shape.T / (us * 1e-6)), active_experts=active, routed_rows=R,
            hbm_bytes=B, flops=flops, t_hbm_us=round(t_hbm, 2), t_fp8_us=round(t_fp8, 2),
            binds="hbm" if t_hbm >= t_fp8 else "fp8", roofline_frac=round(t_roof / us, 3),
            roofline_frac_graph=None if us_graph is None else round(t_roof / us_graph, 3),
            status=status,
            stage_us={n: round(float(v), 1) for n, v in zip(ops.STAGE_NAMES, stage)})),
            flush=True)
        del layer, inp
        torch.cuda.empty_cache()


if __name__ == "__main__":
    main()
