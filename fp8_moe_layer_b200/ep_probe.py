"""Time of the expert-parallel dispatch (moe_ep_dispatch: send plan + row gather) on one GPU,
against the HBM roofline of the bytes it must move.

Workload: the DeepSeek-V3 layer shape (d = 7168, E = 256, k = 8) with T = 8192 tokens on one of
n = 8 ranks; routing ids are the top-k of uniform random scores (distinct experts per token),
weights their renormalised softmax. Algorithmic bytes of one call: the hidden rows read once
(T * 2d), the ids and weights read (T * k * 8), the send rows written (rows * (2d + 8 * kl)) and
the combine map written (T * n * 8). Each timed call follows an L2 flush (a 512 MB write);
CUDA events on the launching stream, median of the calls.

    python -m fp8_moe_layer_b200.ep_probe [--T 8192 --ranks 8 --iters 20]
"""
import argparse
import json
import os
import statistics

import torch

from fp8_moe_layer_b200 import ops

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def hbm_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            return float(json.load(f)["hbm_gbs"]), "of measured"
    return 6650.0, "of fallback"


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--T", type=int, default=8192)
    ap.add_argument("--d", type=int, default=7168)
    ap.add_argument("--E", type=int, default=256)
    ap.add_argument("--k", type=int, default=8)
    ap.add_argument("--ranks", type=int, default=8)
    ap.add_argument("--iters", type=int, default=20)
    a = ap.parse_args()
    dev = torch.device("cuda")
    g = torch.Generator(device=dev)
    g.manual_seed(0)
    hidden = torch.randn(a.T, a.d, device=dev, generator=g).to(torch.bfloat16)
    scores = torch.rand(a.T, a.E, device=dev, generator=g)
    top = scores.topk(a.k, dim=1)
    ids = top.indices.to(torch.int32).contiguous()
    w = torch.softmax(top.values, dim=1).contiguous()
    ws = ops.alloc_workspace(ops.dims(a.T, a.d, a.E, 16, a.k))
    flush = torch.empty(512 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()
    times = []
    out = None
    for i in range(a.iters + 3):
        flush.fill_(i & 255)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        out = ops.moe_ep_dispatch(hidden, ids, w, a.k, None, a.E, a.ranks, ws=ws)
        e1.record(stream)
        torch.cuda.synchronize()
        if i >= 3:
            times.append(e0.elapsed_time(e1) * 1e3)
    assert ops.device_status(ws) == ops.MOE_OK
    counts = out["send_counts"].tolist()
    rows = sum(counts)
    kl = ops.ep_local_k(a.E, a.k, a.ranks)
    alg = a.T * 2 * a.d + a.T * a.k * 8 + rows * (2 * a.d + 8 * kl) + a.T * a.ranks * 8
    us = statistics.median(times)
    peak, src = hbm_peak()
    gbs = alg / (us * 1e-6) / 1e9
    print(json.dumps(dict(kernel="moe_ep_dispatch", T=a.T, d=a.d, E=a.E, k=a.k, ranks=a.ranks,
                          rows=rows, rows_per_token=rows / a.T, counts=counts,
                          alg_bytes=alg, us_median=round(us, 2),
                          us_min=round(min(times), 2), achieved_gbs=round(gbs, 1),
                          peak_gbs=peak, frac=round(gbs / peak, 3), peak_source=src,
                          note="includes the wrapper's output allocations; events bracket "
                               "the two kernels and the host call")))


if __name__ == "__main__":
    main()
