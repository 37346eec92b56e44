"""k-aware batching on the host: a batch with per-token k split into tiers of equal k.

"MoE-Prism" (gist.science), section 2B, describes a k-aware runtime: requests are grouped by their
routing budget k so that each group runs a MoE segment specialised (and graph-captured) for that
k. The kernels of this library read k_t per token, so a mixed-k batch already runs in one
``moe_forward`` call (and one "elastic" graph). This module is the tiered alternative for an
engine that keeps one fixed-k graph per tier: the tokens of each distinct k are gathered (in
their original order), run as a fixed-k call, and their outputs scattered back. Every token's
routing and output are those of the one-call elastic layer; only the grouping of the work, and
so the K-split choices of each call, differ.

    python -m fp8_moe_layer_b200.ktiers [--workloads prism_T64 prism_T2048]

times the elastic single call against the tiered calls (eager, and replayed from fixed-k graphs
for T <= 512) on the MoE-Prism-shaped layer, L2 flushed between steps.
"""
from __future__ import annotations

import argparse
import json
from typing import Dict, List, Optional, Tuple

import numpy as np
import torch


def k_tiers(k_per_token) -> List[Tuple[int, np.ndarray]]:
    """Partition of the token indices by k: [(k, indices in ascending order)], k ascending."""
    k = np.asarray(k_per_token.cpu() if isinstance(k_per_token, torch.Tensor) else k_per_token)
    if k.ndim != 1:
        raise ValueError("k_per_token must be one-dimensional")
    order = np.argsort(k, kind="stable")
    ks = k[order]
    cuts = np.flatnonzero(np.diff(ks)) + 1
    return [(int(ks[g[0]]), np.sort(order[g])) for g in np.split(np.arange(len(k)), cuts)
            if len(g)]


class KTieredLayer:
    """Runs a per-token-k batch of an ``ops.MoELayerFP8`` as one fixed-k call per distinct k.

    ``graphs=True`` replays each tier from a CUDA graph captured for (token bucket, that k)
    (``graphs.MoEGraphExecutor``, one executor per k)."""

    def __init__(self, layer, graphs: bool = False,
                 buckets=(1, 2, 4, 8, 16, 32, 64, 128, 256, 512)):
        self.layer = layer
        self.graphs = graphs
        self.buckets = buckets
        self._ex: Dict[int, object] = {}

    def _run(self, k: int, h: torch.Tensor) -> torch.Tensor:
        if not self.graphs:
            return self.layer(h, k=k)
        if k not in self._ex:
            from .graphs import MoEGraphExecutor
            self._ex[k] = MoEGraphExecutor(self.layer, buckets=self.buckets, k=k)
        return self._ex[k](h)

    def __call__(self, hidden: torch.Tensor, k_per_token_host,
                 y: Optional[torch.Tensor] = None) -> torch.Tensor:
        T, d = hidden.shape
        y = torch.empty(T, d, dtype=torch.bfloat16, device=hidden.device) if y is None else y
        for k, idx in k_tiers(k_per_token_host):
            if len(idx) == T:
                y.copy_(self._run(k, hidden))
                continue
            index = torch.from_numpy(idx).to(hidden.device)
            y.index_copy_(0, index, self._run(k, hidden.index_select(0, index)))
        return y


def main():
    from . import inputs as I
    from . import ops
    ap = argparse.ArgumentParser()
    ap.add_argument("--workloads", nargs="+", default=["prism_T64", "prism_T2048"])
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    args = ap.parse_args()
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    flush_rd = torch.ones((256 << 20) // 4, dtype=torch.float32, device="cuda")

    def timed(fn):
        for _ in range(args.warmup):
            fn()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(args.steps)]
        for i in range(args.steps):
            flush.fill_(i & 0xFF)
            flush_rd.sum()
            torch.cuda._sleep(400_000)     # ~0.2 ms: the host enqueues the step meanwhile
            ev[i][0].record()
            fn()
            ev[i][1].record()
        torch.cuda.synchronize()
        return round(float(np.median([a.elapsed_time(b) for a, b in ev])) * 1e3, 2)

    for name in args.workloads:
        shape = I.WORKLOADS[name]
        inp = I.make_inputs(shape, seed=0, quant_device="cuda")
        layer = ops.MoELayerFP8(inp)
        h = inp.hidden.cuda()
        kpt_host = inp.k_per_token
        kpt = kpt_host.cuda()
        row = dict(workload=name, T=shape.T, tiers=[(k, len(i)) for k, i in k_tiers(kpt_host)])
        row["elastic_us"] = timed(lambda: layer(h, kpt))
        tiered = KTieredLayer(layer)
        row["tiered_us"] = timed(lambda: tiered(h, kpt_host))
        if shape.T <= 512:
            from .graphs import MoEGraphExecutor
            ex = MoEGraphExecutor(layer, buckets=(shape.T,))
            row["elastic_graph_us"] = timed(lambda: ex(h, kpt))
            tg = KTieredLayer(layer, graphs=True, buckets=tuple(2 ** i for i in range(10)))
            row["tiered_graph_us"] = timed(lambda: tg(h, kpt_host))
        y_e = layer(h, kpt).float()
        y_t = tiered(h, kpt_host).float()
        row["max_abs_diff_tiered_vs_elastic"] = float((y_e - y_t).abs().max())
        row["status"] = ops.device_status(layer.ws)
        print(json.dumps(row), flush=True)
        del layer, inp
        torch.cuda.empty_cache()


if __name__ == "__main__":
    main()
