"""CUDA-graph execution of the layer, one graph per (token bucket, k profile).

"MoE-Prism" (gist.science), section 2B, describes a segmented graph executor: CUDA graphs cut at
the attention/MoE boundary, the MoE segments specialised per routing budget k so that dynamic k
keeps the launch savings of graphs. This is the MoE segment of that scheme for this library:
moe_forward (all of its kernels, with their programmatic-launch edges) is captured once per
(bucket of T, k profile) and replayed; the profile is the fixed k, or "elastic" for a per-token
k array (the kernels read k_t from device memory, so one graph serves every k vector of that
bucket). A batch smaller than its bucket is padded with copies of its first token, which route
to that token's experts, so padding never activates an extra expert (no extra weight bytes).
"""
from __future__ import annotations

from typing import Dict, Optional, Sequence, Tuple

import torch

from . import ops


class MoEGraphExecutor:
    """Replays captured moe_forward graphs for a device-resident layer (ops.MoELayerFP8)."""

    def __init__(self, layer: "ops.MoELayerFP8", buckets: Sequence[int] = (1, 2, 4, 8, 16, 32, 64,
                                                                          128, 256, 512),
                 k: Optional[int] = None):
        self.layer = layer
        self.k = layer.shape.k if k is None else int(k)   # the fixed-k profile's k
        self.buckets = sorted(set(int(b) for b in buckets))
        self.graphs: Dict[Tuple[int, str], dict] = {}
        self.stream = torch.cuda.Stream(device=layer.device)

    def bucket(self, T: int) -> int:
        for b in self.buckets:
            if b >= T:
                return b
        raise ValueError(f"{T} tokens exceed the largest bucket {self.buckets[-1]}")

    def _capture(self, T_b: int, elastic: bool) -> dict:
        layer, dev = self.layer, self.layer.device
        s = layer.shape
        h = torch.zeros(T_b, s.d, dtype=torch.bfloat16, device=dev)
        kpt = torch.full((T_b,), s.k_max, dtype=torch.int32, device=dev) if elastic else None
        y = torch.empty(T_b, s.d, dtype=torch.bfloat16, device=dev)
        dm = ops.dims(T_b, s.d, s.E, s.F, s.k_max, s.F_shared)
        ws = torch.empty(ops.workspace_bytes(dm), dtype=torch.uint8, device=dev)
        ops.clear_status(ws)

        def run():
            ops.moe_forward(h, layer.router_w, layer.router_bias, self.k, kpt, layer.w13,
                            layer.w13_scale, layer.w2, layer.w2_scale, s.k_max,
                            shared=layer.shared, ws=ws, y=y)

        self.stream.wait_stream(torch.cuda.current_stream(dev))
        with torch.cuda.stream(self.stream):
            run()                               # outside capture: one-time host set-up
        self.stream.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=self.stream):
            run()
        torch.cuda.current_stream(dev).wait_stream(self.stream)
        return dict(graph=g, h=h, kpt=kpt, y=y, ws=ws, T=T_b)

    def __call__(self, hidden: torch.Tensor, k_per_token: Optional[torch.Tensor] = None):
        T = hidden.shape[0]
        elastic = k_per_token is not None
        key = (self.bucket(T), "elastic" if elastic else f"k{self.k}")
        if key not in self.graphs:
            self.graphs[key] = self._capture(key[0], elastic)
        g = self.graphs[key]
        g["h"][:T].copy_(hidden)
        if T < key[0]:
            g["h"][T:].copy_(hidden[:1].expand(key[0] - T, -1))
        if elastic:
            g["kpt"][:T].copy_(k_per_token)
            if T < key[0]:
                g["kpt"][T:].fill_(1)
        g["graph"].replay()
        return g["y"][:T]

    def device_status(self) -> int:
        worst = ops.MOE_OK
        for g in self.graphs.values():
            st = ops.device_status(g["ws"])
            worst = st if st != ops.MOE_OK else worst
        return worst
