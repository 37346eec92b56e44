"""Expert parallelism: the layer's E routed experts split over n_ranks GPUs, one process per GPU.

Rank r holds experts [r * E/n, (r+1) * E/n) (FP8 weights and scales), the router and the shared
expert. A forward pass on rank r's own batch of tokens:

1. ``moe_route_topk`` routes the batch with the full router (every rank scores all E experts);
2. ``moe_ep_dispatch`` writes one send row per (token, rank holding one of its experts): the
   token's bf16 hidden row, the local ids and routing weights of its experts on that rank; the
   rows for one rank form one contiguous segment;
3. an all-to-all exchanges the segments (hidden rows, ids, weights); every rank now holds a batch
   of tokens from all sources, each with up to min(k_max, E/n) local experts;
4. the receiving rank runs ``moe_permute``, ``moe_grouped_ffn_fp8`` and ``moe_combine`` (fp32
   output) over that batch: the per-token partial sums of its experts' weighted outputs;
5. a second all-to-all returns the partial sums in the order they arrived;
6. ``moe_combine`` with one slot per rank (weight 1) adds the partial sums and the shared expert's
   output (computed in step 2's shadow) and rounds once to bf16.

The layer's pages describe this placement: "Routage MoE entre GPU" (viite.ai), the paragraphs on
sending a token's activations over NVLink/NVSwitch to the GPUs holding its experts and returning
the results; "Semantic Parallelism" (gist.science), section 1, the all-to-all of expert
parallelism. Every step's arithmetic runs in the CUDA library; the exchange is
``torch.distributed.all_to_all_single`` (NCCL between GPUs; gloo moves the same bytes between
CPU processes), or, for n virtual ranks sharing one GPU in one process, ``loopback_forward``'s
device copies of the same segments.

The receiving rank sees at most min(k_max, E/n) experts per row, so a token with several experts
on one rank sends its row there once. The result equals the one-GPU layer up to the order of the
fp32 additions in the final sum (experts grouped by rank, then ranks in order).
"""
from __future__ import annotations

import math
from dataclasses import dataclass
from typing import List, Optional, Sequence

import torch

from . import ops


@dataclass
class Dispatched:
    """One rank's dispatch: send rows (rank-major segments), their per-rank counts on the host,
    the final-combine map and the shared expert's output."""
    T: int
    send_hidden: torch.Tensor
    send_ids: torch.Tensor
    send_w: torch.Tensor
    counts: List[int]
    slot_of: torch.Tensor
    slot_w: torch.Tensor
    shared_out: Optional[torch.Tensor]

    def segment(self, dst: int) -> slice:
        start = sum(self.counts[:dst])
        return slice(start, start + self.counts[dst])


class ExpertParallelRank:
    """One rank of an expert-parallel layer.

    router_w [E, d] fp32 and router_bias [E] (or None) are the whole router; w13 [E/n, 2F, d],
    w13_scale [E/n, 2F], w2 [E/n, d, F], w2_scale [E/n, d] are this rank's experts (e4m3 codes as
    uint8 or float8_e4m3fn); shared = (w13 [2F, d], scale [2F], w2 [d, F], scale [d]) or None.
    """

    def __init__(self, rank: int, n_ranks: int, router_w: torch.Tensor,
                 router_bias: Optional[torch.Tensor], k: int, k_max: int, w13: torch.Tensor,
                 w13_scale: torch.Tensor, w2: torch.Tensor, w2_scale: torch.Tensor,
                 shared: Optional[Sequence[torch.Tensor]] = None):
        E, d = router_w.shape
        if not 1 <= n_ranks <= 32 or E % n_ranks:
            raise ValueError(f"{n_ranks} ranks do not divide {E} experts")
        if w13.shape[0] != E // n_ranks or w2.shape[0] != E // n_ranks:
            raise ValueError("w13 / w2 must hold this rank's E / n_ranks experts")
        self.rank, self.n_ranks = rank, n_ranks
        self.E, self.d, self.k, self.k_max = E, d, k, k_max
        self.E_local = E // n_ranks
        self.F = w13.shape[1] // 2
        self.kl = ops.ep_local_k(E, k_max, n_ranks)
        self.router_w, self.router_bias = router_w, router_bias
        self.w13, self.w13_scale, self.w2, self.w2_scale = w13, w13_scale, w2, w2_scale
        self.shared = None
        if shared is not None:
            a, b, c, e = shared
            self.shared = (a.unsqueeze(0), b.unsqueeze(0), c.unsqueeze(0), e.unsqueeze(0))
        self._ident = {}

    # ------------------------------------------------------------------ steps 1-2 (source side)
    def dispatch(self, hidden: torch.Tensor, k_per_token: Optional[torch.Tensor] = None) -> Dispatched:
        T = hidden.shape[0]
        dev = hidden.device
        if T == 0:
            z = torch.empty(0, self.d, dtype=torch.bfloat16, device=dev)
            return Dispatched(0, z, torch.empty(0, self.kl, dtype=torch.int32, device=dev),
                              torch.empty(0, self.kl, dtype=torch.float32, device=dev),
                              [0] * self.n_ranks, None, None, None)
        ids, w = ops.moe_route_topk(hidden, self.router_w, self.router_bias, self.k, k_per_token,
                                    self.k_max, F=self.F)
        out = ops.moe_ep_dispatch(hidden, ids, w, self.k, k_per_token, self.E, self.n_ranks)
        shared_out = self._shared_expert(hidden) if self.shared is not None else None
        counts = [int(c) for c in out["send_counts"].tolist()]   # the host needs the split sizes
        return Dispatched(T, out["send_hidden"], out["send_ids"], out["send_w"], counts,
                          out["slot_of"], out["slot_w"], shared_out)

    def _shared_expert(self, hidden: torch.Tensor) -> torch.Tensor:
        T = hidden.shape[0]
        key = (T, hidden.device)
        if key not in self._ident:
            self._ident[key] = (torch.tensor([0, T], dtype=torch.int32, device=hidden.device),
                                torch.arange(T, dtype=torch.int32, device=hidden.device))
        offsets, perm = self._ident[key]
        a, b, c, e = self.shared
        return ops.moe_grouped_ffn_fp8(hidden, a, b, c, e, offsets, perm, 1)

    # ------------------------------------------------------------------ step 4 (expert side)
    def experts(self, recv_hidden: torch.Tensor, recv_ids: torch.Tensor,
                recv_w: torch.Tensor) -> torch.Tensor:
        """Partial outputs fp32 [n, d] of this rank's experts for n received rows."""
        n = recv_hidden.shape[0]
        if n == 0:
            return torch.empty(0, self.d, dtype=torch.float32, device=recv_hidden.device)
        offsets, perm, inv = ops.moe_permute(recv_ids, self.kl, None, self.E_local, d=self.d,
                                             F=self.F)
        out = ops.moe_grouped_ffn_fp8(recv_hidden, self.w13, self.w13_scale, self.w2,
                                      self.w2_scale, offsets, perm, self.kl)
        _, partial = ops.moe_combine(out, recv_w, inv, want_f32=True)
        return partial

    # ------------------------------------------------------------------ step 6 (source side)
    def combine(self, disp: Dispatched, returned: torch.Tensor) -> torch.Tensor:
        """y bf16 [T, d] from the partial sums returned in send-row order."""
        if disp.T == 0:
            return torch.empty(0, self.d, dtype=torch.bfloat16, device=returned.device)
        return ops.moe_combine(returned, disp.slot_w[:disp.T], disp.slot_of[:disp.T],
                               shared_out=disp.shared_out)

    # ------------------------------------------------------------------ one process per GPU
    def forward(self, hidden: torch.Tensor, exchange: "TorchDistExchange",
                k_per_token: Optional[torch.Tensor] = None) -> torch.Tensor:
        disp = self.dispatch(hidden, k_per_token)
        recv_counts = exchange.counts(disp.counts)
        n = sum(disp.counts)
        recv_hidden = exchange.rows(disp.send_hidden[:n], disp.counts, recv_counts)
        recv_ids = exchange.rows(disp.send_ids[:n], disp.counts, recv_counts)
        recv_w = exchange.rows(disp.send_w[:n], disp.counts, recv_counts)
        partial = self.experts(recv_hidden, recv_ids, recv_w)
        returned = exchange.rows(partial, recv_counts, disp.counts)
        return self.combine(disp, returned)


class TorchDistExchange:
    """The all-to-all of variable-size row segments over a torch.distributed process group:
    NCCL between GPUs (tensors on the current CUDA device), gloo between CPU processes. Rows of
    any dtype travel as bytes."""

    def __init__(self, group=None):
        import torch.distributed as dist
        self.dist = dist
        self.group = group
        self.n_ranks = dist.get_world_size(group)
        backend = dist.get_backend(group)
        self.device = (torch.device("cuda", torch.cuda.current_device()) if backend == "nccl"
                       else torch.device("cpu"))

    def counts(self, send_counts: Sequence[int]) -> List[int]:
        """Rows each source will send to this rank, given the rows this rank sends to each."""
        if len(send_counts) != self.n_ranks:
            raise ValueError("one count per rank")
        s = torch.tensor(list(send_counts), dtype=torch.int64, device=self.device)
        r = torch.empty_like(s)
        self.dist.all_to_all_single(r, s, group=self.group)
        return [int(v) for v in r.tolist()]

    def rows(self, x: torch.Tensor, send_counts: Sequence[int],
             recv_counts: Sequence[int]) -> torch.Tensor:
        """Segment i of x (send_counts[i] rows) goes to rank i; returns the rows received, in
        source-rank order."""
        if x.shape[0] != sum(send_counts):
            raise ValueError("x must hold exactly the rows being sent")
        tail = tuple(x.shape[1:])
        row_bytes = x.element_size() * math.prod(tail)
        xb = x.contiguous().view(torch.uint8).reshape(x.shape[0], row_bytes)
        m = sum(recv_counts)
        out = torch.empty(m, row_bytes, dtype=torch.uint8, device=x.device)
        self.dist.all_to_all_single(out, xb, output_split_sizes=list(recv_counts),
                                    input_split_sizes=list(send_counts), group=self.group)
        return out.view(x.dtype).reshape(m, *tail)


def loopback_forward(ranks: Sequence[ExpertParallelRank], hiddens: Sequence[torch.Tensor],
                     k_per_tokens: Optional[Sequence[Optional[torch.Tensor]]] = None
                     ) -> List[torch.Tensor]:
    """All n ranks of an expert-parallel layer in one process (on one GPU, or several): the same
    dispatch, expert and combine steps, with the two all-to-alls done as device copies of the
    same segments. No kernel waits for another rank."""
    n = len(ranks)
    kpts = list(k_per_tokens) if k_per_tokens is not None else [None] * n
    disps = [r.dispatch(h, kp) for r, h, kp in zip(ranks, hiddens, kpts)]
    partials = []
    for dst in range(n):
        seg = [disps[src].segment(dst) for src in range(n)]
        rh = torch.cat([disps[s].send_hidden[seg[s]] for s in range(n)])
        ri = torch.cat([disps[s].send_ids[seg[s]] for s in range(n)])
        rw = torch.cat([disps[s].send_w[seg[s]] for s in range(n)])
        partials.append(ranks[dst].experts(rh.contiguous(), ri.contiguous(), rw.contiguous()))
    ys = []
    for src in range(n):
        back = []
        for dst in range(n):
            start = sum(disps[s].counts[dst] for s in range(src))
            back.append(partials[dst][start:start + disps[src].counts[dst]])
        ys.append(ranks[src].combine(disps[src], torch.cat(back).contiguous()))
    return ys
