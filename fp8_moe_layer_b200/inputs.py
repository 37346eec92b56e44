"""Seeded synthetic inputs for the FP8 MoE layer, shared by the CUDA path and the oracle.

This module holds no step of the layer's arithmetic: it only draws random tensors and stores
the expert weights in the FP8 e4m3 format the layer consumes (per-output-channel fp32 scale =
amax / 448, the weight format of the W8A8 path described in "La nouvelle bibliotheque megakernel
d'Aleph Alpha ...", section "Comment fonctionne le megakernel" / the W8A8 FP8 paragraph before
it). The FP8 cast of the weights is torch's own ``float8_e4m3fn`` conversion, so the layer's
kernels and the oracle both receive identical bytes.

Recipe (each tensor has its own generator, seeded from ``(seed, tensor name, expert index)`` so
that any one expert can be regenerated alone):

* ``hidden``   bf16 [T, d] ~ N(0, 1) (fp32 draw, RNE cast to bf16)
* ``router_w`` fp32 [E, d] ~ N(0, 0.02)
* ``router_bias`` fp32 [E] or None. Zipf(s) skew: a random permutation ``pi`` of the experts,
  ``p_e ~ (pi(e) + 1) ** -s`` normalised, ``b_e = ln p_e``.  None for a uniform router.
* ``w13`` e4m3 [E, 2F, d] (rows [0, F) gate, [F, 2F) up), ``w2`` e4m3 [E, d, F]: fp32 draws
  ~ N(0, 0.02), quantised row by row with scale ``amax / 448`` (1 when the row is all zero).
* shared expert (when ``F_shared > 0``): the same recipe, one expert.
* ``k_per_token`` int32 [T] drawn uniformly from ``k_choices`` (elastic top-k), else None.
"""
from __future__ import annotations

import hashlib
from dataclasses import dataclass, field
from typing import Optional, Tuple

import torch

E4M3_MAX = 448.0
INIT_STD = 0.02


@dataclass(frozen=True)
class MoEShape:
    """One MoE-layer workload: token count and layer sizes."""

    name: str
    T: int
    d: int
    E: int
    F: int
    k: int
    k_max: int
    F_shared: int = 0
    zipf_s: Optional[float] = None
    k_choices: Optional[Tuple[int, ...]] = None

    @property
    def elastic(self) -> bool:
        return self.k_choices is not None

    def with_T(self, T: int, name: Optional[str] = None) -> "MoEShape":
        return MoEShape(name or f"{self.name.split('_T')[0]}_T{T}", T, self.d, self.E, self.F,
                        self.k, self.k_max, self.F_shared, self.zipf_s, self.k_choices)


def _family(name, d, E, F, k, Ts, F_shared=0, zipf_s=None, k_choices=None):
    k_max = max(k_choices) if k_choices else k
    return {f"{name}_T{T}": MoEShape(f"{name}_T{T}", T, d, E, F, k, k_max, F_shared, zipf_s,
                                     k_choices) for T in Ts}


#: The workloads: a tiny parity layer and four layer shapes taken from the MoE models the pages
#: name (Mixtral 8x7B, Qwen3-30B-A3B, DeepSeek-V3 with one shared expert, and a MoE-Prism style
#: split into 4 sub-experts per Qwen3 expert with a per-token k).
WORKLOADS = {}
WORKLOADS.update(_family("tiny", 128, 8, 256, 2, [16]))
WORKLOADS.update(_family("mixtral", 4096, 8, 14336, 2, [1, 32, 512]))
WORKLOADS.update(_family("qwen3", 2048, 128, 768, 8, [1, 64, 4096], zipf_s=1.1))
WORKLOADS.update(_family("deepseek", 7168, 256, 2048, 8, [128, 8192], F_shared=2048,
                         zipf_s=1.2))
WORKLOADS.update(_family("prism", 2048, 512, 192, 2, [64, 2048], k_choices=(2, 4, 8, 16, 32)))


def _generator(seed: int, *tags) -> torch.Generator:
    """A CPU generator whose seed is a hash of (seed, tags): independent, reproducible streams."""
    h = hashlib.sha256(repr((int(seed),) + tuple(tags)).encode()).digest()
    return torch.Generator(device="cpu").manual_seed(int.from_bytes(h[:8], "little") >> 1)


def quantize_weight_rows(w: torch.Tensor, device=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """Store fp32 weight rows as e4m3 bytes + a per-row fp32 scale (amax / 448, 1 if amax = 0).

    Uses torch's float8_e4m3fn cast (round to nearest even). Returns (uint8 codes, fp32 scales)
    on the CPU.
    """
    dev = torch.device(device) if device is not None else w.device
    w = w.to(dev, torch.float32)
    amax = w.abs().amax(dim=-1)
    scale = torch.where(amax > 0, amax / E4M3_MAX, torch.ones_like(amax))
    codes = (w / scale.unsqueeze(-1)).to(torch.float8_e4m3fn).view(torch.uint8)
    return codes.cpu(), scale.cpu()


def expert_weights(shape: MoEShape, seed: int, e: int, quant_device=None):
    """Regenerate routed expert ``e`` (or the shared expert for ``e == -1``) alone.

    Returns (w13 codes [2F, d], w13 scale [2F], w2 codes [d, F], w2 scale [d]).
    """
    F = shape.F_shared if e < 0 else shape.F
    tag = "shared" if e < 0 else "expert"
    g13 = _generator(seed, shape.d, F, tag, "w13", e)
    g2 = _generator(seed, shape.d, F, tag, "w2", e)
    w13 = torch.randn(2 * F, shape.d, generator=g13) * INIT_STD
    w2 = torch.randn(shape.d, F, generator=g2) * INIT_STD
    q13, s13 = quantize_weight_rows(w13, quant_device)
    q2, s2 = quantize_weight_rows(w2, quant_device)
    return q13, s13, q2, s2


@dataclass
class MoEInputs:
    """All inputs of one layer call, on the CPU (bf16 hidden; e4m3 weights as uint8 bytes)."""

    shape: MoEShape
    hidden: torch.Tensor                      # bf16 [T, d]
    router_w: torch.Tensor                    # fp32 [E, d]
    router_bias: Optional[torch.Tensor]       # fp32 [E] or None
    k_per_token: Optional[torch.Tensor]       # int32 [T] or None
    w13: torch.Tensor                         # uint8 [E, 2F, d]
    w13_scale: torch.Tensor                   # fp32 [E, 2F]
    w2: torch.Tensor                          # uint8 [E, d, F]
    w2_scale: torch.Tensor                    # fp32 [E, d]
    w13_shared: Optional[torch.Tensor] = None  # uint8 [2Fs, d]
    w13s_scale: Optional[torch.Tensor] = None  # fp32 [2Fs]
    w2_shared: Optional[torch.Tensor] = None   # uint8 [d, Fs]
    w2s_scale: Optional[torch.Tensor] = None   # fp32 [d]
    seed: int = 0
    extra: dict = field(default_factory=dict)


def make_hidden(shape: MoEShape, seed: int = 0) -> torch.Tensor:
    g = _generator(seed, "hidden", shape.T, shape.d)
    return torch.randn(shape.T, shape.d, generator=g).to(torch.bfloat16)


def make_router(shape: MoEShape, seed: int = 0):
    g = _generator(seed, "router", shape.E, shape.d)
    router_w = torch.randn(shape.E, shape.d, generator=g) * INIT_STD
    bias = None
    if shape.zipf_s is not None:
        gp = _generator(seed, "zipf", shape.E)
        rank = torch.randperm(shape.E, generator=gp).to(torch.float64)
        p = (rank + 1.0) ** (-float(shape.zipf_s))
        p = p / p.sum()
        bias = torch.log(p).to(torch.float32)
    return router_w.contiguous(), bias


def make_k_per_token(shape: MoEShape, seed: int = 0) -> Optional[torch.Tensor]:
    if not shape.elastic:
        return None
    g = _generator(seed, "k_per_token", shape.T)
    choices = torch.tensor(shape.k_choices, dtype=torch.int32)
    idx = torch.randint(0, len(choices), (shape.T,), generator=g)
    return choices[idx].contiguous()


def make_inputs(shape: MoEShape, seed: int = 0, quant_device=None) -> MoEInputs:
    """Draw every input of ``shape``. ``quant_device`` only chooses where torch casts to FP8."""
    hidden = make_hidden(shape, seed)
    router_w, bias = make_router(shape, seed)
    E, F, d = shape.E, shape.F, shape.d
    w13 = torch.empty(E, 2 * F, d, dtype=torch.uint8)
    s13 = torch.empty(E, 2 * F, dtype=torch.float32)
    w2 = torch.empty(E, d, F, dtype=torch.uint8)
    s2 = torch.empty(E, d, dtype=torch.float32)
    for e in range(E):
        w13[e], s13[e], w2[e], s2[e] = expert_weights(shape, seed, e, quant_device)
    inp = MoEInputs(shape, hidden, router_w, bias, make_k_per_token(shape, seed),
                    w13, s13, w2, s2, seed=seed)
    if shape.F_shared:
        inp.w13_shared, inp.w13s_scale, inp.w2_shared, inp.w2s_scale = expert_weights(
            shape, seed, -1, quant_device)
    return inp
