"""Seeded synthetic inputs for the fine-grained MoE layer.

This module only draws random tensors with fixed seeds and holds the workload
shapes. It contains none of the layer's arithmetic (no routing, no FFN, no
statistics), so both the fp64 oracle tests and the CUDA path can take their
inputs from it without sharing any of the method.

Workloads (shapes follow the pages' models; the pages' own data -- real chat
traffic on trained Kimi K3 / Mixtral weights -- is not available, so these
seeded tensors stand in for it):

* ``c1``  tiny fp32 layer, H=256, E=16, K=2, D=512, T=64, seed 0.
* ``c2``  Mixtral-shaped bf16 layer, H=4096, E=8, K=2, D=14336, seed 1.
* ``c3``  fine-grained decode layer, H=4096, E=128, K=8, D=1024, shared
          expert Ds=4096, Zipf(s=1.1) logit offset, seed 2.
* ``c4``  256-expert decode under heavy skew, as c3 with E=256, Zipf(s=1.3)
          offset and a dynamic bias B ~ U(-0.5, 0.5), seed 3.
* ``c5``  prefill-scale layer, as c3 with T=16384, seed 4.

Distributions: x ~ N(0, 1); every weight matrix ~ N(0, 1/fan_in) drawn in
fp32 and rounded to bf16 (round-to-nearest-even) for the bf16 workloads.
Skew: the fixed per-expert offset ``-(1/3) * s * ln(e + 1)`` is added to the
drawn bias B (expert 0 hottest). It is part of the *input* B, not of the
layer's semantics.

Seeds: every tensor has its own ``torch.Generator('cpu')`` so one expert's
weights can be drawn without drawing the others:
``base = seed * 1_000_003``; W_r <- base+1; B <- base+2; shared expert
(Ws1 then Ws2) <- base+999; expert e (W1[e] then W2[e]) <- base+1000+e;
x for T tokens on replica r <- base+500_000+T+7919*r.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch

CAPACITY_FACTOR = (5, 4)   # capacity_factor 1.25 as an exact fraction
ZIPF_BETA = 1.0 / 3.0      # scale of the Zipf logit offset (see module doc)


@dataclass(frozen=True)
class Workload:
    key: str
    name: str
    dtype: str          # "f32" or "bf16"
    H: int
    E: int
    K: int
    D: int
    Ds: int             # 0 = no shared expert
    Ts: tuple
    seed: int
    zipf_s: float = 0.0
    bias_uniform: float = 0.0   # half-width of U(-a, a) dynamic bias, 0 = none
    extra: dict = field(default_factory=dict)


WORKLOADS = {
    "c1": Workload("c1", "tiny fp32 MoE layer", "f32", 256, 16, 2, 512, 0, (64,), 0),
    "c2": Workload("c2", "Mixtral-shaped bf16 MoE layer", "bf16", 4096, 8, 2, 14336, 0,
                   (1, 8, 64, 512, 4096), 1),
    "c3": Workload("c3", "fine-grained decode MoE layer (128 experts + shared)", "bf16",
                   4096, 128, 8, 1024, 4096, (1, 16, 32, 64, 128), 2, zipf_s=1.1),
    "c4": Workload("c4", "256-expert decode MoE layer under heavy skew (+ shared)", "bf16",
                   4096, 256, 8, 1024, 4096, (16, 64, 128, 256), 3, zipf_s=1.3,
                   bias_uniform=0.5),
    "c5": Workload("c5", "prefill-scale fine-grained MoE layer (128 experts + shared)", "bf16",
                   4096, 128, 8, 1024, 4096, (16384,), 4, zipf_s=1.1),
}


def _gen(s: int) -> torch.Generator:
    return torch.Generator("cpu").manual_seed(int(s))


def _normal(shape, std: float, g: torch.Generator, dtype: torch.dtype) -> torch.Tensor:
    t = torch.randn(*shape, generator=g, dtype=torch.float32)
    if std != 1.0:
        t.mul_(std)
    return t.to(dtype) if dtype != torch.float32 else t


def torch_dtype(wl: Workload) -> torch.dtype:
    return torch.float32 if wl.dtype == "f32" else torch.bfloat16


def _base(wl: Workload) -> int:
    return wl.seed * 1_000_003


def draw_x(wl: Workload, T: int, replica: int = 0) -> torch.Tensor:
    """Token activations x [T, H] ~ N(0, 1)."""
    g = _gen(_base(wl) + 500_000 + T + 7919 * replica)
    return _normal((T, wl.H), 1.0, g, torch_dtype(wl))


def draw_gumbel(T: int, E: int, seed: int) -> torch.Tensor:
    """Standard Gumbel draws g [T, E] fp32, g = -log(-log(u)) with u uniform in
    (0, 1): the random input of noisy routing, drawn here so that the oracle
    and the GPU path see the same numbers."""
    g = _gen(seed * 7 + 3)
    u = torch.rand((T, E), generator=g, dtype=torch.float64)
    u = u.clamp(min=1e-12, max=1.0 - 1e-12)
    return (-torch.log(-torch.log(u))).to(torch.float32)


def draw_router(wl: Workload) -> torch.Tensor:
    """Gate weight W_r [E, H] ~ N(0, 1/H) (nn.Linear(H, E, bias=False) layout)."""
    return _normal((wl.E, wl.H), 1.0 / math.sqrt(wl.H), _gen(_base(wl) + 1), torch_dtype(wl))


def draw_bias(wl: Workload) -> torch.Tensor:
    """Expert bias input B [E] fp32: drawn dynamic bias plus the Zipf skew offset."""
    b = torch.zeros(wl.E, dtype=torch.float64)
    if wl.bias_uniform > 0:
        u = torch.rand(wl.E, generator=_gen(_base(wl) + 2), dtype=torch.float64)
        b += (2.0 * u - 1.0) * wl.bias_uniform
    if wl.zipf_s > 0:
        e = torch.arange(wl.E, dtype=torch.float64)
        b += -ZIPF_BETA * wl.zipf_s * torch.log(e + 1.0)
    return b.to(torch.float32)


def draw_expert(wl: Workload, e: int):
    """(W1[e] [D, H] ~ N(0, 1/H), W2[e] [H, D] ~ N(0, 1/D))."""
    g = _gen(_base(wl) + 1000 + e)
    w1 = _normal((wl.D, wl.H), 1.0 / math.sqrt(wl.H), g, torch_dtype(wl))
    w2 = _normal((wl.H, wl.D), 1.0 / math.sqrt(wl.D), g, torch_dtype(wl))
    return w1, w2


def draw_shared(wl: Workload):
    """(Ws1 [Ds, H], Ws2 [H, Ds]) or (None, None) when the workload has no shared expert."""
    if wl.Ds == 0:
        return None, None
    g = _gen(_base(wl) + 999)
    ws1 = _normal((wl.Ds, wl.H), 1.0 / math.sqrt(wl.H), g, torch_dtype(wl))
    ws2 = _normal((wl.H, wl.Ds), 1.0 / math.sqrt(wl.Ds), g, torch_dtype(wl))
    return ws1, ws2


def draw_all_experts(wl: Workload):
    """Stacked W1 [E, D, H] and W2 [E, H, D] (host memory: 2*E*D*H elements)."""
    dt = torch_dtype(wl)
    w1 = torch.empty((wl.E, wl.D, wl.H), dtype=dt)
    w2 = torch.empty((wl.E, wl.H, wl.D), dtype=dt)
    for e in range(wl.E):
        a, b = draw_expert(wl, e)
        w1[e].copy_(a)
        w2[e].copy_(b)
    return w1, w2


def draw_layer(wl: Workload):
    """All weights of one layer as host tensors (dict)."""
    w1, w2 = draw_all_experts(wl)
    ws1, ws2 = draw_shared(wl)
    return {"w_router": draw_router(wl), "bias": draw_bias(wl), "w1": w1, "w2": w2,
            "ws1": ws1, "ws2": ws2}


def with_shape(wl: Workload, **kw) -> Workload:
    """A copy of a workload with some fields replaced (used for edge cases)."""
    d = dict(wl.__dict__)
    d.update(kw)
    return Workload(**d)


def to_f64(t):
    """Exact widening of an fp32/bf16 tensor to a float64 numpy array."""
    if t is None:
        return None
    return t.to(torch.float64).numpy()


class LazyF64:
    """Indexable view that widens one expert slab to float64 on access."""

    def __init__(self, t: torch.Tensor):
        self.t = t

    def __getitem__(self, e):
        return self.t[e].to(torch.float64).numpy()

    def __len__(self):
        return self.t.shape[0]


def sample_tokens(T: int, n: int, seed: int) -> torch.Tensor:
    """A seeded sorted sample of n distinct token indices from [0, T) (all if n >= T)."""
    if n >= T:
        return torch.arange(T)
    g = _gen(seed * 31 + 7)
    return torch.sort(torch.randperm(T, generator=g)[:n]).values
