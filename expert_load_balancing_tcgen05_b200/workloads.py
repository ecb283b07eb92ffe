"""Seeded synthetic inputs for the routing workloads.

This module only draws random inputs with the stated shapes and
distributions; it holds none of the routing arithmetic, so both the CUDA
library and the CPU oracle can be fed from it.  Everything is drawn with a
``torch.Generator`` seeded per workload (seed = 1000 + workload number),
on the device the caller names.

Workloads (shapes and value distributions):

1. tiny_softmax   T=512, d=128, N=8, K=2, softmax, no groups, no bias;
                  fp32 x ~ N(0,1), fp32 W ~ N(0, 1/d).
2. v3_router      T=4096, d=7168, N=256, K=8, sigmoid, 8 groups keep 4,
                  group score = sum of top-2 biased keys, weights x2.5;
                  bf16 x ~ N(0,1), bf16 W ~ N(0,1/d), bias ~ U(-0.01, 0.01).
3. collapse       as 2 with T=16384 and a logit offset of +2.0 on five
                  "celebrity" experts {4, 12, 77, 140, 203}; 100 bias steps.
4. softmax_dispatch T=65536, d=4096, N=128, K=8, softmax, no groups, bf16;
                  FP8 copy on dispatch; expert outputs y ~ N(0,1) bf16
                  [T*K, d] for combine.
5. prefill_replicas T=131072, d=7168, N=256, K=8, grouped sigmoid as 2 with
                  Zipf(s=1.1) popularity as logit offsets -1.1*ln(e+1);
                  32 hottest experts replicated -> 288 slots.
metric            T=16384, d=7168, N=256, K=8: the shapes of 3 with bias and
                  without the celebrity offsets (the throughput workload).
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import torch

CELEBRITY_EXPERTS = (4, 12, 77, 140, 203)


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    number: int
    T: int
    d: int
    N: int
    K: int
    fn: int                 # 0 softmax, 1 sigmoid
    n_groups: int = 1
    topk_groups: int = 1
    group_topn: int = 2
    renorm: bool = True
    scale: float = 1.0
    dtype: torch.dtype = torch.bfloat16
    has_bias: bool = False
    offset_kind: str = "none"   # none | celebrity | zipf
    fp8: bool = False
    combine: bool = False
    n_replicas: int = 0
    bias_steps: int = 0

    @property
    def seed(self) -> int:
        return 1000 + self.number

    @property
    def n_slots(self) -> int:
        return self.N + self.n_replicas

    def with_T(self, T: int) -> "Workload":
        return dataclasses.replace(self, T=T)

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


WORKLOADS = {
    "tiny_softmax": Workload("tiny_softmax", 1, 512, 128, 8, 2, fn=0, dtype=torch.float32),
    "v3_router": Workload("v3_router", 2, 4096, 7168, 256, 8, fn=1, n_groups=8, topk_groups=4,
                          scale=2.5, has_bias=True),
    "collapse": Workload("collapse", 3, 16384, 7168, 256, 8, fn=1, n_groups=8, topk_groups=4,
                         scale=2.5, has_bias=True, offset_kind="celebrity", bias_steps=100),
    "softmax_dispatch": Workload("softmax_dispatch", 4, 65536, 4096, 128, 8, fn=0, fp8=True,
                                 combine=True),
    "prefill_replicas": Workload("prefill_replicas", 5, 131072, 7168, 256, 8, fn=1, n_groups=8,
                                 topk_groups=4, scale=2.5, has_bias=True, offset_kind="zipf",
                                 n_replicas=32),
    "metric": Workload("metric", 6, 16384, 7168, 256, 8, fn=1, n_groups=8, topk_groups=4,
                       scale=2.5, has_bias=True),
}


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def logit_offsets(wl: Workload) -> Optional[torch.Tensor]:
    """Per-expert logit offsets of the workload recipe (fp32, CPU)."""
    if wl.offset_kind == "none":
        return None
    off = torch.zeros(wl.N, dtype=torch.float32)
    if wl.offset_kind == "celebrity":
        for e in CELEBRITY_EXPERTS:
            if e < wl.N:
                off[e] = 2.0
    elif wl.offset_kind == "zipf":
        # popularity rank_e = e + 1, logit offset log(rank^-1.1) = -1.1 ln(rank)
        off = torch.tensor([-1.1 * math.log(e + 1) for e in range(wl.N)], dtype=torch.float32)
    else:
        raise ValueError(wl.offset_kind)
    return off


def make_inputs(wl: Workload, device="cpu", seed: Optional[int] = None, with_y: bool = False):
    """x [T,d], W [N,d] in the workload dtype, bias [N] fp32 (or None), logit
    offsets [N] fp32 (or None), and for combine workloads y [T*K, d] bf16."""
    seed = wl.seed if seed is None else seed
    g = _gen(seed, device)
    x = torch.randn(wl.T, wl.d, generator=g, device=device, dtype=torch.float32).to(wl.dtype)
    W = (torch.randn(wl.N, wl.d, generator=g, device=device, dtype=torch.float32)
         / math.sqrt(wl.d)).to(wl.dtype)
    bias = None
    if wl.has_bias:
        bias = (torch.rand(wl.N, generator=g, device=device, dtype=torch.float32) * 0.02 - 0.01)
    off = logit_offsets(wl)
    if off is not None:
        off = off.to(device)
    out = {"x": x, "W": W, "bias": bias, "off": off}
    if with_y:
        gy = _gen(seed + 7919, device)
        out["y"] = torch.randn(wl.T * wl.K, wl.d, generator=gy, device=device,
                               dtype=torch.float32).to(torch.bfloat16)
    return out


def make_scores(T: int, N: int, seed: int, device="cpu", quantum: float = 0.0) -> torch.Tensor:
    """fp32 score matrices in [0,1) for selection-only cases; quantum > 0
    rounds them down to multiples of it so that ties occur."""
    g = _gen(seed, device)
    s = torch.rand(T, N, generator=g, device=device, dtype=torch.float32)
    if quantum > 0:
        s = torch.floor(s / quantum) * quantum
    return s.contiguous()


def make_bias(N: int, seed: int, device="cpu", amplitude: float = 0.01) -> torch.Tensor:
    g = _gen(seed, device)
    return (torch.rand(N, generator=g, device=device, dtype=torch.float32) * 2 - 1) * amplitude


def make_assignments(T: int, K: int, N: int, seed: int, device="cpu", skew: float = 0.0):
    """Random [T,K] int32 expert ids, distinct within a token; skew > 0
    favours low expert ids (Zipf-like)."""
    g = _gen(seed, device)
    wts = torch.ones(N, dtype=torch.float32, device=device)
    if skew > 0:
        wts = torch.tensor([(e + 1) ** (-skew) for e in range(N)], dtype=torch.float32,
                           device=device)
    idx = torch.multinomial(wts.expand(T, N), K, replacement=False, generator=g)
    return idx.to(torch.int32).contiguous()
