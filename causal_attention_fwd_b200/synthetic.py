"""Seeded synthetic inputs and the named workloads.

This module is the one piece that both the CUDA path's tests/benchmark and the
CPU oracle's tests use.  It holds no attention arithmetic: it draws Q, K, V and
dO from a seeded CPU generator and rounds them to bf16, and it lists the five
workload shapes.

Recipe: ``torch.Generator().manual_seed(seed)``; draw, in this order, Q, K, V,
dO as float32 standard normals of shapes [B,S,Hq,D], [B,S,Hkv,D], [B,S,Hkv,D],
[B,S,Hq,D]; multiply by ``sigma``; round to bf16 (round-to-nearest-even).  The
same bf16 bits go to the GPU and, widened to float64, to the oracle.
"""
from __future__ import annotations

import dataclasses
import math

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    Hq: int
    Hkv: int
    S: int
    D: int
    sigma: float = 1.0
    causal: bool = True

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.D)

    @property
    def fwd_flops(self) -> float:
        """Causal forward FLOPs, counted as half of the dense 4*B*Hq*S^2*D."""
        dense = 4.0 * self.B * self.Hq * self.S * self.S * self.D
        return dense / 2 if self.causal else dense

    @property
    def bwd_flops(self) -> float:
        """Causal backward FLOPs, counted as half of the dense 10*B*Hq*S^2*D."""
        dense = 10.0 * self.B * self.Hq * self.S * self.S * self.D
        return dense / 2 if self.causal else dense

    def describe(self) -> str:
        return (f"B={self.B} S={self.S} Hq={self.Hq} Hkv={self.Hkv} D={self.D} "
                f"causal={int(self.causal)} inputs~N(0,{self.sigma:g}^2) scale=1/sqrt({self.D})")


# The five workloads: tiny smoke; GPT-2-small-class GQA; 1B-class training
# step (the headline); 8B-class GQA; long-sequence flat-memory.
WORKLOADS = {
    "tiny": Workload("tiny", 1, 1, 1, 128, 64),
    "gpt2s_gqa": Workload("gpt2s_gqa", 2, 12, 4, 1024, 64),
    "llm1b": Workload("llm1b", 4, 32, 8, 2048, 64),
    "llm8b_gqa": Workload("llm8b_gqa", 2, 32, 8, 8192, 128),
    "longseq": Workload("longseq", 1, 16, 16, 32768, 128, sigma=0.5),
}
WORKLOAD_ORDER = ["tiny", "gpt2s_gqa", "llm1b", "llm8b_gqa", "longseq"]
WORKLOAD_SEED = {name: 1000 + n + 1 for n, name in enumerate(WORKLOAD_ORDER)}


def make_inputs(B: int, Hq: int, Hkv: int, S: int, D: int, seed: int,
                sigma: float = 1.0, with_dout: bool = True):
    """Seeded bf16 CPU tensors (q, k, v, dout) in the [B, S, H, D] layout."""
    g = torch.Generator().manual_seed(int(seed))

    def draw(h):
        x = torch.randn((B, S, h, D), generator=g, dtype=torch.float32)
        if sigma != 1.0:
            x = x * sigma
        return x.to(torch.bfloat16)

    q = draw(Hq)
    k = draw(Hkv)
    v = draw(Hkv)
    dout = draw(Hq) if with_dout else None
    return q, k, v, dout


def workload_inputs(w: Workload, seed: int | None = None, with_dout: bool = True):
    return make_inputs(w.B, w.Hq, w.Hkv, w.S, w.D,
                       WORKLOAD_SEED.get(w.name, 1000) if seed is None else seed,
                       w.sigma, with_dout)
