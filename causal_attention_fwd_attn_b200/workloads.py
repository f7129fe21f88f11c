"""Workload table and seeded synthetic inputs.

This module holds no attention arithmetic: only the five workload shapes, their
input distributions and a seeded generator.  Both the CUDA path's tests and the
oracle's tests draw their inputs from here, so the two sides see bit-identical
bf16 values.

Input recipe: for workload index c, tensor t in (Q, K, V, dO) -> seed 1000*c + t;
fp32 ``torch.randn`` from a CPU ``torch.Generator`` with that seed, times the
workload's standard deviation, rounded to bf16 (round to nearest even).  Shapes
are contiguous ``[B, H, T, d]``.  No padding masks, no grouped heads: every
element is iid Gaussian, as the workloads state.
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    T: int
    d: int
    sigma_q: float
    sigma_k: float
    sigma_v: float
    sigma_do: float
    causal: int = 1

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    @property
    def BH(self) -> int:
        return self.B * self.H

    def flops_fwd(self) -> float:
        """Causal forward FLOPs, 2*B*H*T^2*d (the causal convention: half of dense)."""
        return 2.0 * self.BH * self.T * self.T * self.d

    def flops_bwd(self) -> float:
        """Causal backward FLOPs, 2.5x the forward."""
        return 2.5 * self.flops_fwd()

    def flops_total(self) -> float:
        return self.flops_fwd() + self.flops_bwd()

    def describe(self) -> str:
        return (f"B={self.B} H={self.H} T={self.T} d={self.d} causal={self.causal} "
                f"scale=1/sqrt({self.d})")


# The five workloads: a tiny parity case, a GPT-2-small attention layer, a ~200M
# decoder layer, a head-dim-128 layer and a long ragged sequence.
WORKLOADS = [
    Workload("tiny_b1h2t128d64", 1, 2, 128, 64, 1.0, 1.0, 1.0, 1.0),
    Workload("gpt2small_b8h12t1024d64", 8, 12, 1024, 64, 1.0, 1.0, 1.0, 1.0),
    Workload("decoder200m_b4h16t2048d64", 4, 16, 2048, 64, 1.0, 1.0, 1.0, 1.0),
    Workload("hd128_b2h16t4096d128", 2, 16, 4096, 128, 1.0, 1.0, 0.5, 0.5),
    Workload("ragged_b1h32t8000d128", 1, 32, 8000, 128, 3.0, 3.0, 1.0, 1.0),
]

TENSOR_INDEX = {"q": 0, "k": 1, "v": 2, "dO": 3}


def seed_for(workload_index: int, tensor: str) -> int:
    return 1000 * workload_index + TENSOR_INDEX[tensor]


def gaussian_bf16(shape, sigma: float, seed: int) -> torch.Tensor:
    """fp32 randn(shape) * sigma from a seeded CPU generator, rounded to bf16."""
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    x = torch.randn(*shape, generator=g, dtype=torch.float32)
    if sigma != 1.0:
        x.mul_(sigma)
    return x.to(torch.bfloat16)


def make_inputs(workload_index: int, w: Workload | None = None, seed_offset: int = 0):
    """Seeded bf16 CPU tensors q, k, v, dO for a workload (or a variant ``w`` of it)."""
    w = w or WORKLOADS[workload_index]
    shape = (w.B, w.H, w.T, w.d)
    sig = {"q": w.sigma_q, "k": w.sigma_k, "v": w.sigma_v, "dO": w.sigma_do}
    return {t: gaussian_bf16(shape, sig[t], seed_for(workload_index, t) + seed_offset)
            for t in ("q", "k", "v", "dO")}


def custom(B, H, T, d, sigma=1.0, causal=1, name=None) -> Workload:
    """A workload of any shape with one sigma for all four tensors (tests, edge cases)."""
    return Workload(name or f"b{B}h{H}t{T}d{d}", B, H, T, d, sigma, sigma, sigma, sigma,
                    causal)
