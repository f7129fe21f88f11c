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
    # "default": bf16 outputs, bf16 tensor-core operands.  "accuracy": fp32 O, dQ, dK,
    # dV, D from the fp32 O, P and dS split into hi + lo bf16 operands (the mode a
    # workload needs when its outputs reach magnitudes where bf16 rounding alone
    # exceeds the 2e-2 absolute tolerance).
    mode: str = "default"

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
    Workload("ragged_b1h32t8000d128", 1, 32, 8000, 128, 3.0, 3.0, 1.0, 1.0, mode="accuracy"),
]

# Option settings of each mode (the library's option bits are named after them).
# "accuracy_fp16" runs the bf16 inputs through the library's bf16 -> fp16 conversion
# (part of the step) and the fp16-operand kernels.
MODES = {
    "default": {"o_f32": False, "grad_f32": False, "precise": False, "fp16": False,
                "desc": "bf16 O, dQ, dK, dV; P and dS enter the tensor-core products as bf16"},
    "accuracy": {"o_f32": True, "grad_f32": True, "precise": True, "fp16": False,
                 "desc": "fp32 O, dQ, dK, dV; D from the fp32 O; P and dS enter the "
                         "tensor-core products as two bf16 terms hi + lo"},
    "accuracy_fp16": {"o_f32": True, "grad_f32": True, "precise": False, "fp16": True,
                      "desc": "bf16 Q, K, V, dO converted to fp16 in the step (exact for "
                              "magnitudes in [2^-14, 65504]); fp32 O, dQ, dK, dV; D from the "
                              "fp32 O; every tensor-core operand fp16 (P and dS with 11 "
                              "significant bits)"},
}

TENSOR_INDEX = {"q": 0, "k": 1, "v": 2, "dO": 3}


def seed_for(workload_index: int, tensor: str) -> int:
    return 1000 * workload_index + TENSOR_INDEX[tensor]


def gaussian_bf16(shape, sigma: float, seed: int, dtype=torch.bfloat16) -> torch.Tensor:
    """fp32 randn(shape) * sigma from a seeded CPU generator, rounded (to nearest even)
    to bf16, or to another floating type `dtype` (fp16 for the fp16-operand mode)."""
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    x = torch.randn(*shape, generator=g, dtype=torch.float32)
    if sigma != 1.0:
        x.mul_(sigma)
    return x.to(dtype)


def make_inputs(workload_index: int, w: Workload | None = None, seed_offset: int = 0,
                dtype=torch.bfloat16):
    """Seeded bf16 (or `dtype`) CPU tensors q, k, v, dO for a workload (or a variant
    ``w`` of it)."""
    w = w or WORKLOADS[workload_index]
    shape = (w.B, w.H, w.T, w.d)
    sig = {"q": w.sigma_q, "k": w.sigma_k, "v": w.sigma_v, "dO": w.sigma_do}
    return {t: gaussian_bf16(shape, sig[t], seed_for(workload_index, t) + seed_offset, dtype)
            for t in ("q", "k", "v", "dO")}


def custom(B, H, T, d, sigma=1.0, causal=1, name=None, mode="default") -> Workload:
    """A workload of any shape with one sigma for all four tensors (tests, edge cases)."""
    return Workload(name or f"b{B}h{H}t{T}d{d}", B, H, T, d, sigma, sigma, sigma, sigma,
                    causal, mode)


def find(name: str):
    """(index, workload) of the named workload."""
    for i, w in enumerate(WORKLOADS):
        if w.name == name:
            return i, w
    raise KeyError(f"unknown workload {name}; choose from {[w.name for w in WORKLOADS]}")


# ------------------------------------------------------------------ AdamW ----
# Parameter tensors of a GPT-2-small-shaped model (embed 768, 12 layers, 50257-token
# vocabulary, 1024 positions): 148 tensors, 124.4M parameters.  Rank-2 tensors take
# decoupled weight decay; vectors (biases, norm scales and shifts) do not.
def gpt2small_param_shapes(n_layer=12, n_embd=768, vocab=50257, n_ctx=1024):
    shapes = [(vocab, n_embd), (n_ctx, n_embd)]
    for _ in range(n_layer):
        shapes += [(n_embd,), (n_embd,), (3 * n_embd, n_embd), (3 * n_embd,),
                   (n_embd, n_embd), (n_embd,), (n_embd,), (n_embd,),
                   (4 * n_embd, n_embd), (4 * n_embd,), (n_embd, 4 * n_embd), (n_embd,)]
    shapes += [(n_embd,), (n_embd,)]
    return shapes


def make_adamw_inputs(shapes, seed: int):
    """Seeded fp32 CPU tensors for one AdamW step: per shape a parameter ~ N(0, 0.02^2),
    a gradient ~ N(0, 0.01^2), a first moment ~ N(0, 0.001^2) and a second moment
    |N(0, 1e-4)| (the state after some earlier steps).  Returns a list of dicts."""
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    out = []
    for shp in shapes:
        out.append({"param": torch.randn(*shp, generator=g) * 0.02,
                    "grad": torch.randn(*shp, generator=g) * 0.01,
                    "exp_avg": torch.randn(*shp, generator=g) * 1e-3,
                    "exp_avg_sq": (torch.randn(*shp, generator=g) * 1e-4).abs(),
                    "decay": len(shp) >= 2})
    return out
