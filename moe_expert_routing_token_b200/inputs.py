"""Seeded synthetic inputs for the routing workloads.

This module only draws random numbers and shapes them; it holds none of the
routing arithmetic, so both the CUDA path and the CPU oracle can take their
inputs from it.  Every tensor is drawn on the CPU with a seeded
``torch.Generator`` (fp32 normal draws; bf16 tensors are those draws rounded
to nearest-even by ``.to(torch.bfloat16)``), so the same seed gives the same
bytes on every machine.

Workloads (shapes and distributions of the SGLang routing pages'
DeepSeek-V2/V3 and MiniMax-style routers):

=========  =====================================================================
softmax    softmax top-k: E=8, k=2, renormalise, fp32 logits N(0, 1), M=64
sigmoid    sigmoid + correction_bias, one group: E=256, k=8, renormalise,
           bf16 logits N(0, 2^2), fp32 bias N(0, 0.05^2), M in 1..16384
biased     biased grouped top-k (DeepSeek-V3 shape): E=256 in 8 groups of 32,
           topk_group=4, k=8, renormalise, routed scaling 2.5, same draws
grouped    softmax grouped top-k (DeepSeek-V2 shape): E=160 in 8 groups of 20,
           topk_group=3, k=6, no renormalise, fp32 logits N(0, 1.5^2)
fused      router projection: hidden bf16 (M, 7168) N(0, 1), router weight bf16
           (7168, 256) N(0, 0.02^2), then the ``biased`` routing
top1       small-E router projection: hidden bf16 (M, 7168) N(0, 1), router
           weight bf16 (8, 7168) N(0, 0.02^2) in the (E, K) layout, softcap 30
           (the pages give no value), then top-1
=========  =====================================================================
"""
from __future__ import annotations

import dataclasses

import torch

WORKLOADS = ("softmax", "sigmoid", "biased", "grouped", "fused", "top1")


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    E: int
    topk: int
    renormalize: bool
    num_expert_group: int
    topk_group: int
    routed_scaling_factor: float
    dtype: torch.dtype          # logits dtype (fused: hidden/weight dtype)
    logit_std: float
    bias_std: float | None      # None: no correction_bias
    K: int = 0                  # hidden size (fused, top1)
    weight_std: float = 0.0     # router weight std (fused, top1)
    softcap: float = 0.0        # logit softcapping constant (top1)


SPECS = {
    "softmax": Workload("softmax", 8, 2, True, 1, 1, 1.0, torch.float32, 1.0, None),
    "sigmoid": Workload("sigmoid", 256, 8, True, 1, 1, 1.0, torch.bfloat16, 2.0, 0.05),
    "biased": Workload("biased", 256, 8, True, 8, 4, 2.5, torch.bfloat16, 2.0, 0.05),
    "grouped": Workload("grouped", 160, 6, False, 8, 3, 1.0, torch.float32, 1.5, None),
    "fused": Workload("fused", 256, 8, True, 8, 4, 2.5, torch.bfloat16, 1.0, 0.05,
                      K=7168, weight_std=0.02),
    "top1": Workload("top1", 8, 1, False, 1, 1, 1.0, torch.bfloat16, 1.0, None,
                     K=7168, weight_std=0.02, softcap=30.0),
}

# Token counts the pages' workloads are quoted at.
SIZES = {
    "softmax": (64,),
    "sigmoid": (1, 16, 64, 256, 4096, 16384),
    "biased": (4096, 32),
    "grouped": (16384,),
    "fused": (8192, 64),
    "top1": (8192, 64),
}


def default_seed(name: str, M: int) -> int:
    return 1000 * (WORKLOADS.index(name) + 1) + int(M).bit_length()


def _normal(gen: torch.Generator, shape, std: float, dtype: torch.dtype) -> torch.Tensor:
    t = torch.randn(*shape, generator=gen, dtype=torch.float32) * std
    return t.to(dtype)


def make(name: str, M: int, seed: int | None = None) -> dict:
    """Return a dict of CPU tensors for workload ``name`` with ``M`` tokens.

    Keys: ``logits`` (M, E) [not for fused or top1], ``bias`` (E,) fp32 or
    None, ``hidden`` (M, K) and ``weight`` [fused: (K, E); top1: (E, K)], plus
    ``spec`` and ``seed``.
    """
    spec = SPECS[name]
    seed = default_seed(name, M) if seed is None else int(seed)
    gen = torch.Generator().manual_seed(seed)
    out = {"spec": spec, "seed": seed}
    if name == "fused":
        out["hidden"] = _normal(gen, (M, spec.K), spec.logit_std, spec.dtype)
        out["weight"] = _normal(gen, (spec.K, spec.E), spec.weight_std, spec.dtype)
    elif name == "top1":
        out["hidden"] = _normal(gen, (M, spec.K), spec.logit_std, spec.dtype)
        out["weight"] = _normal(gen, (spec.E, spec.K), spec.weight_std, spec.dtype)
    else:
        out["logits"] = _normal(gen, (M, spec.E), spec.logit_std, spec.dtype)
    out["bias"] = (None if spec.bias_std is None
                   else _normal(gen, (spec.E,), spec.bias_std, torch.float32))
    return out


def random_logits(M: int, E: int, std: float, dtype: torch.dtype, seed: int) -> torch.Tensor:
    """Plain N(0, std^2) logits of any shape (for sweeps and edge cases)."""
    gen = torch.Generator().manual_seed(int(seed))
    return _normal(gen, (M, E), std, dtype)


def random_bias(E: int, std: float, seed: int) -> torch.Tensor:
    gen = torch.Generator().manual_seed(int(seed))
    return _normal(gen, (E,), std, torch.float32)


def routed_ids(M: int, k: int, E: int, seed: int):
    """A routing result's shape for the permutation step: per token k distinct
    experts drawn uniformly (ids int32 (M, k)) and positive weights summing to
    one per token (fp32 (M, k)).  Balanced routers (the correction bias exists
    to balance load) spread tokens over experts about uniformly."""
    gen = torch.Generator().manual_seed(int(seed))
    ids = torch.argsort(torch.rand(M, E, generator=gen), dim=1)[:, :k].to(torch.int32).contiguous()
    w = torch.rand(M, k, generator=gen) + 0.05
    return ids, (w / w.sum(dim=1, keepdim=True)).to(torch.float32)
