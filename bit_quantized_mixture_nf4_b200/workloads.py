"""Seeded synthetic workloads for the NF4 MoE expert layer.

This module only draws inputs: activations, full-precision expert weights,
router logits and output gradients, with the shapes and value distributions of
the layer families the expert-layer pages discuss (OLMoE, Qwen3-MoE, Mixtral,
gpt-oss shaped stacks).  It holds none of the layer's arithmetic: quantization,
routing, grouping and the expert math live in the CUDA library and, separately,
in the CPU oracle.  Both sides are fed from here.

Streams per workload: seed+0 activations, seed+1 weights, seed+2 router,
seed+3 output gradient.  Everything is drawn in fp32 and rounded to bf16
(round-to-nearest-even, by torch) where the layer takes bf16.
"""
from __future__ import annotations

import dataclasses
import math

import torch

NF4, FP4, MXFP4, INT8, FP8, BF16_WEIGHTS = 0, 1, 2, 3, 4, 5   # storage formats (e4b_codebook)


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    E: int
    H: int
    I: int
    k: int
    renorm: bool
    T: int
    seed: int
    codebook: int = NF4
    router: str = "linear"      # "linear": logits = x R^T ; "zipf": N(0,1) + alpha*ln(rank^-s)
    router_std: float = 0.02
    zipf_s: float = 1.1
    zipf_alpha: float = 0.70

    @property
    def P(self) -> int:
        return self.T * self.k

    def with_tokens(self, T: int) -> "Workload":
        return dataclasses.replace(self, T=T)

    def weight_bytes_per_expert(self) -> float:
        """Packed 4-bit storage of one expert: 3*H*I elements at 0.5 B + 4 B / 64."""
        return 3 * self.H * self.I * (0.5 + 4.0 / 64)


# Tiny layer: E=8, H=256, I=512, top-2 renormalised, T=64; router [E,H] ~ N(0,1/H)
# so logits are ~ N(0,1).
TINY = Workload("tiny", E=8, H=256, I=512, k=2, renorm=True, T=64, seed=101,
                router_std=1.0 / math.sqrt(256))
# OLMoE-1B-7B shaped: E=64, H=2048, I=1024, top-8, no renormalisation, T=4096.
OLMOE = Workload("olmoe", E=64, H=2048, I=1024, k=8, renorm=False, T=4096, seed=202)
# Qwen3-30B-A3B shaped: E=128, H=2048, I=768, top-8 renormalised; decode T in
# {1,2,4,8}, prefill T=8192; Zipf(s=1.1) expert popularity in the logits.
QWEN3 = Workload("qwen3", E=128, H=2048, I=768, k=8, renorm=True, T=8192, seed=303, router="zipf")
# Mixtral-8x7B shaped: E=8, H=4096, I=14336, top-2 renormalised, T=16384.
MIXTRAL = Workload("mixtral", E=8, H=4096, I=14336, k=2, renorm=True, T=16384, seed=404)
# gpt-oss-20b shaped, FP4 codebook: E=32, H=I=2880, top-4 renormalised, T in {1, 2048}.
GPTOSS = Workload("gptoss", E=32, H=2880, I=2880, k=4, renorm=True, T=2048, seed=505, codebook=FP4)

ALL = {w.name: w for w in (TINY, OLMOE, QWEN3, MIXTRAL, GPTOSS)}


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def activations(w: Workload, device="cpu") -> torch.Tensor:
    """x ~ N(0,1), [T, H], rounded to bf16."""
    g = _gen(w.seed + 0, device)
    return torch.randn(w.T, w.H, generator=g, device=device, dtype=torch.float32).to(torch.bfloat16)


def weights(w: Workload, device="cpu"):
    """Full-precision expert stacks, N(0, 0.02) fp32:
    gate_up [E, 2I, H] (gate rows first) and down [E, H, I]."""
    g = _gen(w.seed + 1, device)
    gate_up = torch.randn(w.E, 2 * w.I, w.H, generator=g, device=device, dtype=torch.float32).mul_(0.02)
    down = torch.randn(w.E, w.H, w.I, generator=g, device=device, dtype=torch.float32).mul_(0.02)
    return gate_up, down


def router_logits(w: Workload, x: torch.Tensor) -> torch.Tensor:
    """fp32 router logits [T, E] for activations x (on x's device).

    linear: a seeded router R [E, H] ~ N(0, router_std) applied to x.
    zipf:   N(0,1) noise plus alpha * ln(rank_e ** -s), with expert ranks from a
            seeded permutation, so a few experts take most selections."""
    device = x.device
    g = _gen(w.seed + 2, device)
    if w.router == "linear":
        R = torch.randn(w.E, w.H, generator=g, device=device, dtype=torch.float32).mul_(w.router_std)
        return (x.float() @ R.t()).contiguous()
    noise = torch.randn(w.T, w.E, generator=g, device=device, dtype=torch.float32)
    rank = torch.randperm(w.E, generator=g, device=device).to(torch.float32) + 1.0
    bias = w.zipf_alpha * (-w.zipf_s) * torch.log(rank)
    return (noise + bias[None, :]).contiguous()


def grad_output(w: Workload, device="cpu") -> torch.Tensor:
    """grad_out ~ N(0,1), [T, H], rounded to bf16."""
    g = _gen(w.seed + 3, device)
    return torch.randn(w.T, w.H, generator=g, device=device, dtype=torch.float32).to(torch.bfloat16)


def bf16_bits(t: torch.Tensor):
    """uint16 view (as numpy) of a bf16 tensor, for byte-level comparisons."""
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view("uint16")
