"""Seeded synthetic inputs shared by the CPU oracle, the tests and the bench.

This module holds only the input recipe (shapes, distributions, seeds). It
holds none of the MoE layer's arithmetic: no quantisation, routing, grouping,
expert FFN or combine lives here.

Recipe (OLMoE-shaped layer, hidden H=2048, expert intermediate I=1024,
E=64 experts, top-8):

* activations x ~ N(0, 1), rounded to BF16 (round-to-nearest-even);
* router weights of layer l ~ N(0, 0.02), seed 100 + l;
* expert e, matrix m (0 gate, 1 up, 2 down) of layer l ~ N(0, 0.02),
  seed 10000 + (l*E + e)*3 + m;
* skewed routing: a per-expert logit offset log(Zipf(s=1.2)) where the
  expert's index is its rank;
* slot-cache decode routing: per layer and token stream, drawn so that each
  expert of the previous step is kept with probability 0.5.

Every tensor has its own seed, so a test can regenerate any single expert
without generating the rest. On the CPU the values come from torch's seeded
CPU generator; a bench that asks for device="cuda" gets the same recipe drawn
by torch's CUDA generator (other values, same distribution), which only timing
runs use.
"""
from __future__ import annotations

import numpy as np
import torch

X_SEED = 1
ROUTER_SEED = 100
EXPERT_SEED = 10000
DRAWN_ROUTING_SEED = 500
WEIGHT_STD = 0.02

GATE, UP, DOWN = 0, 1, 2


def normal_bf16(shape, std: float, seed: int, device="cpu") -> torch.Tensor:
    """N(0, std^2) samples drawn in fp32 from a seeded generator, rounded to BF16."""
    g = torch.Generator(device=device).manual_seed(int(seed))
    v = torch.randn(tuple(shape), generator=g, dtype=torch.float32, device=device)
    if std != 1.0:
        v.mul_(std)
    return v.to(torch.bfloat16)


def activations(T: int, H: int, seed: int = X_SEED, device="cpu") -> torch.Tensor:
    return normal_bf16((T, H), 1.0, seed, device)


def router_weight(layer: int, E: int, H: int, device="cpu") -> torch.Tensor:
    return normal_bf16((E, H), WEIGHT_STD, ROUTER_SEED + layer, device)


def expert_seed(layer: int, E: int, e: int, m: int) -> int:
    return EXPERT_SEED + (layer * E + e) * 3 + m


def expert_matrix(layer: int, E: int, e: int, m: int, H: int, I: int,
                  device="cpu") -> torch.Tensor:
    """One expert matrix in the nn.Linear [out][in] convention.

    gate and up are [I][H]; down is [H][I].
    """
    shape = (H, I) if m == DOWN else (I, H)
    return normal_bf16(shape, WEIGHT_STD, expert_seed(layer, E, e, m), device)


def expert_bank(layer: int, E: int, H: int, I: int, device="cpu"):
    """All experts of one layer as three stacked BF16 tensors (gate, up, down)."""
    gate = torch.stack([expert_matrix(layer, E, e, GATE, H, I, device) for e in range(E)])
    up = torch.stack([expert_matrix(layer, E, e, UP, H, I, device) for e in range(E)])
    down = torch.stack([expert_matrix(layer, E, e, DOWN, H, I, device) for e in range(E)])
    return gate, up, down


def zipf_log_bias(E: int, s: float = 1.2) -> np.ndarray:
    """bias_e = log(p_e) with p_e proportional to (e+1)^(-s): rank = index + 1."""
    r = np.arange(1, E + 1, dtype=np.float64)
    p = r ** (-s)
    p /= p.sum()
    return np.log(p).astype(np.float32)


def drawn_routing(layer: int, E: int, k: int, steps: int,
                  keep_p: float = 0.5, stream: int = 0) -> np.ndarray:
    """Expert ids [steps][k] for decode at one token per step.

    Step 0 picks k distinct experts uniformly. Each later step keeps every
    expert of the previous step independently with probability keep_p, then
    fills the remaining places uniformly (without replacement) from the experts
    the previous step did not use. Ids within a step are ascending. Decode at
    T tokens per step draws T independent streams (stream = 0 .. T-1, seed
    500 + layer + 1000 * stream; stream 0 is the one-token recipe).
    """
    rng = np.random.Generator(np.random.PCG64(DRAWN_ROUTING_SEED + layer + 1000 * stream))
    out = np.empty((steps, k), dtype=np.int32)
    prev = np.sort(rng.choice(E, size=k, replace=False))
    out[0] = prev
    for s in range(1, steps):
        kept = prev[rng.random(k) < keep_p]
        others = np.setdiff1d(np.arange(E), prev)
        new = rng.choice(others, size=k - kept.size, replace=False)
        prev = np.sort(np.concatenate([kept, new]))
        out[s] = prev
    return out


__all__ = [
    "normal_bf16", "activations", "router_weight", "expert_matrix", "expert_bank",
    "expert_seed", "zipf_log_bias", "drawn_routing", "GATE", "UP", "DOWN",
    "WEIGHT_STD",
]
