"""Seeded synthetic inputs for the attention layer stack.

This module only draws random numbers. It holds none of the attention
arithmetic, so both the CUDA path and the float64 CPU oracle can take their
inputs from here without sharing any of the method's code.

Recipe: every tensor is drawn in float32 from a CPU ``torch.Generator`` seeded
with ``1234 + 100*config + 10*layer + tensor_id`` (q=0, k=1, v=2, ve=3,
gate=4, dO=5), as N(0, 1) (dO may use another standard deviation), and then
cast to the layer dtype. The same cast tensors go to the GPU and, widened
exactly to float64, to the oracle. The pages train on real text (ClimbMix /
FineWeb-EDU); these seeded tensors shaped like the d12/d24 layers stand in for
those activations.
"""
from __future__ import annotations

import torch

TENSOR_IDS = {"q": 0, "k": 1, "v": 2, "ve": 3, "gate": 4, "dO": 5}


def seed_for(config: int, layer: int, name: str) -> int:
    return 1234 + 100 * config + 10 * layer + TENSOR_IDS[name]


def draw(shape, seed: int, dtype: torch.dtype, std: float = 1.0) -> torch.Tensor:
    """N(0, std^2) in float32 from a seeded CPU generator, then cast to ``dtype``."""
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    x = torch.randn(*shape, generator=g, dtype=torch.float32)
    if std != 1.0:
        x = x * std
    return x.to(dtype)


def layer_inputs(B, T, H, Hk, D, has_ve, dtype, config=0, layer=0, dO_std=1.0):
    """All host tensors of one layer, layout (B, T, heads, D); gate is (B, T, Hk).

    ``ve`` and ``gate`` are None when the layer carries no value embedding.
    """
    out = {
        "q": draw((B, T, H, D), seed_for(config, layer, "q"), dtype),
        "k": draw((B, T, Hk, D), seed_for(config, layer, "k"), dtype),
        "v": draw((B, T, Hk, D), seed_for(config, layer, "v"), dtype),
        "dO": draw((B, T, H, D), seed_for(config, layer, "dO"), dtype, std=dO_std),
        "ve": None,
        "gate": None,
    }
    if has_ve:
        out["ve"] = draw((B, T, Hk, D), seed_for(config, layer, "ve"), dtype)
        out["gate"] = draw((B, T, Hk), seed_for(config, layer, "gate"), dtype)
    return out
