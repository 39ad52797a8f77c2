"""The five workloads: per-layer shapes, windows and value-embedding switches.

Page "5만원으로 나만의 ChatGPT 훈련하는 방법" (apidog.com), section
"1. GPT 모델 (nanochat/gpt.py)", architecture list: the sliding-window pattern
is a string such as "SSSL" in which short windows alternate with full context,
and value embeddings sit on alternating layers. The d12/d24 shapes and the
window sizes are the workload definitions this library is measured on.
"""
from __future__ import annotations

from dataclasses import dataclass, field


def window_pattern(pattern: str, short: int, long: int, n_layer: int) -> list[int]:
    """Expand a pattern string such as "SSSL" to one window per layer.

    The pattern repeats over the layers; 'S' maps to ``short`` and 'L' to
    ``long``. A window is the number of keys a query sees, itself included.
    """
    pattern = pattern.upper()
    if not pattern or any(c not in "SL" for c in pattern):
        raise ValueError(f"window pattern must be a non-empty string of S/L, got {pattern!r}")
    return [short if pattern[i % len(pattern)] == "S" else long for i in range(n_layer)]


def alternating_ve(n_layer: int) -> list[bool]:
    """Value embedding on alternating layers, the last layer included."""
    return [(i % 2) == ((n_layer - 1) % 2) for i in range(n_layer)]


@dataclass
class Workload:
    config: int                 # 1..5, also the seed component
    name: str
    B: int
    T: int
    H: int
    Hk: int
    D: int
    windows: list[int]
    ve: list[bool]
    dtype: str                  # "f32" or "bf16"
    rope_base: float = 10000.0
    eps: float = 1e-6
    dO_std: float = 1.0
    notes: str = ""
    extra: dict = field(default_factory=dict)

    @property
    def n_layer(self) -> int:
        return len(self.windows)

    def pairs(self, W: int) -> int:
        """Unmasked (query, key) pairs per (batch, head): sum_i min(i+1, W)."""
        T = self.T
        if W >= T:
            return T * (T + 1) // 2
        return W * (W + 1) // 2 + (T - W) * W

    def flops(self, convention: str = "algorithmic") -> float:
        """fwd+bwd FLOPs over the unmasked region, all layers.

        algorithmic: 12*D per pair (fwd QK^T and PV: 4*D; bwd dV, dP, dK, dQ: 8*D).
        flash: 14*D per pair (the FlashAttention convention, bwd = 2.5x fwd).
        """
        per_pair = 12 if convention == "algorithmic" else 14
        return float(sum(per_pair * self.D * self.pairs(W) * self.B * self.H for W in self.windows))


WORKLOADS = {
    1: Workload(1, "microgpt fp32 attention layer", B=32, T=16, H=4, Hk=4, D=4,
                windows=[16], ve=[False], dtype="f32",
                notes="n_embd=16; full causal; no value embedding"),
    2: Workload(2, "nanochat d12 layer", B=8, T=2048, H=6, Hk=6, D=128,
                windows=[2048], ve=[True], dtype="bf16",
                notes="model_dim=768; full causal; value embedding on"),
    3: Workload(3, "d12 SSSL layer stack", B=8, T=2048, H=6, Hk=6, D=128,
                windows=window_pattern("SSSL", 1024, 2048, 4), ve=alternating_ve(4),
                dtype="bf16", notes="4 layers; ve on alternating layers (1 and 3)"),
    4: Workload(4, "nanochat d24 GQA SSSL layer stack", B=4, T=2048, H=12, Hk=4, D=128,
                windows=window_pattern("SSSL", 1024, 2048, 4), ve=[True] * 4,
                dtype="bf16", notes="model_dim=1536; group 3; per-KV-head gate"),
    5: Workload(5, "long-context GQA SSSL layer stack", B=1, T=8192, H=16, Hk=4, D=128,
                windows=window_pattern("SSSL", 2048, 8192, 4), ve=[True] * 4,
                dtype="bf16", dO_std=0.1, notes="group 4; dO ~ N(0, 0.1)"),
}
