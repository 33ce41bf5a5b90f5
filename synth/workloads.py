"""The five benchmark workloads: LLaMA-shaped QLoRA linears.

Shapes are (n_out, k_in) of each linear's weight, stored row-major like a
PyTorch ``Linear.weight``.  M is the number of tokens, r the LoRA rank and
alpha the LoRA alpha (scale s = alpha / r).
"""

from __future__ import annotations

from dataclasses import dataclass, field


@dataclass(frozen=True)
class Linear:
    name: str
    n_out: int
    k_in: int


def llama_layer(hidden: int, mlp: int) -> list[Linear]:
    return [
        Linear("q", hidden, hidden),
        Linear("k", hidden, hidden),
        Linear("v", hidden, hidden),
        Linear("o", hidden, hidden),
        Linear("gate", mlp, hidden),
        Linear("up", mlp, hidden),
        Linear("down", hidden, mlp),
    ]


@dataclass(frozen=True)
class Workload:
    name: str
    linears: list[Linear]
    M: int
    r: int
    alpha: float
    layers: int = 1
    seed: int = 1234
    notes: str = ""
    extra: dict = field(default_factory=dict)

    @property
    def s(self) -> float:
        return self.alpha / self.r


SINGLE_1024 = Workload(
    "single-linear-1024x1024-M128-r8", [Linear("linear", 1024, 1024)], M=128, r=8, alpha=16.0, seed=1235,
    notes="one 1024->1024 linear, 128 tokens, r=8 alpha=16 (s=2); W fp32 N(0,0.02^2)")

LLAMA7B_LAYER = Workload(
    "llama7b-layer-7-linears-M8192-r64", llama_layer(4096, 11008), M=8192, r=64, alpha=16.0, seed=1236,
    notes="LLaMA-7B layer linears, 16x512 tokens, r=64 alpha=16 (s=0.25)")

QUANTIZER_7B = Workload(
    "quantizer-llama7b-shapes-plus-vocab", [
        Linear("q", 4096, 4096), Linear("k", 4096, 4096), Linear("v", 4096, 4096), Linear("o", 4096, 4096),
        Linear("gate", 11008, 4096), Linear("up", 11008, 4096), Linear("down", 4096, 11008),
        Linear("vocab", 32000, 4096)], M=0, r=0, alpha=0.0, seed=1237,
    notes="bf16 N(0,0.02^2) with 0.1% outliers at +/-10 sigma; quantize then dequantize")

LLAMA65B_LAYER = Workload(
    "llama65b-layer-7-linears", llama_layer(8192, 22016), M=8192, r=64, alpha=16.0, seed=1238,
    notes="LLaMA-65B layer linears; forward at 16 tokens and fwd+bwd at 4x2048 tokens",
    extra={"M_decode": 16})

LLAMA33B_STACK = Workload(
    "llama33b-8-layer-stack-M8192-r64", llama_layer(6656, 17920), M=8192, r=64, alpha=16.0, layers=8, seed=1239,
    notes="LLaMA-33B layer linears x 8 layers, 4x2048 tokens, forward then backward")

ALL = [SINGLE_1024, LLAMA7B_LAYER, QUANTIZER_7B, LLAMA65B_LAYER, LLAMA33B_STACK]

