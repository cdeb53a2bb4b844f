"""Seeded synthetic inputs for the MXFP4 quantize / MoE expert-MLP workloads.

This module is shared by the CPU oracle's tests and by the CUDA path's tests and
benchmark.  It holds no MXFP4 arithmetic: it only draws random tensors with
torch's CPU generator, so that both sides see byte-identical inputs.  Weights are
returned in fp32; whoever needs them in MXFP4 quantizes them itself.

Workload recipes (shapes follow the gpt-oss-20b / gpt-oss-120b expert MLP:
hidden H = 2880, expert intermediate I = 2880, top-4 routing):

* ``gemm_small``  – x bf16 [8, 256] ~ N(0,1); W fp32 [512, 256] ~ N(0, 0.02).
* ``quant``       – bf16 [4096, 11520] ~ N(0,1); 1% of elements x50 (outliers);
                    0.5% of the 32-element blocks along the last dim set to zero.
* ``moe_decode``  – T=64 tokens, 32 experts, top-4.
* ``moe_prefill`` – T=8192 tokens, 32 experts, top-4, +2.0 on experts 0..3 of
                    the router logits (load imbalance).
* ``moe_120b``    – T=4096 tokens, 128 experts, top-4.

The router-projection recipe draws bf16 router weights W_r [E, H] ~ N(0, 1/H)
(sub-seed of the layer's seed), so that x . W_r^T ~ N(0, 1) like the logits.

For the MoE recipes x ~ N(0,1) (bf16), router logits ~ N(0,1) (fp32) and each
expert's gate_up weight [2I, H] (rows [0, I) gate, [I, 2I) up) and down weight
[H, I] ~ N(0, 0.02) (fp32), drawn expert by expert from sub-seeds so that any
subset of experts can be regenerated without drawing the others.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import torch

__all__ = [
    "MoEConfig", "MOE_CONFIGS", "gemm_small", "quant_tensor", "moe_activations",
    "expert_weights", "seeded_bf16", "seeded_f32", "router_weights",
]


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    return g


def seeded_f32(shape, seed: int, std: float = 1.0) -> torch.Tensor:
    """fp32 normal(0, std) tensor drawn from a CPU generator seeded with ``seed``."""
    t = torch.randn(*shape, generator=_gen(seed), dtype=torch.float32)
    if std != 1.0:
        t.mul_(std)
    return t


def seeded_bf16(shape, seed: int, std: float = 1.0) -> torch.Tensor:
    """bf16 normal(0, std) tensor: fp32 draw cast with round-to-nearest-even."""
    return seeded_f32(shape, seed, std).to(torch.bfloat16)


def gemm_small(seed: int = 0, M: int = 8, K: int = 256, N: int = 512):
    """Single W4A16 GEMM case: x bf16 [M, K] ~ N(0,1), W fp32 [N, K] ~ N(0, 0.02)."""
    g = _gen(seed)
    x = torch.randn(M, K, generator=g, dtype=torch.float32).to(torch.bfloat16)
    w = torch.randn(N, K, generator=g, dtype=torch.float32).mul_(0.02)
    return x, w


def quant_tensor(seed: int = 1, rows: int = 4096, cols: int = 11520,
                 outlier_frac: float = 0.01, outlier_mul: float = 50.0,
                 zero_block_frac: float = 0.005) -> torch.Tensor:
    """Quantize workload: bf16 [rows, cols] with outliers and all-zero blocks.

    Draw order: normal values, then one uniform per element (outlier mask), then
    one uniform per 32-element block along the last dim (zero-block mask).
    """
    assert cols % 32 == 0
    g = _gen(seed)
    x = torch.randn(rows, cols, generator=g, dtype=torch.float32)
    mask = torch.rand(rows, cols, generator=g) < outlier_frac
    x[mask] *= outlier_mul
    zb = torch.rand(rows, cols // 32, generator=g) < zero_block_frac
    x.view(rows, cols // 32, 32)[zb] = 0.0
    return x.to(torch.bfloat16)


@dataclass(frozen=True)
class MoEConfig:
    name: str
    seed: int
    T: int
    E: int
    top_k: int = 4
    H: int = 2880
    I: int = 2880
    hot_experts: tuple = field(default_factory=tuple)
    hot_bias: float = 0.0
    w_std: float = 0.02

    def pairs(self) -> int:
        return self.T * self.top_k


MOE_CONFIGS = {
    "moe_decode": MoEConfig("moe_decode", seed=2, T=64, E=32),
    "moe_prefill": MoEConfig("moe_prefill", seed=3, T=8192, E=32,
                             hot_experts=(0, 1, 2, 3), hot_bias=2.0),
    "moe_120b": MoEConfig("moe_120b", seed=4, T=4096, E=128),
}


def moe_activations(cfg: MoEConfig, T: int | None = None):
    """Token activations x bf16 [T, H] and router logits fp32 [T, E].

    Draw order: x first, then logits, from one generator seeded with cfg.seed.
    The hot-expert bias (if any) is added to the logits after drawing.
    """
    T = cfg.T if T is None else T
    g = _gen(cfg.seed)
    x = torch.randn(T, cfg.H, generator=g, dtype=torch.float32).to(torch.bfloat16)
    logits = torch.randn(T, cfg.E, generator=g, dtype=torch.float32)
    if cfg.hot_experts:
        logits[:, list(cfg.hot_experts)] += cfg.hot_bias
    return x, logits


def expert_seed(cfg_seed: int, e: int, which: int) -> int:
    """Sub-seed of expert e's weight: which = 0 for gate_up, 1 for down."""
    return cfg_seed * 1_000_003 + 1 + 2 * e + which


def expert_weights(cfg: MoEConfig, e: int):
    """Expert e's fp32 weights: gate_up [2I, H] and down [H, I], ~ N(0, w_std)."""
    w13 = seeded_f32((2 * cfg.I, cfg.H), expert_seed(cfg.seed, e, 0), cfg.w_std)
    w2 = seeded_f32((cfg.H, cfg.I), expert_seed(cfg.seed, e, 1), cfg.w_std)
    return w13, w2


def router_weights(cfg: "MoEConfig") -> torch.Tensor:
    """bf16 router weights [E, H] ~ N(0, 1/H) (std 1/sqrt(H)) from a sub-seed of cfg.seed."""
    return seeded_bf16((cfg.E, cfg.H), cfg.seed * 1_000_003 + 999_983, cfg.H ** -0.5)
