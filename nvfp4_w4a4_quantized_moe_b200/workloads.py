"""Seeded synthetic inputs for the NVFP4 MoE layer (no method arithmetic here).

This module only draws random tensors.  It holds none of the layer's
arithmetic (no quantisation, routing or matmul), so the CPU oracle and the CUDA
library can both take their inputs from it without sharing any code.

Recipe (every tensor bf16 unless stated; drawn in fp32 and rounded to bf16):

* x [T, H]: N(0, 1); with ``x_outlier_p`` > 0 each entry is independently
  multiplied by 20 with that probability (0.1% outliers, decode and prefill).
* router weight [E, H]: N(0, 0.02).  correction bias [E] fp32: N(0, 0.01).
* logit offset [E] fp32: N(0, ``logit_offset_std``) when that is > 0 (prefill:
  0.5, to make expert loads uneven); absent otherwise.
* expert e: gate [I, H], up [I, H], down [H, I], N(0, 0.02); with
  ``w_outlier_p`` > 0 each entry is independently replaced, with that
  probability, by s * U(0.1, 0.5) with a random sign s (the outlier-heavy
  late layers described in the NetsPresso article's outlier analysis).
* routed_scaling_factor 2.5.

Every tensor has its own generator seeded from (seed, tensor name, expert), so
one expert's weights can be drawn without drawing the others.  Generation runs
on ``device``: the CPU for the small configurations, the GPU for full-size ones
(torch's CPU and CUDA generators give different streams for the same seed, so
each configuration names the device it is drawn on).
"""
from __future__ import annotations

import dataclasses
import zlib

import torch


@dataclasses.dataclass(frozen=True)
class LayerConfig:
    name: str
    T: int                 # tokens
    H: int                 # hidden size
    I: int                 # expert intermediate size
    E: int                 # routed experts
    k: int                 # experts per token
    rsf: float = 2.5       # routed_scaling_factor
    x_outlier_p: float = 0.0
    logit_offset_std: float = 0.0
    w_outlier_p: float = 0.0
    gen_device: str = "cpu"

    @property
    def pairs(self) -> int:
        return self.T * self.k


CONFIGS = {
    # hidden 256, intermediate 128, 8 experts, top-2, 32 tokens
    "tiny": LayerConfig("tiny", T=32, H=256, I=128, E=8, k=2),
    # 16 tokens through the 80-expert layer (memory-bound)
    "decode": LayerConfig("decode", T=16, H=6144, I=2048, E=80, k=8,
                          x_outlier_p=0.001, gen_device="cuda"),
    # 8192 tokens, skewed expert loads (compute-bound grouped GEMM)
    "prefill": LayerConfig("prefill", T=8192, H=6144, I=2048, E=80, k=8,
                           x_outlier_p=0.001, logit_offset_std=0.5, gen_device="cuda"),
    # 128 experts with 1% weight outliers, 4096 tokens
    "outlier": LayerConfig("outlier", T=4096, H=6144, I=2048, E=128, k=8,
                           w_outlier_p=0.01, gen_device="cuda"),
    # a prefill-shaped layer small enough for profiler captures (16 experts)
    "prefill16": LayerConfig("prefill16", T=2048, H=6144, I=2048, E=16, k=8,
                             x_outlier_p=0.001, logit_offset_std=0.5, gen_device="cuda"),
    # offline weight quantiser over one 80-expert layer (weights only)
    "quantiser": LayerConfig("quantiser", T=0, H=6144, I=2048, E=80, k=8,
                             gen_device="cuda"),
}


def _gen(seed: int, name: str, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed((seed * 1_000_003 + zlib.crc32(name.encode())) & 0x7FFF_FFFF_FFFF)
    return g


def _normal(shape, std, seed, name, device) -> torch.Tensor:
    g = _gen(seed, name, device)
    return torch.randn(shape, generator=g, device=device, dtype=torch.float32) * std


def hidden_states(cfg: LayerConfig, seed: int = 0, device=None) -> torch.Tensor:
    """x [T, H] bf16."""
    device = device or cfg.gen_device
    x = _normal((cfg.T, cfg.H), 1.0, seed, f"{cfg.name}/x", device)
    if cfg.x_outlier_p > 0:
        g = _gen(seed, f"{cfg.name}/x_outlier", device)
        mask = torch.rand((cfg.T, cfg.H), generator=g, device=device) < cfg.x_outlier_p
        x = torch.where(mask, x * 20.0, x)
    return x.to(torch.bfloat16)


def router_params(cfg: LayerConfig, seed: int = 0, device=None):
    """(router weight [E, H] bf16, correction bias [E] fp32, logit offset [E] fp32 or None)."""
    device = device or cfg.gen_device
    wg = _normal((cfg.E, cfg.H), 0.02, seed, f"{cfg.name}/router", device).to(torch.bfloat16)
    bias = _normal((cfg.E,), 0.01, seed, f"{cfg.name}/bias", device)
    off = None
    if cfg.logit_offset_std > 0:
        off = _normal((cfg.E,), cfg.logit_offset_std, seed, f"{cfg.name}/logit_offset", device)
    return wg, bias, off


def _weight(shape, cfg, seed, name, device) -> torch.Tensor:
    w = _normal(shape, 0.02, seed, name, device)
    if cfg.w_outlier_p > 0:
        g = _gen(seed, name + "/outlier", device)
        mask = torch.rand(shape, generator=g, device=device) < cfg.w_outlier_p
        mag = torch.rand(shape, generator=g, device=device) * 0.4 + 0.1
        sign = torch.where(torch.rand(shape, generator=g, device=device) < 0.5, -1.0, 1.0)
        w = torch.where(mask, sign * mag, w)
    return w.to(torch.bfloat16)


def expert_weights(cfg: LayerConfig, e: int, seed: int = 0, device=None):
    """(gate [I, H], up [I, H], down [H, I]) bf16 for expert e."""
    device = device or cfg.gen_device
    gate = _weight((cfg.I, cfg.H), cfg, seed, f"{cfg.name}/e{e}/gate", device)
    up = _weight((cfg.I, cfg.H), cfg, seed, f"{cfg.name}/e{e}/up", device)
    down = _weight((cfg.H, cfg.I), cfg, seed, f"{cfg.name}/e{e}/down", device)
    return gate, up, down


def stacked_expert_weights(cfg: LayerConfig, seed: int = 0, device=None):
    """(gate [E, I, H], up [E, I, H], down [E, H, I]) bf16, all experts."""
    device = device or cfg.gen_device
    gate = torch.empty((cfg.E, cfg.I, cfg.H), dtype=torch.bfloat16, device=device)
    up = torch.empty_like(gate)
    down = torch.empty((cfg.E, cfg.H, cfg.I), dtype=torch.bfloat16, device=device)
    for e in range(cfg.E):
        gate[e], up[e], down[e] = expert_weights(cfg, e, seed, device)
    return gate, up, down


def random_bytes(shape, seed: int, name: str, low: int = 0, high: int = 256,
                 device="cpu") -> torch.Tensor:
    """Uniform random uint8 in [low, high): synthetic packed codes or scale
    codes for tests that feed identical quantised operands to both sides."""
    g = _gen(seed, name, device)
    return torch.randint(low, high, shape, generator=g, device=device, dtype=torch.int32).to(torch.uint8)


def random_floats(shape, seed: int, name: str, std: float = 1.0, device="cpu") -> torch.Tensor:
    """N(0, std) fp32 (e.g. synthetic router logits for selection tests)."""
    return _normal(shape, std, seed, name, device)
