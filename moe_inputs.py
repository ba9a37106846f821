"""Seeded synthetic inputs for the gpt-oss MoE feed-forward block.

This module is shared by the CUDA path's tests/bench and by the CPU oracle's
tests. It only draws random numbers and packs them into the storage formats
the block consumes (bf16 bit patterns, packed E2M1 nibbles, E8M0 bytes); it
holds none of the block's arithmetic.

Workloads follow the write-ups of the gpt-oss open-weight models:
  * d_model = d_ff = 2880, 32 experts (20b) or 128 experts (120b), top-4
    ("gpt-oss 架构分层" section 2.2/2.4 of the pnsm.cn overview; the config.json
    read-out ``num_local_experts: 128, experts_per_token: 4`` on youleyou.com).
  * MoE weights in MXFP4 (4-bit E2M1 codes, one E8M0 scale per 32 elements).

Value distributions (every ``N(0, v)`` is read as mean 0, VARIANCE v):
  x ~ N(0, 1) -> bf16; router W ~ N(0, 1/d) -> bf16; router bias ~ N(0, 0.1) fp32;
  E2M1 codes uniform over the 16 codes; E8M0 exponents uniform in {120,121,122};
  expert biases ~ N(0, 0.02) -> bf16; RMSNorm scale = 1 + N(0, 0.1) -> bf16.

Draw order from one ``numpy.random.Generator(PCG64(seed))`` per layer:
  x, router_w, router_b, w13_codes, w13_scales, b13, w2_codes, w2_scales, b2,
  norm_scale.  (For a stack, x is drawn once from the stack seed and layer l
  uses ``SeedSequence(seed).spawn(layers)[l]`` for its weights.)
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, List, Optional

import numpy as np

__all__ = [
    "MoEConfig", "CONFIGS", "f32_to_bf16_bits", "bf16_bits_to_f32",
    "make_tokens", "make_layer", "make_stack", "zipf_bias",
]


@dataclasses.dataclass(frozen=True)
class MoEConfig:
    name: str
    T: int                 # tokens
    d: int                 # d_model
    F: int                 # d_ff
    E: int                 # experts
    k: int = 4             # experts per token
    eps: float = 1e-5      # RMSNorm epsilon (the write-ups give none)
    layers: int = 1
    bias: str = "normal"   # "normal": N(0, 0.1); "zipf": 2*log(Zipf(1.1) popularity)
    scale_lo: int = 120    # E8M0 exponent range (inclusive)
    scale_hi: int = 122
    seed: int = 0

    @property
    def pairs(self) -> int:
        return self.T * self.k


CONFIGS: Dict[str, MoEConfig] = {
    "tiny": MoEConfig("tiny", T=16, d=128, F=128, E=8),
    "decode20b": MoEConfig("decode20b", T=32, d=2880, F=2880, E=32),
    "prefill20b": MoEConfig("prefill20b", T=8192, d=2880, F=2880, E=32),
    "decode120b": MoEConfig("decode120b", T=64, d=2880, F=2880, E=128),
    "stack20b": MoEConfig("stack20b", T=2048, d=2880, F=2880, E=32, layers=24, bias="zipf"),
}


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16 (round to nearest even); returns uint16 bit patterns."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    rnd = ((u >> 16) & 1) + 0x7FFF
    return ((u + rnd) >> 16).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to float32."""
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def zipf_bias(rng: np.random.Generator, E: int, s: float = 1.1, coef: float = 2.0) -> np.ndarray:
    """Router bias ``coef * log p_e`` for a Zipf(s) popularity p over the experts.

    Rank r (1-based) has popularity r^-s / H; which expert gets which rank is a
    random permutation drawn from ``rng``.
    """
    ranks = np.arange(1, E + 1, dtype=np.float64)
    p = ranks ** (-s)
    p /= p.sum()
    perm = rng.permutation(E)
    bias = np.empty(E, dtype=np.float64)
    bias[perm] = coef * np.log(p)
    return bias.astype(np.float32)


def make_tokens(rng: np.random.Generator, T: int, d: int) -> np.ndarray:
    """x ~ N(0, 1), stored as bf16 bits [T, d]."""
    return f32_to_bf16_bits(rng.standard_normal((T, d), dtype=np.float32))


def _normal_bf16(rng, shape, var):
    return f32_to_bf16_bits(rng.standard_normal(shape, dtype=np.float32) * np.float32(math.sqrt(var)))


def make_layer(cfg: MoEConfig, rng: np.random.Generator, with_x: bool = True) -> Dict[str, np.ndarray]:
    """One layer's inputs in the boundary layout.

    Layouts (row-major):
      x          uint16 (bf16) [T, d]
      router_w   uint16 (bf16) [E, d]
      router_b   float32       [E]
      w13_codes  uint8  [E, 2F, d/2]   rows [0,F) gate, [F,2F) linear; element 2m
                                        of a row is the low nibble of byte m
      w13_scales uint8  [E, 2F, d/32]  E8M0 exponent of each 32-element block
      b13        uint16 (bf16) [E, 2F]
      w2_codes   uint8  [E, d, F/2]
      w2_scales  uint8  [E, d, F/32]
      b2         uint16 (bf16) [E, d]
      norm_scale uint16 (bf16) [d]
    """
    T, d, F, E = cfg.T, cfg.d, cfg.F, cfg.E
    out: Dict[str, np.ndarray] = {}
    if with_x:
        out["x"] = make_tokens(rng, T, d)
    out["router_w"] = _normal_bf16(rng, (E, d), 1.0 / d)
    if cfg.bias == "zipf":
        out["router_b"] = zipf_bias(rng, E)
    else:
        out["router_b"] = (rng.standard_normal(E, dtype=np.float32) * np.float32(math.sqrt(0.1))).astype(np.float32)
    out["w13_codes"] = rng.integers(0, 256, size=(E, 2 * F, d // 2), dtype=np.uint8)
    out["w13_scales"] = rng.integers(cfg.scale_lo, cfg.scale_hi + 1, size=(E, 2 * F, d // 32), dtype=np.uint8)
    out["b13"] = _normal_bf16(rng, (E, 2 * F), 0.02)
    out["w2_codes"] = rng.integers(0, 256, size=(E, d, F // 2), dtype=np.uint8)
    out["w2_scales"] = rng.integers(cfg.scale_lo, cfg.scale_hi + 1, size=(E, d, F // 32), dtype=np.uint8)
    out["b2"] = _normal_bf16(rng, (E, d), 0.02)
    out["norm_scale"] = f32_to_bf16_bits(
        np.float32(1.0) + rng.standard_normal(d, dtype=np.float32) * np.float32(math.sqrt(0.1)))
    return out


def make_config_inputs(cfg: MoEConfig, layer: int = 0) -> Dict[str, np.ndarray]:
    """Inputs of a single-layer config (or of layer ``layer`` of a stack, without x)."""
    if cfg.layers == 1:
        return make_layer(cfg, np.random.Generator(np.random.PCG64(cfg.seed)))
    seeds = np.random.SeedSequence(cfg.seed).spawn(cfg.layers)
    return make_layer(cfg, np.random.Generator(np.random.PCG64(seeds[layer])), with_x=False)


def make_stack(cfg: MoEConfig, layers: Optional[List[int]] = None) -> Dict[str, object]:
    """A stack's token batch and the weights of the requested layers."""
    x = make_tokens(np.random.Generator(np.random.PCG64(cfg.seed)), cfg.T, cfg.d)
    idx = list(range(cfg.layers)) if layers is None else list(layers)
    return {"x": x, "layers": {l: make_config_inputs(cfg, l) for l in idx}}


def custom_layer(T: int, d: int, F: int, E: int, k: int = 4, seed: int = 0, bias: str = "normal",
                 scale_lo: int = 120, scale_hi: int = 122, eps: float = 1e-5) -> Dict[str, np.ndarray]:
    """Inputs for an arbitrary (test) shape with the same distributions."""
    cfg = MoEConfig("custom", T=T, d=d, F=F, E=E, k=k, bias=bias, scale_lo=scale_lo,
                    scale_hi=scale_hi, seed=seed, eps=eps)
    return make_layer(cfg, np.random.Generator(np.random.PCG64(seed)))
