"""Seeded synthetic inputs for the NF4 fused-expert MoE layer.

This module only draws random numbers and lays them out.  It holds none of the
method's arithmetic (no quantisation, routing, GEMM or activation), so both the
CPU oracle's tests and the CUDA path may take their inputs from here.

Every tensor is drawn from numpy's PCG64 generator keyed by
``[seed, tag, index]`` so that one expert of one stack can be regenerated on
its own (the full-size parity tests rebuild only the experts a sampled token
touches).

Shapes follow the fused-stack layout of transformers v5 MoE layers, as the page
"Why does load_in_4bit still OOM on a Mixture-of-Experts model?" describes it in
"Why it happens": ``gate_up_proj [E, 2I, H]`` and ``down_proj [E, H, I]``.

Workload recipes (stand-ins for the real checkpoints and datasets the pages
use, which are not available here):

* weights: fp32 N(0, 0.02^2) per element;
* activations x: fp32 N(0, 1), rounded to bf16 (round to nearest even);
* router logits, "normal": fp32 N(0, 1);
* router logits, "zipf" / "dirichlet": ``log p_e + Gumbel(0, 1)`` with an expert
  popularity p (Zipf(s) over a seeded random permutation of expert ids, or a
  Dirichlet(alpha) draw), i.e. a Plackett-Luce top-k draw without replacement;
* LoRA A [E, r, H], B [E, 2I, r]: bf16 from fp32 N(0, 0.01^2).
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import numpy as np

# Tags that key the generator sub-streams.
TAG_GATE_UP = 1
TAG_DOWN = 2
TAG_X = 3
TAG_LOGITS = 4
TAG_LORA_A = 5
TAG_LORA_B = 6
TAG_POPULARITY = 7


def _rng(seed: int, tag: int, index: int = 0) -> np.random.Generator:
    return np.random.default_rng([int(seed), int(tag), int(index)])


@dataclasses.dataclass(frozen=True)
class LayerConfig:
    """One MoE layer shape plus its routing recipe."""

    name: str
    E: int
    H: int
    I: int
    k: int
    routing: str = "normal"  # "normal" | "zipf" | "dirichlet"
    zipf_s: float = 1.1
    dirichlet_alpha: float = 0.3
    lora_r: int = 0
    lora_alpha: float = 0.0
    weight_std: float = 0.02
    lora_std: float = 0.01


# The five layer shapes the measurements use.  Token counts are per call.
CONFIGS = {
    "tiny": LayerConfig("tiny", E=8, H=256, I=128, k=2),
    "olmoe": LayerConfig("olmoe", E=64, H=2048, I=1024, k=8),
    "qwen3": LayerConfig("qwen3", E=128, H=2048, I=768, k=8, routing="zipf"),
    "qwen3_lora": LayerConfig("qwen3_lora", E=128, H=2048, I=768, k=8,
                              lora_r=8, lora_alpha=16.0),
    "gptoss": LayerConfig("gptoss", E=32, H=2880, I=2880, k=4, routing="dirichlet"),
}

TOKENS = {
    "tiny": (64,),
    "olmoe": (1, 4, 8, 2048),
    "qwen3": (4096,),
    "qwen3_lora": (4096,),
    "gptoss": (1, 8192),
}


def gate_up_expert(cfg: LayerConfig, e: int, seed: int = 0) -> np.ndarray:
    """fp32 [2I, H] slice of gate_up_proj for expert e."""
    g = _rng(seed, TAG_GATE_UP, e)
    return (g.standard_normal((2 * cfg.I, cfg.H), dtype=np.float32)
            * np.float32(cfg.weight_std))


def down_expert(cfg: LayerConfig, e: int, seed: int = 0) -> np.ndarray:
    """fp32 [H, I] slice of down_proj for expert e."""
    g = _rng(seed, TAG_DOWN, e)
    return (g.standard_normal((cfg.H, cfg.I), dtype=np.float32)
            * np.float32(cfg.weight_std))


def gate_up_stack(cfg: LayerConfig, seed: int = 0) -> np.ndarray:
    return np.stack([gate_up_expert(cfg, e, seed) for e in range(cfg.E)])


def down_stack(cfg: LayerConfig, seed: int = 0) -> np.ndarray:
    return np.stack([down_expert(cfg, e, seed) for e in range(cfg.E)])


def activations_f32(cfg: LayerConfig, M: int, seed: int = 0) -> np.ndarray:
    """fp32 N(0,1) [M, H]; round with :func:`to_bf16_bits` for the bf16 input."""
    return _rng(seed, TAG_X, M).standard_normal((M, cfg.H), dtype=np.float32)


def to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bit patterns (uint16), round to nearest, ties to even.

    Input-preparation helper: rounding of generated fp32 data to the bf16 type
    the layer consumes.  NaN inputs are not produced by these recipes.
    """
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    lsb = (u >> np.uint64(16)) & np.uint64(1)
    r = (u + np.uint64(0x7FFF) + lsb) >> np.uint64(16)
    return r.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """bf16 bit patterns (uint16) -> fp32, exact."""
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def activations_bf16(cfg: LayerConfig, M: int, seed: int = 0) -> np.ndarray:
    return to_bf16_bits(activations_f32(cfg, M, seed))


def popularity(cfg: LayerConfig, seed: int = 0) -> Optional[np.ndarray]:
    """Expert popularity p (sums to 1) for skewed recipes, None for "normal"."""
    g = _rng(seed, TAG_POPULARITY, 0)
    if cfg.routing == "zipf":
        order = g.permutation(cfg.E)          # hot experts are not ids 0..7
        rank = np.empty(cfg.E, dtype=np.float64)
        rank[order] = np.arange(1, cfg.E + 1, dtype=np.float64)
        p = rank ** (-cfg.zipf_s)
        return p / p.sum()
    if cfg.routing == "dirichlet":
        p = g.dirichlet(np.full(cfg.E, cfg.dirichlet_alpha))
        return np.maximum(p, 1e-30) / np.maximum(p, 1e-30).sum()
    return None


def router_logits(cfg: LayerConfig, M: int, seed: int = 0, replica: int = 0) -> np.ndarray:
    """fp32 [M, E] router logits following the config's routing recipe."""
    g = _rng(seed, TAG_LOGITS, M * 1009 + replica)
    if cfg.routing == "normal":
        return g.standard_normal((M, cfg.E), dtype=np.float32)
    p = popularity(cfg, seed)
    gumbel = g.gumbel(size=(M, cfg.E))
    return (np.log(p)[None, :] + gumbel).astype(np.float32)


def lora_A(cfg: LayerConfig, seed: int = 0) -> np.ndarray:
    """bf16 bits [E, r, H]."""
    g = _rng(seed, TAG_LORA_A, 0)
    a = g.standard_normal((cfg.E, cfg.lora_r, cfg.H), dtype=np.float32) * np.float32(cfg.lora_std)
    return to_bf16_bits(a)


def lora_B(cfg: LayerConfig, seed: int = 0) -> np.ndarray:
    """bf16 bits [E, 2I, r]."""
    g = _rng(seed, TAG_LORA_B, 0)
    b = g.standard_normal((cfg.E, 2 * cfg.I, cfg.lora_r), dtype=np.float32) * np.float32(cfg.lora_std)
    return to_bf16_bits(b)


def lora_scale(cfg: LayerConfig) -> float:
    """Standard LoRA scale alpha / r (0 when the layer has no adapter)."""
    return 0.0 if cfg.lora_r == 0 else cfg.lora_alpha / cfg.lora_r


def small_config(name: str, E: int, H: int, I: int, k: int, **kw) -> LayerConfig:
    """A parity-test shape (several tiles plus ragged tails)."""
    return LayerConfig(name, E=E, H=H, I=I, k=k, **kw)


def expected_touched(p: Optional[np.ndarray], E: int, slots: int) -> float:
    """Rough expected number of distinct experts hit by ``slots`` draws."""
    if p is None:
        p = np.full(E, 1.0 / E)
    return float(np.sum(1.0 - (1.0 - p) ** slots))


__all__ = [n for n in dir() if not n.startswith("_") and n not in ("annotations", "math")]
