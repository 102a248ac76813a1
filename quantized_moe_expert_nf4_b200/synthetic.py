"""Device-side set-up of a synthetic MoE layer for tests and benchmarks.

Draws the seeded inputs of :mod:`workloads`, moves them to the GPU and packs
the fused stacks with the library's own quantiser (``e4b_quantize_stack``, NF4
unless an FP4 stack is asked for).
No arithmetic of the method happens here.
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import numpy as np
import torch

from . import e4b, workloads


@dataclasses.dataclass
class DeviceLayer:
    cfg: workloads.LayerConfig
    gu_packed: torch.Tensor
    gu_absmax: torch.Tensor
    dn_packed: torch.Tensor
    dn_absmax: torch.Tensor
    lora_A: Optional[torch.Tensor]
    lora_B: Optional[torch.Tensor]
    stack: e4b.ExpertStack

    @property
    def nbytes(self) -> int:
        n = sum(t.numel() * t.element_size() for t in (self.gu_packed, self.gu_absmax, self.dn_packed, self.dn_absmax))
        for t in (self.lora_A, self.lora_B):
            if t is not None:
                n += t.numel() * t.element_size()
        return n


def _quantize_expert_by_expert(cfg, make_expert, N, K, seed, device, quant_type, chunk=8):
    E = cfg.E
    packed = torch.empty((E, N * K // 2), dtype=torch.uint8, device=device)
    absmax = torch.empty((E, N * K // 64), dtype=torch.float32, device=device)
    for e0 in range(0, E, chunk):
        e1 = min(E, e0 + chunk)
        W = torch.from_numpy(np.stack([make_expert(cfg, e, seed) for e in range(e0, e1)])).to(device)
        e4b.e4b_quantize_stack(W, packed[e0:e1], absmax[e0:e1], quant_type)
    return packed, absmax


def make_device_layer(cfg: workloads.LayerConfig, seed: int = 0, device: str = "cuda",
                      quant_type: int = e4b.E4B_QUANT_NF4) -> DeviceLayer:
    """Quantise the layer's seeded fp32 stacks on the GPU (expert chunks at a time)."""
    gp, ga = _quantize_expert_by_expert(cfg, workloads.gate_up_expert, 2 * cfg.I, cfg.H, seed, device, quant_type)
    dp, da = _quantize_expert_by_expert(cfg, workloads.down_expert, cfg.H, cfg.I, seed, device, quant_type)
    la = lb = None
    if cfg.lora_r:
        la = torch.from_numpy(workloads.lora_A(cfg, seed).view(np.int16)).view(torch.bfloat16).to(device)
        lb = torch.from_numpy(workloads.lora_B(cfg, seed).view(np.int16)).view(torch.bfloat16).to(device)
    torch.cuda.synchronize()
    stack = e4b.ExpertStack(gp, ga, dp, da, cfg.E, cfg.H, cfg.I, la, lb, cfg.lora_alpha, quant_type)
    return DeviceLayer(cfg, gp, ga, dp, da, la, lb, stack)


def bf16_tensor(bits: np.ndarray, device="cuda") -> torch.Tensor:
    """uint16 bf16 bit patterns -> bf16 tensor."""
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(device)


def inputs(cfg: workloads.LayerConfig, M: int, seed: int = 0, replica: int = 0, device: str = "cuda"):
    """(x bf16 [M, H], logits fp32 [M, E]) on the device."""
    x = bf16_tensor(workloads.activations_bf16(cfg, M, seed), device)
    logits = torch.from_numpy(workloads.router_logits(cfg, M, seed, replica)).to(device)
    return x, logits
