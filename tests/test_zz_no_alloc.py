"""The allocation-free small-batch forward against the regular forward.

Hosts with a fixed device-memory pool, or that may not call any allocator
while decoding, use e4b_moe_expert_forward_decode_noalloc(): it keeps its
scratch in a static device array instead of a caller workspace.  This test
calls it through the C ABI twice in a row (the second call sees the first
call's leftovers in the shared array) and compares both results with the
regular forward on the same inputs.  Both run the same deterministic decode
kernels, only with their scratch in a different place, so the results must be
bit-identical (the layer tolerance against the oracle is checked on the
regular forward's own tests).  It is collected last so a failure here cannot
hide others.
"""
import numpy as np
import pytest
import torch

from quantized_moe_expert_nf4_b200 import e4b, synthetic, workloads
from gpu_util import require_gpu

pytestmark = pytest.mark.gpu


def _regular(layer, x, logits):
    cfg = layer.cfg
    out = torch.empty((x.shape[0], cfg.H), dtype=torch.bfloat16, device="cuda")
    ws = e4b.workspace(e4b.e4b_moe_expert_forward_workspace_size(x.shape[0], layer.stack, cfg.k))
    e4b.e4b_moe_expert_forward(x, logits, cfg.k, True, layer.stack, out, ws)
    torch.cuda.synchronize()
    return out


def _noalloc(layer, x, logits):
    cfg = layer.cfg
    out = torch.full((x.shape[0], cfg.H), float("nan"), dtype=torch.bfloat16, device="cuda")
    e4b.e4b_moe_expert_forward_decode_noalloc(x, logits, cfg.k, True, layer.stack, out)
    torch.cuda.synchronize()
    assert e4b.last_path() == "forward.decode.noalloc"
    return out


# OLMoE-shaped (one span of 128 k per warp), gpt-oss-shaped (H = 2880: two
# spans per warp and a ragged last span), the LoRA layer, and a tiny layer.
@pytest.mark.parametrize("name,M", [("olmoe", 8), ("olmoe", 1), ("tiny", 3), ("gptoss", 1), ("gptoss", 8),
                                    ("qwen3_lora", 8)])
def test_noalloc_matches_regular_forward_twice(name, M):
    require_gpu()
    cfg = workloads.CONFIGS[name]
    layer = synthetic.make_device_layer(cfg)
    # two different batches, so the second call starts from the first one's scratch
    for rep in range(2):
        x, logits = synthetic.inputs(cfg, M, replica=rep)
        ref = _regular(layer, x, logits)
        got = _noalloc(layer, x, logits)
        assert torch.isfinite(ref.float()).all()
        assert torch.equal(got.view(torch.int16), ref.view(torch.int16)), f"noalloc {name} M={M} call {rep}"


def test_noalloc_rejects_shapes_beyond_its_scratch():
    require_gpu()
    cfg = workloads.small_config("big", E=32, H=128, I=8192, k=32)
    layer = synthetic.make_device_layer(cfg)
    x, logits = synthetic.inputs(cfg, 2)
    out = torch.empty((2, cfg.H), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(e4b.E4BError, match="static scratch"):
        e4b.e4b_moe_expert_forward_decode_noalloc(x, logits, cfg.k, True, layer.stack, out)
    x9, logits9 = synthetic.inputs(workloads.CONFIGS["tiny"], 9)
    tiny = synthetic.make_device_layer(workloads.CONFIGS["tiny"])
    with pytest.raises(e4b.E4BError, match="1 to 8 tokens"):
        e4b.e4b_moe_expert_forward_decode_noalloc(x9, logits9, 2, True, tiny.stack,
                                                  torch.empty((9, 256), dtype=torch.bfloat16, device="cuda"))
