"""The layer backward on the GPU vs the float64 oracle's per-token backward.

The oracle's backward is pinned by finite differences of its forward (see
tests/test_oracle_backward.py).  Tolerance, as for the forward: relative
Frobenius <= 1e-2 and max-abs <= 2e-2 * max|ref| for every gradient; the GPU
rounds the decoded weights, h, dz and da to bf16 once each and accumulates in
fp32.
"""
import numpy as np
import pytest
import torch

from oracle import backward, moe, nf4, routing
from quantized_moe_expert_nf4_b200 import e4b, synthetic, workloads
from gpu_util import bf16_to_f64, rel_errors, require_gpu

pytestmark = pytest.mark.gpu


def _oracle_stack(cfg):
    gp, ga = nf4.quantize_stack(workloads.gate_up_stack(cfg))
    dp, da = nf4.quantize_stack(workloads.down_stack(cfg))
    la = lb = None
    if cfg.lora_r:
        la = workloads.bf16_bits_to_f32(workloads.lora_A(cfg)).astype(np.float64)
        lb = workloads.bf16_bits_to_f32(workloads.lora_B(cfg)).astype(np.float64)
    return moe.ExpertStack(gp, ga, dp, da, cfg.E, cfg.H, cfg.I, la, lb, workloads.lora_scale(cfg))


def _check(got, ref, what):
    fro, mx = rel_errors(got, ref)
    print(f"[parity] backward {what}: rel_fro={fro:.2e} max={mx:.2e}")
    assert fro <= 1e-2 and mx <= 2e-2, what


CASES = [
    ("tiny", workloads.CONFIGS["tiny"], 64, True),
    ("tiny_tc", workloads.CONFIGS["tiny"], 300, True),    # 600 routed rows: the recompute runs on tcgen05
    ("ragged", workloads.small_config("ragged", E=12, H=192, I=320, k=3), 37, True),
    ("lora", workloads.small_config("lora", E=6, H=128, I=192, k=2, lora_r=8, lora_alpha=16.0), 50, True),
    ("lora_full_softmax", workloads.small_config("lora", E=6, H=128, I=192, k=2, lora_r=8, lora_alpha=16.0), 33,
     False),
    ("zipf", workloads.small_config("zipf", E=16, H=256, I=128, k=4, routing="zipf"), 90, False),
]


@pytest.mark.parametrize("name,cfg,M,renorm", CASES, ids=[c[0] for c in CASES])
def test_backward_matches_oracle(name, cfg, M, renorm):
    require_gpu()
    layer = synthetic.make_device_layer(cfg)
    x, logits = synthetic.inputs(cfg, M)
    rng = np.random.default_rng(123)
    dout_bits = workloads.to_bf16_bits(rng.standard_normal((M, cfg.H)).astype(np.float32))
    dout = torch.from_numpy(dout_bits.view(np.int16)).view(torch.bfloat16).cuda()
    dx = torch.full((M, cfg.H), float("nan"), dtype=torch.float32, device="cuda")
    dl = torch.full((M, cfg.E), float("nan"), dtype=torch.float32, device="cuda")
    dA = dB = None
    if cfg.lora_r:
        dA = torch.full((cfg.E, cfg.lora_r, cfg.H), float("nan"), dtype=torch.float32, device="cuda")
        dB = torch.full((cfg.E, 2 * cfg.I, cfg.lora_r), float("nan"), dtype=torch.float32, device="cuda")
    ws = e4b.workspace(e4b.e4b_moe_expert_backward_workspace_size(M, layer.stack, cfg.k))
    e4b.e4b_moe_expert_backward(x, logits, cfg.k, renorm, layer.stack, dout, dx, dl, dA, dB, ws)
    torch.cuda.synchronize()
    assert e4b.last_path() == "backward.grouped"
    assert e4b.workspace_error(ws) == e4b.E4B_KERNEL_ERR_NONE

    st = _oracle_stack(cfg)
    lg = logits.cpu().numpy()
    ids = routing.topk(lg, cfg.k)
    rdx, rdl, rdA, rdB = backward.layer_backward(bf16_to_f64(x), lg.astype(np.float64), ids, st,
                                                 workloads.bf16_bits_to_f32(dout_bits).astype(np.float64), renorm)
    _check(dx.cpu().numpy().astype(np.float64), rdx, f"{name} dx")
    _check(dl.cpu().numpy().astype(np.float64), rdl, f"{name} dlogits")
    if cfg.lora_r:
        _check(dA.cpu().numpy().astype(np.float64), rdA, f"{name} dA")
        _check(dB.cpu().numpy().astype(np.float64), rdB, f"{name} dB")
    # deterministic: a second call gives identical bits
    dx2 = torch.empty_like(dx)
    dl2 = torch.empty_like(dl)
    e4b.e4b_moe_expert_backward(x, logits, cfg.k, renorm, layer.stack, dout, dx2, dl2, dA, dB, ws)
    torch.cuda.synchronize()
    assert torch.equal(dx.view(torch.int32), dx2.view(torch.int32))
    assert torch.equal(dl.view(torch.int32), dl2.view(torch.int32))


def test_backward_requires_adapter_gradients_and_handles_empty():
    require_gpu()
    cfg = workloads.small_config("lora", E=6, H=128, I=192, k=2, lora_r=8, lora_alpha=16.0)
    layer = synthetic.make_device_layer(cfg)
    x, logits = synthetic.inputs(cfg, 4)
    dout = torch.zeros((4, cfg.H), dtype=torch.bfloat16, device="cuda")
    dx = torch.empty((4, cfg.H), dtype=torch.float32, device="cuda")
    dl = torch.empty((4, cfg.E), dtype=torch.float32, device="cuda")
    ws = e4b.workspace(e4b.e4b_moe_expert_backward_workspace_size(4, layer.stack, cfg.k))
    with pytest.raises(e4b.E4BError, match="needs dA and dB"):
        e4b.e4b_moe_expert_backward(x, logits, cfg.k, True, layer.stack, dout, dx, dl, None, None, ws)
    dA = torch.full((cfg.E, 8, cfg.H), 7.0, dtype=torch.float32, device="cuda")
    dB = torch.full((cfg.E, 2 * cfg.I, 8), 7.0, dtype=torch.float32, device="cuda")
    e4b.e4b_moe_expert_backward(x[:0], logits[:0], cfg.k, True, layer.stack, dout[:0], dx[:0], dl[:0], dA, dB, None)
    torch.cuda.synchronize()
    assert e4b.last_path() == "backward.empty"
    assert float(dA.abs().max()) == 0.0 and float(dB.abs().max()) == 0.0
