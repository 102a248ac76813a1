"""GPU quantiser vs the oracle: bit-exact packed bytes and absmax."""
import os

import numpy as np
import pytest
import torch

from oracle import nf4
from quantized_moe_expert_nf4_b200 import e4b, workloads
from gpu_util import require_gpu

pytestmark = pytest.mark.gpu
GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _gpu_quantize(W: torch.Tensor):
    E, N, K = W.shape
    packed = torch.empty((E, N * K // 2), dtype=torch.uint8, device="cuda")
    absmax = torch.empty((E, N * K // 64), dtype=torch.float32, device="cuda")
    e4b.e4b_nf4_quantize_stack(W, packed, absmax)
    torch.cuda.synchronize()
    assert e4b.last_path() == "quantize"
    return packed.cpu().numpy(), absmax.cpu().numpy()


@pytest.mark.parametrize("E,N,K", [(1, 1, 64), (3, 5, 64), (2, 7, 192), (3, 2, 96), (4, 33, 128), (2, 9, 320)])
def test_quantize_bit_exact_fp32(E, N, K):
    require_gpu()
    rng = np.random.default_rng(E * 100 + N * 10 + K)
    W = (rng.standard_normal((E, N, K)) * 0.02).astype(np.float32)
    W[0, 0, :64] = 0.0                                # an all-zero block
    W.reshape(-1)[-5] = 0.0
    gp, ga = _gpu_quantize(torch.from_numpy(W).cuda())
    op, oa = nf4.quantize_stack(W)
    assert np.array_equal(ga.view(np.uint32), oa.view(np.uint32))
    assert np.array_equal(gp, op)


def test_quantize_bit_exact_bf16_input():
    require_gpu()
    rng = np.random.default_rng(5)
    W32 = (rng.standard_normal((3, 64, 128)) * 0.05).astype(np.float32)
    bits = workloads.to_bf16_bits(W32)
    Wb = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).cuda()
    gp, ga = _gpu_quantize(Wb)
    op, oa = nf4.quantize_stack(workloads.bf16_bits_to_f32(bits))
    assert np.array_equal(ga, oa) and np.array_equal(gp, op)


def test_quantize_decision_points_and_hand_worked_block():
    require_gpu()
    rows = [l.split() for l in open(os.path.join(GOLDEN, "nf4_block_example.txt")) if l.strip() and not l.startswith("#")]
    w = np.zeros((1, 1, 64), np.float32)
    want = np.full(64, 7, np.uint8)
    for i, (wv, c) in enumerate(rows):
        w[0, 0, i] = np.float32(float(wv))
        want[i] = int(c)
    gp, ga = _gpu_quantize(torch.from_numpy(w).cuda())
    assert ga.tolist() == [[2.0]]
    assert np.array_equal(nf4.unpack_codes(gp[0]), want)
    # every decision point and its float32 neighbours, scaled by absmax 1
    cb = nf4.codebook_f64()
    vals = []
    for c in range(15):
        m = np.float32((cb[c] + cb[c + 1]) / 2)
        vals += [m, np.nextafter(m, np.float32(-2)), np.nextafter(m, np.float32(2))]
    vals = np.array(vals, np.float32)
    n = (len(vals) + 62) // 63 * 63
    blk = np.zeros((n // 63, 64), np.float32)
    blk[:, 0] = 1.0
    blk[:, 1:].reshape(-1)[:len(vals)] = vals
    Wt = blk.reshape(1, -1, 64)
    gp, ga = _gpu_quantize(torch.from_numpy(Wt).cuda())
    op, oa = nf4.quantize_stack(Wt)
    assert np.array_equal(gp, op) and np.array_equal(ga, oa)


@pytest.mark.parametrize("name", ["olmoe", "gptoss"])
def test_quantize_full_size_stack_sampled_experts(name):
    """Full-size gate_up stack on the GPU; three experts re-quantised by the oracle."""
    require_gpu()
    cfg = workloads.CONFIGS[name]
    W = torch.from_numpy(workloads.gate_up_stack(cfg)).cuda()
    gp, ga = _gpu_quantize(W)
    for e in (0, cfg.E // 2, cfg.E - 1):
        op, oa = nf4.quantize_expert(workloads.gate_up_expert(cfg, e))
        assert np.array_equal(gp[e], op) and np.array_equal(ga[e], oa)


def test_quantize_rejects_bad_arguments():
    require_gpu()
    W = torch.zeros((2, 3, 5), device="cuda")
    with pytest.raises(e4b.E4BError, match="multiple of 64"):
        e4b.e4b_nf4_quantize_stack(W, torch.empty(64, dtype=torch.uint8, device="cuda"),
                                   torch.empty(64, dtype=torch.float32, device="cuda"))
