"""GPU routing vs the oracle: bit-exact ids, offsets, perm, inv; weights to 2e-6."""
import numpy as np
import pytest
import torch

from oracle import routing
from quantized_moe_expert_nf4_b200 import e4b, workloads
from gpu_util import require_gpu

pytestmark = pytest.mark.gpu


def _gpu_route(logits: np.ndarray, k: int, renormalize=True):
    M, E = logits.shape
    dev = lambda n, d: torch.full((max(n, 1),), -7, dtype=d, device="cuda")
    ids, w = dev(M * k, torch.int32), torch.zeros(max(M * k, 1), device="cuda")
    offs, perm, inv = dev(E + 1, torch.int32), dev(M * k, torch.int32), dev(M * k, torch.int32)
    ws = e4b.workspace(e4b.e4b_moe_route_permute_workspace_size(M, E, k))
    e4b.e4b_moe_route_permute(torch.from_numpy(logits).cuda().reshape(M, E), k, renormalize, ids, w, offs, perm,
                              inv, ws)
    torch.cuda.synchronize()
    c = lambda t, n: t.cpu().numpy()[:n]
    return c(ids, M * k).reshape(M, k), c(w, M * k).reshape(M, k), c(offs, E + 1), c(perm, M * k), c(inv, M * k)


def _check(logits, k, renormalize=True):
    M, E = logits.shape
    gi, gw, go, gp, gv = _gpu_route(logits, k, renormalize)
    oi, ow, oo, op, ov = routing.route_permute(logits, k, renormalize)
    assert np.array_equal(gi, oi)
    assert np.array_equal(go, oo)
    assert np.array_equal(gp, op)
    assert np.array_equal(gv, ov)
    assert np.all(np.abs(gw - ow) <= 2e-6 * np.abs(ow) + 1e-12)


@pytest.mark.parametrize("M,E,k", [(1, 64, 8), (4, 64, 8), (8, 64, 8), (64, 8, 2), (1, 32, 4), (3, 128, 8),
                                   (512, 128, 8), (600, 33, 5), (1, 1, 1), (2, 1024, 32), (300, 1000, 7)])
def test_route_small_and_tiled(M, E, k):
    require_gpu()
    rng = np.random.default_rng(M * 7 + E)
    _check(rng.standard_normal((M, E)).astype(np.float32), k)


@pytest.mark.parametrize("name,M", [("olmoe", 2048), ("qwen3", 4096), ("qwen3_lora", 4096), ("gptoss", 8192),
                                    ("gptoss", 1), ("olmoe", 8)])
def test_route_config_workloads(name, M):
    require_gpu()
    cfg = workloads.CONFIGS[name]
    _check(workloads.router_logits(cfg, M), cfg.k)


def test_route_ties_and_full_softmax():
    require_gpu()
    rng = np.random.default_rng(3)
    logits = rng.integers(-2, 3, size=(5000, 16)).astype(np.float32)   # ties everywhere, tiled path
    _check(logits, 4)
    _check(logits[:100], 4)                                             # small path
    _check(rng.standard_normal((70, 24)).astype(np.float32), 3, renormalize=False)
    _check(rng.standard_normal((9000, 24)).astype(np.float32), 3, renormalize=False)
    z = np.array([[0.0, -0.0, 0.0, -0.0]], np.float32)
    _check(z, 4)


def test_route_empty_batch_and_errors():
    require_gpu()
    gi, gw, go, gp, gv = _gpu_route(np.zeros((0, 8), np.float32), 2)
    assert go.tolist() == [0] * 9
    with pytest.raises(e4b.E4BError, match="workspace"):
        M, E, k = 9000, 16, 4
        lg = torch.zeros((M, E), device="cuda")
        o = [torch.empty(M * k, dtype=torch.int32, device="cuda") for _ in range(3)]
        e4b.e4b_moe_route_permute(lg, k, True, o[0], torch.empty(M * k, device="cuda"),
                                  torch.empty(E + 1, dtype=torch.int32, device="cuda"), o[1], o[2], None)
