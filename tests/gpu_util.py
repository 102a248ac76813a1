"""Helpers shared by the GPU parity tests (not a test module)."""
import numpy as np
import pytest
import torch

from quantized_moe_expert_nf4_b200 import e4b

# Tolerances of the layer output against the float64 oracle (relative Frobenius and max-abs bars).
REL_FRO_TOL = 1e-2
MAX_ABS_TOL = 2e-2


def require_gpu():
    if not torch.cuda.is_available():
        pytest.fail("needs a CUDA device (run with -m gpu on a B200)")
    e4b.load_library()


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().view(torch.int16).numpy().view(np.uint16)


def bf16_to_f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def rel_errors(got: np.ndarray, ref: np.ndarray):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    fro = np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-300)
    mx = np.max(np.abs(got - ref)) / max(np.max(np.abs(ref)), 1e-300)
    return float(fro), float(mx)


def assert_close_layer(got, ref, what=""):
    fro, mx = rel_errors(got, ref)
    print(f"[parity] {what}: rel_fro={fro:.3e} max_abs/max|ref|={mx:.3e}")
    assert fro <= REL_FRO_TOL, f"{what}: relative Frobenius error {fro:.3e} > {REL_FRO_TOL}"
    assert mx <= MAX_ABS_TOL, f"{what}: max-abs error {mx:.3e} > {MAX_ABS_TOL} * max|ref|"
    return fro, mx
