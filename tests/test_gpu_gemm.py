"""GPU grouped NF4 GEMM vs the float64 oracle (every epilogue and output type)."""
import numpy as np
import pytest
import torch

from oracle import moe, nf4
from quantized_moe_expert_nf4_b200 import e4b, workloads
from gpu_util import bf16_to_f64, rel_errors, require_gpu

pytestmark = pytest.mark.gpu


def _case(E, N, K, counts, a_rows, seed, lora_r=0):
    rng = np.random.default_rng(seed)
    W = (rng.standard_normal((E, N, K)) * 0.02).astype(np.float32)
    packed, absmax = nf4.quantize_stack(W)
    A32 = rng.standard_normal((a_rows, K)).astype(np.float32)
    Abits = workloads.to_bf16_bits(A32)
    offs = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    rows = int(offs[-1])
    ridx = rng.integers(0, a_rows, size=rows).astype(np.int32)
    la = lb = None
    if lora_r:
        la = workloads.to_bf16_bits((rng.standard_normal((E, lora_r, K)) * 0.05).astype(np.float32))
        lb = workloads.to_bf16_bits((rng.standard_normal((E, N, lora_r)) * 0.05).astype(np.float32))
    return dict(E=E, N=N, K=K, packed=packed, absmax=absmax, Abits=Abits, offs=offs, rows=rows, ridx=ridx,
                la=la, lb=lb, r=lora_r)


def _t_bf16(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def _run_gpu(c, epi, out_dtype, use_ridx=True, scale=2.0):
    ncols = c["N"] // 2 if epi == e4b.E4B_EPI_SWIGLU else c["N"]
    out = torch.full((c["rows"] + 1, ncols), float("nan"), dtype=out_dtype, device="cuda")   # +1 guard row
    ws = e4b.workspace(e4b.e4b_grouped_nf4_gemm_workspace_size(c["rows"], c["N"], c["K"], c["r"]))
    e4b.e4b_grouped_nf4_gemm(
        _t_bf16(c["Abits"]), torch.from_numpy(c["ridx"]).cuda() if use_ridx else None,
        torch.from_numpy(c["offs"]).cuda(), c["rows"], torch.from_numpy(c["packed"]).cuda(),
        torch.from_numpy(c["absmax"]).cuda(), c["N"], c["K"], out, epi,
        _t_bf16(c["la"]) if c["r"] else None, _t_bf16(c["lb"]) if c["r"] else None, scale, ws)
    torch.cuda.synchronize()
    assert e4b.workspace_error(ws) == e4b.E4B_KERNEL_ERR_NONE, "a kernel gave up a bounded wait"
    res = out.float().cpu().numpy().astype(np.float64)
    assert np.all(np.isnan(res[c["rows"]])), "guard row written"
    return res[:c["rows"]], e4b.last_path()


def _oracle(c, epi, use_ridx=True, scale=2.0):
    A = workloads.bf16_bits_to_f32(c["Abits"]).astype(np.float64)
    la = workloads.bf16_bits_to_f32(c["la"]).astype(np.float64) if c["r"] else None
    lb = workloads.bf16_bits_to_f32(c["lb"]).astype(np.float64) if c["r"] else None
    return moe.grouped_nf4_gemm(A, c["ridx"] if use_ridx else None, c["offs"], c["packed"], c["absmax"],
                                c["N"], c["K"], la, lb, scale, swiglu=(epi == e4b.E4B_EPI_SWIGLU))


def gemm_tolerance(path, epi, out_dtype):
    """Relative Frobenius tolerance of one grouped GEMM against the float64 oracle.

    Warp-MMA path: the only rounding of a weight is its codebook entry to bf16
    (relative error <= 2^-9; absmax is applied in fp32 per 64-block), so a plain
    fp32 output stays within 2e-3 and SwiGLU, the product of two such results,
    within 4e-3.  Tensor-core path: the decoded weight is rounded three times
    (codebook entry, absmax and their product, each <= 2^-9 relative, rms about
    2^-9 together), so 4e-3 plain and 6e-3 for SwiGLU.  bf16 outputs add one
    rounding of 2^-9: 1e-2 for both paths.
    """
    if out_dtype == torch.bfloat16:
        return 1e-2
    tc = path.startswith("gemm.tc")
    if epi == e4b.E4B_EPI_NONE:
        return 4e-3 if tc else 2e-3
    return 6e-3 if tc else 4e-3


CASES = [
    # E, N, K, counts (ragged, with empty groups), a_rows
    (3, 128, 256, [5, 0, 70], 40),
    (4, 192, 128, [1, 130, 0, 64], 200),
    (2, 64, 64, [0, 1], 3),
    (8, 256, 192, [17, 3, 0, 0, 65, 1, 33, 128], 100),
    # several n tiles with a ragged last one, several token tiles per group
    (4, 640, 320, [300, 0, 129, 77], 256),
]


@pytest.mark.parametrize("ci", range(len(CASES)))
@pytest.mark.parametrize("epi", [e4b.E4B_EPI_NONE, e4b.E4B_EPI_SWIGLU])
@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
def test_grouped_gemm_matches_oracle(ci, epi, out_dtype):
    require_gpu()
    E, N, K, counts, a_rows = CASES[ci]
    c = _case(E, N, K, counts, a_rows, seed=ci)
    got, path = _run_gpu(c, epi, out_dtype)
    ref = _oracle(c, epi)
    fro, mx = rel_errors(got, ref)
    tol = gemm_tolerance(path, epi, out_dtype)
    print(f"[parity] gemm case {ci} epi {epi} {out_dtype} path {path}: rel_fro={fro:.2e} max={mx:.2e}")
    assert fro <= tol and mx <= 2 * tol


@pytest.mark.parametrize("epi", [e4b.E4B_EPI_NONE, e4b.E4B_EPI_SWIGLU])
def test_grouped_gemm_lora(epi):
    require_gpu()
    c = _case(4, 256, 128, [3, 0, 80, 20], 64, seed=11, lora_r=8)
    got, path = _run_gpu(c, epi, torch.float32)
    ref = _oracle(c, epi)
    fro, mx = rel_errors(got, ref)
    tol = gemm_tolerance(path, epi, torch.float32)
    assert fro <= tol and mx <= 2 * tol
    # the delta matters: without it the result is off
    ref0 = _oracle(dict(c, r=0), epi)
    assert rel_errors(ref0, ref)[0] > 1e-2


def test_grouped_gemm_identity_rows_and_all_ones():
    require_gpu()
    c = _case(3, 64, 128, [10, 0, 6], 16, seed=3)
    got, path = _run_gpu(c, e4b.E4B_EPI_NONE, torch.float32, use_ridx=False)
    assert rel_errors(got, _oracle(c, e4b.E4B_EPI_NONE, use_ridx=False))[0] <= gemm_tolerance(
        path, e4b.E4B_EPI_NONE, torch.float32)
    # all codes 15, absmax 1 -> every output is the row sum of A (exact for small integers)
    c["packed"][:] = 0xFF
    c["absmax"][:] = 1.0
    c["Abits"] = workloads.to_bf16_bits(np.random.default_rng(4).integers(-3, 4, size=(16, 128)).astype(np.float32))
    got, _ = _run_gpu(c, e4b.E4B_EPI_NONE, torch.float32)
    A = workloads.bf16_bits_to_f32(c["Abits"]).astype(np.float64)
    want = A[c["ridx"]].sum(axis=1)[:, None] * np.ones((1, 64))
    assert np.array_equal(got, want)


def test_grouped_gemm_positive_control_flipped_nibble():
    require_gpu()
    c = _case(2, 64, 128, [8, 8], 16, seed=5)
    ref = _oracle(c, e4b.E4B_EPI_NONE)
    c["packed"][1, 0] ^= 0x88        # flip one byte of the second expert
    got, _ = _run_gpu(c, e4b.E4B_EPI_NONE, torch.float32)
    rows = slice(8, 16)
    assert np.max(np.abs(got[rows, 0] - ref[rows, 0])) > 1e-4


# The tensor-core kernel in each of its tile shapes (forced through the
# E4B_GEMM / E4B_TC_SHAPE switches, which apply to every call of the process):
# wide = 2 x 128 weight rows x 256 routed rows, double = 2 x 128 x 128 with two
# accumulator sets, narrow = 128 x 256 with two accumulator sets (plain
# epilogue only; a SwiGLU call takes the wide shape), tmem = 2 x 128 x 192 with
# the decoded weights in tensor memory (a LoRA or MXFP4 call takes the default).
TC_SHAPES = ["wide", "double", "narrow", "tmem"]
TC_CASES = CASES + [
    # several 256-row token tiles per group and a one-row group
    (3, 256, 512, [700, 1, 300], 500),
]


@pytest.mark.parametrize("shape", TC_SHAPES)
@pytest.mark.parametrize("ci", range(len(TC_CASES)))
@pytest.mark.parametrize("epi", [e4b.E4B_EPI_NONE, e4b.E4B_EPI_SWIGLU])
def test_grouped_gemm_tensor_core_shapes(monkeypatch, shape, ci, epi):
    require_gpu()
    monkeypatch.setenv("E4B_GEMM", "tc")
    monkeypatch.setenv("E4B_TC_SHAPE", shape)
    E, N, K, counts, a_rows = TC_CASES[ci]
    c = _case(E, N, K, counts, a_rows, seed=100 + ci)
    for use_ridx in (True, False):
        if not use_ridx:
            c["Abits"] = np.resize(c["Abits"], (max(1, c["rows"]), K))  # one A row per routed row
        got, path = _run_gpu(c, epi, torch.float32, use_ridx=use_ridx)
        assert path.startswith("gemm.tc"), path
        ref = _oracle(c, epi, use_ridx=use_ridx)
        fro, mx = rel_errors(got, ref)
        tol = gemm_tolerance(path, epi, torch.float32)
        print(f"[parity] tc {shape} case {ci} epi {epi} ridx {use_ridx}: rel_fro={fro:.2e} max={mx:.2e}")
        assert fro <= tol and mx <= 2 * tol


@pytest.mark.parametrize("shape", TC_SHAPES)
def test_grouped_gemm_tensor_core_bf16_and_exact_sums(monkeypatch, shape):
    require_gpu()
    monkeypatch.setenv("E4B_GEMM", "tc")
    monkeypatch.setenv("E4B_TC_SHAPE", shape)
    c = _case(4, 640, 320, [300, 0, 129, 77], 256, seed=7)
    for epi in (e4b.E4B_EPI_NONE, e4b.E4B_EPI_SWIGLU):
        got, path = _run_gpu(c, epi, torch.bfloat16)
        assert path.startswith("gemm.tc"), path
        fro, mx = rel_errors(got, _oracle(c, epi))
        assert fro <= 1e-2 and mx <= 2e-2
    # all codes 15, absmax 1: every output is the row sum of A, exact for small integers
    c["packed"][:] = 0xFF
    c["absmax"][:] = 1.0
    c["Abits"] = workloads.to_bf16_bits(np.random.default_rng(8).integers(-3, 4, size=(256, 320)).astype(np.float32))
    got, _ = _run_gpu(c, e4b.E4B_EPI_NONE, torch.float32)
    A = workloads.bf16_bits_to_f32(c["Abits"]).astype(np.float64)
    want = A[c["ridx"]].sum(axis=1)[:, None] * np.ones((1, 640))
    assert np.array_equal(got, want)


@pytest.mark.parametrize("shape", TC_SHAPES)
@pytest.mark.parametrize("r", [3, 8, 16])
@pytest.mark.parametrize("epi", [e4b.E4B_EPI_NONE, e4b.E4B_EPI_SWIGLU])
def test_grouped_gemm_tensor_core_lora(monkeypatch, shape, r, epi):
    """The tensor-core kernel's LoRA step (one K=16 MMA per tile on lora_B rows
    and bf16(scale * x . lora_A^T)): the extra rounding of the products to bf16
    is 2^-9 of the delta, inside the path's tolerance."""
    require_gpu()
    monkeypatch.setenv("E4B_GEMM", "tc")
    monkeypatch.setenv("E4B_TC_SHAPE", shape)
    c = _case(4, 640, 320, [300, 0, 129, 77], 256, seed=40 + r, lora_r=r)
    for use_ridx in (True, False):
        if not use_ridx:
            c["Abits"] = np.resize(c["Abits"], (c["rows"], c["K"]))
        got, path = _run_gpu(c, epi, torch.float32, use_ridx=use_ridx)
        assert path.startswith("gemm.tc"), path
        ref = _oracle(c, epi, use_ridx=use_ridx)
        fro, mx = rel_errors(got, ref)
        tol = gemm_tolerance(path, epi, torch.float32)
        print(f"[parity] tc lora {shape} r={r} epi {epi} ridx {use_ridx}: rel_fro={fro:.2e} max={mx:.2e}")
        assert fro <= tol and mx <= 2 * tol
        # the delta matters
        assert rel_errors(_oracle(dict(c, r=0), epi, use_ridx=use_ridx), ref)[0] > 1e-2


# The persistent regime of the tensor-core kernel: more than two tiles per CTA
# (the grid is min(tiles, SMs) and each CTA walks tiles with a stride of the
# grid), so accumulator hand-offs, barrier phases and ring slots carry over
# from tile to tile.  Group sizes are Zipf-like with empty groups, one-row
# groups and groups one row short of / past a 256-row tile; every output
# element is compared with the float64 oracle.
MULTI_COUNTS = [2900, 1500, 0, 1, 1000, 700, 0, 513, 256, 255, 1, 600, 300, 0, 900, 75]
MULTI_N, MULTI_K = 2048, 1024
_multi_cache = {}


def _multi_case(lora_r=0):
    key = ("case", lora_r)
    if key not in _multi_cache:
        _multi_cache[key] = _case(len(MULTI_COUNTS), MULTI_N, MULTI_K, MULTI_COUNTS, 4096, seed=77 + lora_r,
                                  lora_r=lora_r)
    return _multi_cache[key]


def _multi_oracle(c, epi, lora_r):
    key = ("ref", lora_r, epi)
    if key not in _multi_cache:
        _multi_cache[key] = _oracle(c, epi)
    return _multi_cache[key]


def _tc_tile_count(counts, n_out_cols, wrows, bn):
    n_tiles = -(-n_out_cols // wrows)
    return sum(-(-c // bn) for c in counts) * n_tiles


@pytest.mark.parametrize("shape", TC_SHAPES)
@pytest.mark.parametrize("epi", [e4b.E4B_EPI_NONE, e4b.E4B_EPI_SWIGLU])
def test_grouped_gemm_tensor_core_persistent_full_output(monkeypatch, shape, epi):
    require_gpu()
    monkeypatch.setenv("E4B_GEMM", "tc")
    monkeypatch.setenv("E4B_TC_SHAPE", shape)
    swiglu = epi == e4b.E4B_EPI_SWIGLU
    eff_shape = "wide" if (shape == "narrow" and swiglu) else shape
    bn = 128 if eff_shape == "double" else 256
    wrows = 128 if (swiglu or eff_shape == "narrow") else 256
    tiles = _tc_tile_count(MULTI_COUNTS, MULTI_N // 2 if swiglu else MULTI_N, wrows, bn)
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    assert tiles > 2 * sms, f"{tiles} tiles do not give every CTA a third tile"
    c = _multi_case()
    got, path = _run_gpu(c, epi, torch.float32)
    assert path.startswith("gemm.tc"), path
    ref = _multi_oracle(c, epi, 0)
    fro, mx = rel_errors(got, ref)
    tol = gemm_tolerance(path, epi, torch.float32)
    print(f"[parity] tc persistent {shape} epi {epi} tiles {tiles}: rel_fro={fro:.2e} max={mx:.2e}")
    assert fro <= tol and mx <= 2 * tol
    # and per routed row: a fault confined to a few late tiles must not hide in the norm
    row_err = np.linalg.norm(got - ref, axis=1) / np.maximum(np.linalg.norm(ref, axis=1), 1e-30)
    assert float(row_err.max()) <= 4 * tol, f"worst row {int(row_err.argmax())}: {row_err.max():.2e}"


def test_grouped_gemm_tensor_core_persistent_lora(monkeypatch):
    require_gpu()
    monkeypatch.setenv("E4B_GEMM", "tc")
    c = _multi_case(lora_r=8)
    got, path = _run_gpu(c, e4b.E4B_EPI_SWIGLU, torch.float32)
    assert path.startswith("gemm.tc"), path
    ref = _multi_oracle(c, e4b.E4B_EPI_SWIGLU, 8)
    fro, mx = rel_errors(got, ref)
    tol = gemm_tolerance(path, e4b.E4B_EPI_SWIGLU, torch.float32)
    print(f"[parity] tc persistent lora: rel_fro={fro:.2e} max={mx:.2e}")
    assert fro <= tol and mx <= 2 * tol
    row_err = np.linalg.norm(got - ref, axis=1) / np.maximum(np.linalg.norm(ref, axis=1), 1e-30)
    assert float(row_err.max()) <= 4 * tol
