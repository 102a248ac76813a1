"""GPU grouped NF4 dgrad (input gradient through the frozen base) vs the float64 oracle.

Tolerance: the kernels round each decoded weight three times (codebook entry,
absmax and their product, each <= 2^-9 relative, so <= 3 * 2^-9 ~ 5.9e-3 per
weight) and accumulate in fp32, so an fp32 result stays within 6e-3 relative
Frobenius (max-abs within twice that of max|ref|); a bf16 result adds one
rounding of 2^-9: 1e-2.  (A numpy model with exactly these roundings gives
2.5e-3 to 2.8e-3 on the cases below.)
"""
import numpy as np
import pytest
import torch

from oracle import backward, nf4
from quantized_moe_expert_nf4_b200 import e4b, workloads
from gpu_util import rel_errors, require_gpu

pytestmark = pytest.mark.gpu


def _case(E, N, K, counts, dy_rows, seed, lora_r=0):
    rng = np.random.default_rng(seed)
    W = (rng.standard_normal((E, N, K)) * 0.02).astype(np.float32)
    packed, absmax = nf4.quantize_stack(W)
    dYbits = workloads.to_bf16_bits(rng.standard_normal((dy_rows, N)).astype(np.float32))
    offs = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    rows = int(offs[-1])
    ridx = rng.integers(0, dy_rows, size=rows).astype(np.int32)
    la = lb = None
    if lora_r:
        la = workloads.to_bf16_bits((rng.standard_normal((E, lora_r, K)) * 0.05).astype(np.float32))
        lb = workloads.to_bf16_bits((rng.standard_normal((E, N, lora_r)) * 0.05).astype(np.float32))
    return dict(E=E, N=N, K=K, packed=packed, absmax=absmax, dYbits=dYbits, offs=offs, rows=rows, ridx=ridx,
                la=la, lb=lb, r=lora_r)


def _t_bf16(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def _run_gpu(c, out_dtype, use_ridx=True, scale=2.0):
    out = torch.full((c["rows"] + 1, c["K"]), float("nan"), dtype=out_dtype, device="cuda")   # +1 guard row
    ws = e4b.workspace(e4b.e4b_grouped_nf4_gemm_dgrad_workspace_size(c["rows"], c["N"], c["K"], c["r"]))
    e4b.e4b_grouped_nf4_gemm_dgrad(
        _t_bf16(c["dYbits"]), torch.from_numpy(c["ridx"]).cuda() if use_ridx else None,
        torch.from_numpy(c["offs"]).cuda(), c["rows"], torch.from_numpy(c["packed"]).cuda(),
        torch.from_numpy(c["absmax"]).cuda(), c["N"], c["K"], out,
        _t_bf16(c["la"]) if c["r"] else None, _t_bf16(c["lb"]) if c["r"] else None, scale, ws)
    torch.cuda.synchronize()
    path = e4b.last_path()
    assert e4b.workspace_error(ws) == e4b.E4B_KERNEL_ERR_NONE
    res = out.float().cpu().numpy().astype(np.float64)
    assert np.all(np.isnan(res[c["rows"]])), "guard row written"
    return res[:c["rows"]], path


def _oracle(c, use_ridx=True, scale=2.0):
    dY = workloads.bf16_bits_to_f32(c["dYbits"]).astype(np.float64)
    la = workloads.bf16_bits_to_f32(c["la"]).astype(np.float64) if c["r"] else None
    lb = workloads.bf16_bits_to_f32(c["lb"]).astype(np.float64) if c["r"] else None
    return backward.grouped_nf4_gemm_dgrad(dY, c["ridx"] if use_ridx else None, c["offs"], c["packed"],
                                           c["absmax"], c["N"], c["K"], la, lb, scale)


def _tol(out_dtype):
    return 1e-2 if out_dtype == torch.bfloat16 else 6e-3


CASES = [
    # E, N (contraction), K (columns of dX), counts (ragged, with empty groups), dY rows
    (3, 128, 256, [5, 0, 70], 40),
    (4, 192, 128, [1, 130, 0, 64], 200),
    (2, 64, 64, [0, 1], 3),
    (8, 256, 192, [17, 3, 0, 0, 65, 1, 33, 128], 100),
    (4, 640, 320, [300, 0, 129, 77], 256),
]


@pytest.mark.parametrize("kernel", ["mma", "tc"])
@pytest.mark.parametrize("ci", range(len(CASES)))
@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
def test_grouped_dgrad_matches_oracle(monkeypatch, kernel, ci, out_dtype):
    """Both kernels (warp MMA; tcgen05 with the transposing decoders), forced."""
    require_gpu()
    monkeypatch.setenv("E4B_DGRAD", kernel)
    c = _case(*CASES[ci], seed=ci)
    got, path = _run_gpu(c, out_dtype)
    ref = _oracle(c)
    fro, mx = rel_errors(got, ref)
    print(f"[parity] dgrad case {ci} {out_dtype} path {path}: rel_fro={fro:.2e} max={mx:.2e}")
    assert path == f"dgrad.{kernel}"
    assert fro <= _tol(out_dtype) and mx <= 2 * _tol(out_dtype)


@pytest.mark.parametrize("shape", ["wide", "double"])
def test_grouped_dgrad_tensor_core_shapes_and_size_choice(monkeypatch, shape):
    """Both tile shapes of the tensor-core dgrad, a column count that is not a
    multiple of the 256-column tile, and the automatic choice for >= 512 rows."""
    require_gpu()
    monkeypatch.setenv("E4B_TC_SHAPE", shape)
    c = _case(3, 320, 704, [600, 0, 45], 700, seed=21)
    got, path = _run_gpu(c, torch.float32)
    assert path == "dgrad.tc"
    fro, mx = rel_errors(got, _oracle(c))
    assert fro <= 6e-3 and mx <= 1.2e-2


@pytest.mark.parametrize("kernel", ["mma", "tc"])
@pytest.mark.parametrize("r", [3, 8, 16])
def test_grouped_dgrad_lora(monkeypatch, kernel, r):
    require_gpu()
    monkeypatch.setenv("E4B_DGRAD", kernel)
    c = _case(4, 192, 256, [33, 0, 100, 7], 90, seed=10 + r, lora_r=r)
    got, _ = _run_gpu(c, torch.float32, scale=16.0 / r)
    ref = _oracle(c, scale=16.0 / r)
    fro, mx = rel_errors(got, ref)
    assert fro <= 6e-3 and mx <= 1.2e-2
    # the adapter's share is not negligible here, so the check covers it
    base = _oracle(dict(c, r=0, la=None, lb=None))
    assert rel_errors(base, ref)[0] > 5e-2


def test_grouped_dgrad_identity_rows():
    require_gpu()
    c = _case(3, 128, 128, [40, 24, 0], 64, seed=3)
    got, _ = _run_gpu(c, torch.float32, use_ridx=False)
    ref = _oracle(c, use_ridx=False)
    assert rel_errors(got, ref)[0] <= 6e-3


def test_grouped_dgrad_positive_control_flipped_nibble():
    """A wrong nibble in one weight row must show in the columns it feeds."""
    require_gpu()
    c = _case(2, 128, 128, [50, 30], 80, seed=4)
    ref = _oracle(c)
    bad = dict(c)
    bad["packed"] = c["packed"].copy()
    bad["packed"][0, :32] ^= 0x88   # row 0 of expert 0: flip the top bit of 64 codes
    got, _ = _run_gpu(bad, torch.float32)
    assert rel_errors(got[:50], ref[:50])[0] > 1e-2


def test_grouped_dgrad_is_the_adjoint_of_the_gpu_gemm():
    """<dY, gemm(A)> = <dgrad(dY), A> with both products from the library."""
    require_gpu()
    rng = np.random.default_rng(6)
    E, N, K = 3, 256, 192
    W = (rng.standard_normal((E, N, K)) * 0.02).astype(np.float32)
    packed, absmax = nf4.quantize_stack(W)
    offs = np.array([0, 100, 100, 230], dtype=np.int32)
    rows = 230
    A = torch.randn(rows, K, dtype=torch.float32).to(torch.bfloat16).cuda()
    dY = torch.randn(rows, N, dtype=torch.float32).to(torch.bfloat16).cuda()
    tp, ta, to = torch.from_numpy(packed).cuda(), torch.from_numpy(absmax).cuda(), torch.from_numpy(offs).cuda()
    y = torch.empty(rows, N, dtype=torch.float32, device="cuda")
    ws = e4b.workspace(e4b.e4b_grouped_nf4_gemm_workspace_size(rows, N, K, 0))
    e4b.e4b_grouped_nf4_gemm(A, None, to, rows, tp, ta, N, K, y, workspace=ws)
    dx = torch.empty(rows, K, dtype=torch.float32, device="cuda")
    wsd = e4b.workspace(e4b.e4b_grouped_nf4_gemm_dgrad_workspace_size(rows, N, K, 0))
    e4b.e4b_grouped_nf4_gemm_dgrad(dY, None, to, rows, tp, ta, N, K, dx, workspace=wsd)
    torch.cuda.synchronize()
    lhs = float((dY.double() * y.double()).sum())
    rhs = float((dx.double() * A.double()).sum())
    scale = float(dY.double().abs().mean() * y.double().abs().mean()) * rows * N
    assert abs(lhs - rhs) <= 1e-2 * scale


def test_grouped_dgrad_empty_and_errors():
    require_gpu()
    c = _case(2, 64, 64, [0, 0], 4, seed=5)
    out = torch.empty((1, 64), dtype=torch.float32, device="cuda")
    e4b.e4b_grouped_nf4_gemm_dgrad(_t_bf16(c["dYbits"]), None, torch.from_numpy(c["offs"]).cuda(), 0,
                                   torch.from_numpy(c["packed"]).cuda(), torch.from_numpy(c["absmax"]).cuda(),
                                   64, 64, out)
    assert e4b.last_path() == "dgrad.empty"
    with pytest.raises(e4b.E4BError, match="N must be"):
        e4b.e4b_grouped_nf4_gemm_dgrad(_t_bf16(c["dYbits"]), None, torch.from_numpy(c["offs"]).cuda(), 0,
                                       torch.from_numpy(c["packed"]).cuda(), torch.from_numpy(c["absmax"]).cuda(),
                                       96, 64, out)


@pytest.mark.parametrize("r", [1, 8, 16])
def test_grouped_lora_grads_match_oracle(r):
    """dA, dB of one grouped projection: ragged and empty groups, a row gather."""
    require_gpu()
    rng = np.random.default_rng(40 + r)
    E, N, K = 4, 192, 256
    counts = [70, 0, 3, 200]
    offs = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    rows = int(offs[-1])
    x_rows = 300
    xbits = workloads.to_bf16_bits(rng.standard_normal((x_rows, K)).astype(np.float32))
    dabits = workloads.to_bf16_bits(rng.standard_normal((rows, N)).astype(np.float32))
    ridx = rng.integers(0, x_rows, size=rows).astype(np.int32)
    la = workloads.to_bf16_bits((rng.standard_normal((E, r, K)) * 0.05).astype(np.float32))
    lb = workloads.to_bf16_bits((rng.standard_normal((E, N, r)) * 0.05).astype(np.float32))
    scale = 16.0 / r
    dA = torch.full((E, r, K), float("nan"), dtype=torch.float32, device="cuda")
    dB = torch.full((E, N, r), float("nan"), dtype=torch.float32, device="cuda")
    ws = e4b.workspace(e4b.e4b_grouped_lora_grads_workspace_size(rows, r))
    e4b.e4b_grouped_lora_grads(_t_bf16(xbits), torch.from_numpy(ridx).cuda(), torch.from_numpy(offs).cuda(), rows,
                               _t_bf16(dabits), N, K, _t_bf16(la), _t_bf16(lb), scale, dA, dB, ws)
    torch.cuda.synchronize()
    assert e4b.last_path() == "lora_grads"
    f = lambda b: workloads.bf16_bits_to_f32(b).astype(np.float64)
    rA, rB = backward.grouped_lora_grads(f(xbits), ridx, offs, f(dabits), f(la), f(lb), scale)
    gA, gB = dA.cpu().numpy().astype(np.float64), dB.cpu().numpy().astype(np.float64)
    assert np.all(gA[1] == 0) and np.all(gB[1] == 0)   # the empty group
    # inputs are exact bf16 values; fp32 accumulation over <= 200 rows and <= 256 terms
    for got, ref in ((gA, rA), (gB, rB)):
        fro, mx = rel_errors(got, ref)
        assert fro <= 1e-4 and mx <= 1e-3
