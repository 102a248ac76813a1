"""GPU grouped MXFP4 GEMM vs the float64 oracle (oracle/mxfp4.py).

Both kernels: the warp-MMA kernel (below 512 routed rows) and the tcgen05
kernel with MXFP4 decoders (from 512 rows), each forced through E4B_GEMM.

Tolerance: e2m1 values are exact in bf16 and the e8m0 scale is a power of two
(applied in fp32 after the warp MMAs, or to the bf16 weight exactly before the
tensor-core MMAs), so the only error is the accumulation over K products:
1e-5 relative Frobenius for fp32 output on the warp MMAs (IEEE fp32 adds),
1e-4 on the tensor cores (whose fp32 accumulation is not specified to round
like IEEE adds); bf16 output adds one rounding of 2^-9: 5e-3.
"""
import numpy as np
import pytest
import torch

from oracle import moe, mxfp4
from quantized_moe_expert_nf4_b200 import e4b, workloads
from gpu_util import rel_errors, require_gpu

pytestmark = pytest.mark.gpu


def _case(E, N, K, counts, a_rows, seed):
    rng = np.random.default_rng(seed)
    blocks = rng.integers(0, 256, size=(E, N * K // 2), dtype=np.uint8)
    scales = rng.integers(118, 129, size=(E, N * K // 32), dtype=np.uint8)
    Abits = workloads.to_bf16_bits(rng.standard_normal((a_rows, K)).astype(np.float32))
    offs = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    rows = int(offs[-1])
    ridx = rng.integers(0, a_rows, size=rows).astype(np.int32)
    return dict(E=E, N=N, K=K, blocks=blocks, scales=scales, Abits=Abits, offs=offs, rows=rows, ridx=ridx)


def _run(c, epi, out_dtype):
    ncols = c["N"] // 2 if epi == e4b.E4B_EPI_SWIGLU else c["N"]
    out = torch.full((c["rows"] + 1, ncols), float("nan"), dtype=out_dtype, device="cuda")
    A = torch.from_numpy(c["Abits"].view(np.int16)).view(torch.bfloat16).cuda()
    ws = e4b.workspace(e4b.e4b_grouped_mxfp4_gemm_workspace_size(c["rows"], c["N"], c["K"]))
    e4b.e4b_grouped_mxfp4_gemm(A, torch.from_numpy(c["ridx"]).cuda(), torch.from_numpy(c["offs"]).cuda(), c["rows"],
                               torch.from_numpy(c["blocks"]).cuda(), torch.from_numpy(c["scales"]).cuda(), c["N"],
                               c["K"], out, epi, ws)
    torch.cuda.synchronize()
    assert e4b.workspace_error(ws) == e4b.E4B_KERNEL_ERR_NONE, "a kernel gave up a bounded wait"
    res = out.float().cpu().numpy().astype(np.float64)
    assert np.all(np.isnan(res[c["rows"]])), "guard row written"
    return res[:c["rows"]], e4b.last_path()


def _oracle(c, epi):
    A = workloads.bf16_bits_to_f32(c["Abits"]).astype(np.float64)
    y = mxfp4.grouped_mxfp4_gemm(A, c["ridx"], c["offs"], c["blocks"], c["scales"], c["N"], c["K"])
    if epi == e4b.E4B_EPI_SWIGLU:
        y = moe.silu(y[:, :c["N"] // 2]) * y[:, c["N"] // 2:]
    return y


CASES = [
    (3, 128, 256, [5, 0, 70], 40),
    (4, 192, 128, [1, 130, 0, 64], 200),
    (2, 64, 64, [0, 1], 3),
    (4, 640, 2880 // 64 * 64, [300, 0, 129, 77], 256),   # gpt-oss-like K (2880 = 45 x 64)
]


@pytest.mark.parametrize("kernel", ["mma", "tc"])
@pytest.mark.parametrize("ci", range(len(CASES)))
@pytest.mark.parametrize("epi", [e4b.E4B_EPI_NONE, e4b.E4B_EPI_SWIGLU])
@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
def test_grouped_mxfp4_gemm_matches_oracle(monkeypatch, kernel, ci, epi, out_dtype):
    require_gpu()
    monkeypatch.setenv("E4B_GEMM", kernel)
    c = _case(*CASES[ci], seed=30 + ci)
    got, path = _run(c, epi, out_dtype)
    assert path.startswith("mxfp4." + kernel), path
    fro, mx = rel_errors(got, _oracle(c, epi))
    tol = 5e-3 if out_dtype == torch.bfloat16 else (1e-4 if kernel == "tc" else 1e-5)
    print(f"[parity] mxfp4 case {ci} epi {epi} {out_dtype}: rel_fro={fro:.2e} max={mx:.2e}")
    assert fro <= tol and mx <= 2 * tol


@pytest.mark.parametrize("kernel", ["mma", "tc"])
def test_grouped_mxfp4_nan_scale_and_nibble_order(monkeypatch, kernel):
    """A NaN scale (255) makes exactly its block's outputs NaN; swapping the
    nibbles of the codes (the other packing order) changes the result."""
    require_gpu()
    monkeypatch.setenv("E4B_GEMM", kernel)
    c = _case(2, 64, 128, [20, 10], 30, seed=40)
    c["scales"][1, :] = 127
    c["scales"][1, 5] = 255    # expert 1, row 1 (its scale blocks 4..7), block 5
    got, _ = _run(c, e4b.E4B_EPI_NONE, torch.float32)
    assert np.all(np.isnan(got[20:, 1])) and not np.isnan(got[20:, [0] + list(range(2, 64))]).any()
    assert not np.isnan(got[:20]).any()
    ref = _oracle(c, e4b.E4B_EPI_NONE)
    swapped = dict(c)
    swapped["blocks"] = ((c["blocks"] & 0x0F) << 4) | (c["blocks"] >> 4)
    got2, _ = _run(swapped, e4b.E4B_EPI_NONE, torch.float32)
    fin = np.isfinite(ref)
    assert rel_errors(got2[fin], ref[fin])[0] > 1e-2


def test_grouped_mxfp4_size_choice():
    """Without a forced kernel: the warp MMAs below 512 routed rows, the
    tensor cores from 512 (both against the oracle)."""
    require_gpu()
    for counts, kind in (([100, 0, 300], "mxfp4.mma"), ([300, 50, 400], "mxfp4.tc")):
        c = _case(3, 128, 256, counts, 500, seed=41)
        got, path = _run(c, e4b.E4B_EPI_SWIGLU, torch.float32)
        assert path.startswith(kind), path
        fro, _ = rel_errors(got, _oracle(c, e4b.E4B_EPI_SWIGLU))
        assert fro <= 1e-4
