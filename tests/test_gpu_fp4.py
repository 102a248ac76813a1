"""FP4 storage on the GPU vs the float64 oracle.

The FP4 stack is the NF4 layout with the e2m1 / 6 codebook: the quantiser is
checked bit for bit, and the grouped GEMM (warp-MMA and tensor-core kernels),
the dgrad product, the layer forward (decode and grouped paths) and the layer
backward against the oracle reading the same bytes as FP4.  The tolerances
are those of the NF4 tests: each FP4 entry is rounded to bf16 with the same
relative error bound (2^-9) as an NF4 entry.  Every test also checks that the
FP4 reading matters: the oracle's NF4 reading of the same bytes is far off.
"""
import numpy as np
import pytest
import torch

from oracle import backward, fp4, moe, nf4, routing
from quantized_moe_expert_nf4_b200 import e4b, synthetic, workloads
from gpu_util import assert_close_layer, bf16_to_f64, rel_errors, require_gpu

pytestmark = pytest.mark.gpu
FP4 = e4b.E4B_QUANT_FP4


def _gpu_quantize(W: torch.Tensor, quant=FP4):
    E, N, K = W.shape
    packed = torch.empty((E, N * K // 2), dtype=torch.uint8, device="cuda")
    absmax = torch.empty((E, N * K // 64), dtype=torch.float32, device="cuda")
    e4b.e4b_quantize_stack(W, packed, absmax, quant)
    torch.cuda.synchronize()
    assert e4b.last_path() == "quantize"
    return packed.cpu().numpy(), absmax.cpu().numpy()


@pytest.mark.parametrize("E,N,K", [(1, 1, 64), (3, 5, 64), (2, 7, 192), (4, 33, 128), (2, 9, 320)])
def test_fp4_quantize_bit_exact(E, N, K):
    require_gpu()
    rng = np.random.default_rng(E * 100 + N * 10 + K + 7)
    W = (rng.standard_normal((E, N, K)) * 0.02).astype(np.float32)
    W[0, 0, :64] = 0.0                                # an all-zero block
    W.reshape(-1)[-5] = -0.0
    gp, ga = _gpu_quantize(torch.from_numpy(W).cuda())
    op, oa = fp4.quantize_stack(W)
    assert np.array_equal(ga.view(np.uint32), oa.view(np.uint32))
    assert np.array_equal(gp, op)
    assert not np.any(nf4.unpack_codes(gp) == 8), "code 8 (-0) is never written"


def test_fp4_quantize_decision_points_and_bf16_input():
    require_gpu()
    mids = fp4.midpoints()
    vals = []
    for m in mids:
        f = np.float32(m)
        vals += [f, np.nextafter(f, np.float32(-2)), np.nextafter(f, np.float32(2))]
    h = np.float32(fp4.codebook_f64()[1] / 2)      # the two decision points that are floats
    vals += [h, -h, np.float32(0.0), np.float32(-0.0)]
    vals = np.array(vals, np.float32)
    n = (len(vals) + 62) // 63 * 63
    blk = np.zeros((n // 63, 64), np.float32)
    blk[:, 0] = 1.0                                  # absmax 1: s = w exactly
    blk[:, 1:].reshape(-1)[:len(vals)] = vals
    Wt = blk.reshape(1, -1, 64)
    gp, ga = _gpu_quantize(torch.from_numpy(Wt).cuda())
    op, oa = fp4.quantize_stack(Wt)
    assert np.array_equal(gp, op) and np.array_equal(ga, oa)
    # bf16 input
    rng = np.random.default_rng(9)
    bits = workloads.to_bf16_bits((rng.standard_normal((3, 64, 128)) * 0.05).astype(np.float32))
    Wb = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).cuda()
    gp, ga = _gpu_quantize(Wb)
    op, oa = fp4.quantize_stack(workloads.bf16_bits_to_f32(bits))
    assert np.array_equal(ga, oa) and np.array_equal(gp, op)


def test_fp4_and_nf4_quantisers_differ_and_each_matches_its_oracle():
    require_gpu()
    rng = np.random.default_rng(10)
    W = (rng.standard_normal((2, 16, 128)) * 0.02).astype(np.float32)
    Wd = torch.from_numpy(W).cuda()
    gp4, _ = _gpu_quantize(Wd, FP4)
    gpn, _ = _gpu_quantize(Wd, e4b.E4B_QUANT_NF4)
    assert np.array_equal(gp4, fp4.quantize_stack(W)[0])
    assert np.array_equal(gpn, nf4.quantize_stack(W)[0])
    assert np.mean(gp4 != gpn) > 0.5


def test_fp4_quantize_rejects_an_unknown_storage_type():
    require_gpu()
    W = torch.zeros((1, 1, 64), dtype=torch.float32, device="cuda")
    p = torch.empty(32, dtype=torch.uint8, device="cuda")
    a = torch.empty(1, dtype=torch.float32, device="cuda")
    with pytest.raises(e4b.E4BError, match="quant_type"):
        e4b.e4b_quantize_stack(W, p, a, 2)


def _t_bf16(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def _gemm_case(E, N, K, counts, a_rows, seed):
    rng = np.random.default_rng(seed)
    packed, absmax = fp4.quantize_stack((rng.standard_normal((E, N, K)) * 0.02).astype(np.float32))
    Abits = workloads.to_bf16_bits(rng.standard_normal((a_rows, K)).astype(np.float32))
    offs = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    ridx = rng.integers(0, a_rows, size=int(offs[-1])).astype(np.int32)
    return dict(E=E, N=N, K=K, packed=packed, absmax=absmax, Abits=Abits, offs=offs, rows=int(offs[-1]), ridx=ridx)


def _gemm_tol(path, epi):
    tc = path.startswith("gemm.tc")
    if epi == e4b.E4B_EPI_NONE:
        return 4e-3 if tc else 2e-3
    return 6e-3 if tc else 4e-3


@pytest.mark.parametrize("kernel", ["mma", "tc"])
@pytest.mark.parametrize("epi", [e4b.E4B_EPI_NONE, e4b.E4B_EPI_SWIGLU])
def test_fp4_grouped_gemm(monkeypatch, kernel, epi):
    require_gpu()
    monkeypatch.setenv("E4B_GEMM", kernel)
    c = _gemm_case(4, 640, 320, [300, 0, 129, 77], 256, seed=11)
    ncols = c["N"] // 2 if epi == e4b.E4B_EPI_SWIGLU else c["N"]
    out = torch.full((c["rows"] + 1, ncols), float("nan"), dtype=torch.float32, device="cuda")
    ws = e4b.workspace(e4b.e4b_grouped_nf4_gemm_workspace_size(c["rows"], c["N"], c["K"], 0))
    e4b.e4b_grouped_4bit_gemm(_t_bf16(c["Abits"]), torch.from_numpy(c["ridx"]).cuda(),
                              torch.from_numpy(c["offs"]).cuda(), c["rows"], torch.from_numpy(c["packed"]).cuda(),
                              torch.from_numpy(c["absmax"]).cuda(), c["N"], c["K"], out, FP4, epi, workspace=ws)
    torch.cuda.synchronize()
    path = e4b.last_path()
    assert path.startswith("gemm." + kernel), path
    assert e4b.workspace_error(ws) == e4b.E4B_KERNEL_ERR_NONE
    got = out.cpu().numpy().astype(np.float64)
    assert np.all(np.isnan(got[c["rows"]])), "guard row written"
    A = workloads.bf16_bits_to_f32(c["Abits"]).astype(np.float64)
    sw = epi == e4b.E4B_EPI_SWIGLU
    ref = moe.grouped_nf4_gemm(A, c["ridx"], c["offs"], c["packed"], c["absmax"], c["N"], c["K"], swiglu=sw,
                               quant="fp4")
    fro, mx = rel_errors(got[:c["rows"]], ref)
    tol = _gemm_tol(path, epi)
    print(f"[parity] fp4 gemm {kernel} epi {epi}: rel_fro={fro:.2e} max={mx:.2e}")
    assert fro <= tol and mx <= 2 * tol
    wrong = moe.grouped_nf4_gemm(A, c["ridx"], c["offs"], c["packed"], c["absmax"], c["N"], c["K"], swiglu=sw)
    assert rel_errors(got[:c["rows"]], wrong)[0] > 5e-2


@pytest.mark.parametrize("kernel", ["mma", "tc"])
def test_fp4_grouped_dgrad(monkeypatch, kernel):
    require_gpu()
    monkeypatch.setenv("E4B_DGRAD", kernel)
    c = _gemm_case(4, 640, 320, [300, 0, 129, 77], 256, seed=12)   # N = 640 contraction, K = 320 columns
    out = torch.full((c["rows"], c["K"]), float("nan"), dtype=torch.float32, device="cuda")
    ws = e4b.workspace(e4b.e4b_grouped_nf4_gemm_dgrad_workspace_size(c["rows"], c["N"], c["K"], 0))
    rng = np.random.default_rng(13)
    dYbits = workloads.to_bf16_bits(rng.standard_normal((256, c["N"])).astype(np.float32))
    e4b.e4b_grouped_4bit_gemm_dgrad(_t_bf16(dYbits), torch.from_numpy(c["ridx"]).cuda(),
                                    torch.from_numpy(c["offs"]).cuda(), c["rows"],
                                    torch.from_numpy(c["packed"]).cuda(), torch.from_numpy(c["absmax"]).cuda(),
                                    c["N"], c["K"], out, FP4, workspace=ws)
    torch.cuda.synchronize()
    path = e4b.last_path()
    assert path.startswith("dgrad." + kernel), path
    assert e4b.workspace_error(ws) == e4b.E4B_KERNEL_ERR_NONE
    got = out.cpu().numpy().astype(np.float64)
    dY = workloads.bf16_bits_to_f32(dYbits).astype(np.float64)
    ref = backward.grouped_nf4_gemm_dgrad(dY, c["ridx"], c["offs"], c["packed"], c["absmax"], c["N"], c["K"],
                                          quant="fp4")
    fro, mx = rel_errors(got, ref)
    print(f"[parity] fp4 dgrad {kernel}: rel_fro={fro:.2e} max={mx:.2e}")
    assert fro <= 6e-3 and mx <= 1.2e-2
    wrong = backward.grouped_nf4_gemm_dgrad(dY, c["ridx"], c["offs"], c["packed"], c["absmax"], c["N"], c["K"])
    assert rel_errors(got, wrong)[0] > 5e-2


def _oracle_stack(cfg):
    gp, ga = fp4.quantize_stack(workloads.gate_up_stack(cfg))
    dp, da = fp4.quantize_stack(workloads.down_stack(cfg))
    la = lb = None
    if cfg.lora_r:
        la = workloads.bf16_bits_to_f32(workloads.lora_A(cfg)).astype(np.float64)
        lb = workloads.bf16_bits_to_f32(workloads.lora_B(cfg)).astype(np.float64)
    return moe.ExpertStack(gp, ga, dp, da, cfg.E, cfg.H, cfg.I, la, lb, workloads.lora_scale(cfg), quant="fp4")


LAYERS = [
    ("tiny", workloads.CONFIGS["tiny"]),
    ("lora", workloads.small_config("lora", E=6, H=128, I=192, k=2, lora_r=8, lora_alpha=16.0)),
    ("ragged", workloads.small_config("ragged", E=12, H=192, I=320, k=3)),
]


@pytest.mark.parametrize("name,cfg", LAYERS, ids=[c[0] for c in LAYERS])
@pytest.mark.parametrize("path,M", [(e4b.E4B_PATH_DECODE, 5), (e4b.E4B_PATH_GROUPED, 64)])
def test_fp4_layer_forward(name, cfg, path, M):
    require_gpu()
    layer = synthetic.make_device_layer(cfg, quant_type=FP4)
    st = _oracle_stack(cfg)
    assert np.array_equal(layer.gu_packed.cpu().numpy(), st.gu_packed)
    assert np.array_equal(layer.dn_absmax.cpu().numpy(), st.dn_absmax)
    x, logits = synthetic.inputs(cfg, M)
    out = torch.full((M, cfg.H), float("nan"), dtype=torch.bfloat16, device="cuda")
    ws = e4b.workspace(e4b.e4b_moe_expert_forward_workspace_size(M, layer.stack, cfg.k))
    e4b.e4b_moe_expert_forward(x, logits, cfg.k, True, layer.stack, out, ws, path=path)
    torch.cuda.synchronize()
    p = e4b.last_path()
    assert p == ("forward.decode" if path == e4b.E4B_PATH_DECODE else "forward.grouped"), p
    assert e4b.workspace_error(ws) == e4b.E4B_KERNEL_ERR_NONE
    lg = logits.cpu().numpy()
    ids = routing.topk(lg, cfg.k)
    w = routing.route_weights(lg, ids)
    ref = moe.moe_forward_per_token(bf16_to_f64(x), ids, w, st)
    assert_close_layer(bf16_to_f64(out), ref, f"fp4 {name} M={M} {p}")
    st_nf4 = moe.ExpertStack(st.gu_packed, st.gu_absmax, st.dn_packed, st.dn_absmax, cfg.E, cfg.H, cfg.I,
                             st.lora_A, st.lora_B, st.lora_scale)
    assert rel_errors(bf16_to_f64(out), moe.moe_forward_per_token(bf16_to_f64(x), ids, w, st_nf4))[0] > 5e-2


def test_fp4_layer_backward():
    require_gpu()
    cfg = workloads.small_config("lora", E=6, H=128, I=192, k=2, lora_r=8, lora_alpha=16.0)
    M = 50
    layer = synthetic.make_device_layer(cfg, quant_type=FP4)
    x, logits = synthetic.inputs(cfg, M)
    rng = np.random.default_rng(14)
    dout_bits = workloads.to_bf16_bits(rng.standard_normal((M, cfg.H)).astype(np.float32))
    dout = torch.from_numpy(dout_bits.view(np.int16)).view(torch.bfloat16).cuda()
    dx = torch.full((M, cfg.H), float("nan"), dtype=torch.float32, device="cuda")
    dl = torch.full((M, cfg.E), float("nan"), dtype=torch.float32, device="cuda")
    dA = torch.full((cfg.E, cfg.lora_r, cfg.H), float("nan"), dtype=torch.float32, device="cuda")
    dB = torch.full((cfg.E, 2 * cfg.I, cfg.lora_r), float("nan"), dtype=torch.float32, device="cuda")
    ws = e4b.workspace(e4b.e4b_moe_expert_backward_workspace_size(M, layer.stack, cfg.k))
    e4b.e4b_moe_expert_backward(x, logits, cfg.k, True, layer.stack, dout, dx, dl, dA, dB, ws)
    torch.cuda.synchronize()
    assert e4b.workspace_error(ws) == e4b.E4B_KERNEL_ERR_NONE
    st = _oracle_stack(cfg)
    lg = logits.cpu().numpy()
    ids = routing.topk(lg, cfg.k)
    ref = backward.layer_backward(bf16_to_f64(x), lg.astype(np.float64), ids, st,
                                  workloads.bf16_bits_to_f32(dout_bits).astype(np.float64), True)
    for got, want, what in ((dx, ref[0], "dx"), (dl, ref[1], "dlogits"), (dA, ref[2], "dA"), (dB, ref[3], "dB")):
        fro, mx = rel_errors(got.cpu().numpy().astype(np.float64), want)
        print(f"[parity] fp4 backward {what}: rel_fro={fro:.2e} max={mx:.2e}")
        assert fro <= 1e-2 and mx <= 2e-2, what
