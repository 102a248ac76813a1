"""The layer forward on the GPU vs the float64 oracle, all five layer shapes.

Small shapes compare every output; the full-size workloads compare sampled
tokens, for which the oracle re-quantises only the experts they touch (its own
quantiser, never the GPU's bytes) and the GPU's packed bytes of those experts
are checked bit for bit on the way.
"""
import numpy as np
import pytest
import torch

from oracle import moe, nf4, routing
from quantized_moe_expert_nf4_b200 import e4b, synthetic, workloads
from gpu_util import assert_close_layer, bf16_to_f64, require_gpu

pytestmark = pytest.mark.gpu


def _forward(layer, x, logits, path=e4b.E4B_PATH_AUTO, renormalize=True):
    cfg = layer.cfg
    M = x.shape[0]
    out = torch.full((M, cfg.H), float("nan"), dtype=torch.bfloat16, device="cuda")
    ws = e4b.workspace(e4b.e4b_moe_expert_forward_workspace_size(M, layer.stack, cfg.k))
    e4b.e4b_moe_expert_forward(x, logits, cfg.k, renormalize, layer.stack, out, ws, path=path)
    torch.cuda.synchronize()
    p = e4b.last_path()
    assert e4b.workspace_error(ws) == e4b.E4B_KERNEL_ERR_NONE, "a kernel gave up a bounded wait"
    return out, p


def _oracle_tokens(cfg, x, logits, tokens, check_gpu_layer=None, renormalize=True):
    """Oracle output rows for `tokens`, quantising only the experts they use."""
    lg = logits.cpu().numpy()
    ids = routing.topk(lg[tokens], cfg.k)
    w = routing.route_weights(lg[tokens], ids, renormalize)
    need = sorted(set(ids.reshape(-1).tolist()))
    E, H, I = cfg.E, cfg.H, cfg.I
    gp = np.zeros((E, I * H), np.uint8)
    ga = np.zeros((E, 2 * I * H // 64), np.float32)
    dp = np.zeros((E, H * I // 2), np.uint8)
    da = np.zeros((E, H * I // 64), np.float32)
    for e in need:
        gp[e], ga[e] = nf4.quantize_expert(workloads.gate_up_expert(cfg, e))
        dp[e], da[e] = nf4.quantize_expert(workloads.down_expert(cfg, e))
        if check_gpu_layer is not None:
            L = check_gpu_layer
            assert np.array_equal(L.gu_packed[e].cpu().numpy(), gp[e])
            assert np.array_equal(L.dn_absmax[e].cpu().numpy(), da[e])
    la = lb = None
    if cfg.lora_r:
        la = workloads.bf16_bits_to_f32(workloads.lora_A(cfg)).astype(np.float64)
        lb = workloads.bf16_bits_to_f32(workloads.lora_B(cfg)).astype(np.float64)
    st = moe.ExpertStack(gp, ga, dp, da, E, H, I, la, lb, workloads.lora_scale(cfg))
    xs = bf16_to_f64(x[torch.as_tensor(tokens, device=x.device)])
    return moe.moe_forward_per_token(xs, ids, w, st)


SMALL = [
    ("tiny", workloads.CONFIGS["tiny"], 64),
    ("ragged", workloads.small_config("ragged", E=12, H=192, I=320, k=3), 37),
    ("lora", workloads.small_config("lora", E=6, H=128, I=192, k=2, lora_r=8, lora_alpha=16.0), 50),
    ("zipf", workloads.small_config("zipf", E=16, H=256, I=128, k=4, routing="zipf"), 300),
    ("dir", workloads.small_config("dir", E=8, H=320, I=192, k=2, routing="dirichlet"), 129),
]


@pytest.mark.parametrize("name,cfg,M", SMALL, ids=[s[0] for s in SMALL])
@pytest.mark.parametrize("path", [e4b.E4B_PATH_GROUPED])
def test_forward_small_all_tokens(name, cfg, M, path):
    require_gpu()
    layer = synthetic.make_device_layer(cfg)
    x, logits = synthetic.inputs(cfg, M)
    out, p = _forward(layer, x, logits, path)
    ref = _oracle_tokens(cfg, x, logits, np.arange(M), check_gpu_layer=layer)
    assert_close_layer(bf16_to_f64(out), ref, f"{name} M={M} {p}")
    # deterministic: a second call gives identical bits
    out2, _ = _forward(layer, x, logits, path)
    assert torch.equal(out.view(torch.int16), out2.view(torch.int16))


FULL = [("olmoe", 2048), ("qwen3", 4096), ("qwen3_lora", 4096), ("gptoss", 8192), ("olmoe", 1), ("olmoe", 4),
        ("olmoe", 8), ("gptoss", 1), ("qwen3_lora", 3)]


@pytest.mark.parametrize("name,M", FULL)
def test_forward_full_size_sampled_tokens(name, M):
    require_gpu()
    cfg = workloads.CONFIGS[name]
    layer = synthetic.make_device_layer(cfg)
    x, logits = synthetic.inputs(cfg, M)
    out, p = _forward(layer, x, logits)
    tokens = np.unique(np.array([0, M - 1, M // 2, M // 3]))[:4]
    ref = _oracle_tokens(cfg, x, logits, tokens, check_gpu_layer=layer)
    got = bf16_to_f64(out[torch.as_tensor(tokens, device="cuda")])
    assert_close_layer(got, ref, f"{name} M={M} {p} tokens {tokens.tolist()}")
    assert torch.isfinite(out.float()).all()


DECODE = [
    ("tiny1", workloads.CONFIGS["tiny"], 1),
    ("tiny8", workloads.CONFIGS["tiny"], 8),
    ("ragged5", workloads.small_config("ragged", E=12, H=192, I=320, k=3), 5),
    ("lora3", workloads.small_config("lora", E=6, H=128, I=192, k=2, lora_r=8, lora_alpha=16.0), 3),
    ("wide2", workloads.small_config("wide", E=40, H=448, I=128, k=6, routing="zipf"), 2),
    ("k32", workloads.small_config("k32", E=33, H=128, I=64, k=32), 7),
    ("odd_kblocks", workloads.small_config("oddkb", E=8, H=2880, I=704, k=2), 8),
]


@pytest.mark.parametrize("name,cfg,M", DECODE, ids=[d[0] for d in DECODE])
def test_forward_decode_path_all_tokens(name, cfg, M):
    require_gpu()
    layer = synthetic.make_device_layer(cfg)
    x, logits = synthetic.inputs(cfg, M)
    out, p = _forward(layer, x, logits, e4b.E4B_PATH_DECODE)
    assert p == "forward.decode" and e4b.last_launches() == 2
    ref = _oracle_tokens(cfg, x, logits, np.arange(M))
    assert_close_layer(bf16_to_f64(out), ref, f"{name} M={M} {p}")
    out2, _ = _forward(layer, x, logits, e4b.E4B_PATH_DECODE)
    assert torch.equal(out.view(torch.int16), out2.view(torch.int16))
    outg, _ = _forward(layer, x, logits, e4b.E4B_PATH_GROUPED)
    assert_close_layer(bf16_to_f64(outg), ref, f"{name} M={M} grouped")


def test_forward_decode_rejects_large_batches():
    require_gpu()
    cfg = workloads.CONFIGS["tiny"]
    layer = synthetic.make_device_layer(cfg)
    x, logits = synthetic.inputs(cfg, 9)
    with pytest.raises(e4b.E4BError, match="decode path"):
        _forward(layer, x, logits, e4b.E4B_PATH_DECODE)


def test_forward_positive_control_wrong_expert_bytes():
    require_gpu()
    cfg = workloads.CONFIGS["tiny"]
    layer = synthetic.make_device_layer(cfg)
    x, logits = synthetic.inputs(cfg, 16)
    ref = _oracle_tokens(cfg, x, logits, np.arange(16))
    layer.gu_packed[:, :1024] ^= 0x11     # corrupt the gate rows of every expert
    out, _ = _forward(layer, x, logits, e4b.E4B_PATH_GROUPED)
    from gpu_util import rel_errors
    assert rel_errors(bf16_to_f64(out), ref)[0] > 1e-2


def test_forward_errors_and_empty():
    require_gpu()
    cfg = workloads.CONFIGS["tiny"]
    layer = synthetic.make_device_layer(cfg)
    x, logits = synthetic.inputs(cfg, 4)
    out = torch.empty((4, cfg.H), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(e4b.E4BError, match="workspace"):
        e4b.e4b_moe_expert_forward(x, logits, cfg.k, True, layer.stack, out, None)
    x0 = x[:0]
    e4b.e4b_moe_expert_forward(x0, logits[:0], cfg.k, True, layer.stack, out[:0], None)
    assert e4b.last_path() == "forward.empty"


@pytest.mark.parametrize("path", [e4b.E4B_PATH_DECODE, e4b.E4B_PATH_GROUPED])
def test_forward_without_renormalisation(path):
    """renormalize = 0: each selected expert keeps its weight from the softmax
    over all E logits (the k weights no longer sum to 1)."""
    require_gpu()
    cfg = workloads.small_config("fullsm", E=12, H=192, I=320, k=3)
    M = 5 if path == e4b.E4B_PATH_DECODE else 40
    layer = synthetic.make_device_layer(cfg)
    x, logits = synthetic.inputs(cfg, M)
    out, p = _forward(layer, x, logits, path, renormalize=False)
    ref = _oracle_tokens(cfg, x, logits, np.arange(M), renormalize=False)
    assert_close_layer(bf16_to_f64(out), ref, f"renormalize=0 M={M} {p}")
    ref_renorm = _oracle_tokens(cfg, x, logits, np.arange(M))
    from gpu_util import rel_errors
    assert rel_errors(bf16_to_f64(out), ref_renorm)[0] > 1e-2   # the flag changes the result


@pytest.mark.parametrize("E,k,M,path", [(8, 1, 6, e4b.E4B_PATH_DECODE), (8, 1, 700, e4b.E4B_PATH_GROUPED),
                                        (4, 4, 300, e4b.E4B_PATH_GROUPED), (4, 4, 7, e4b.E4B_PATH_DECODE)])
def test_forward_degenerate_routing(E, k, M, path):
    """One expert takes every token (k = 1: one group holds all rows, the
    others are empty), or every token takes every expert (k = E)."""
    require_gpu()
    cfg = workloads.small_config(f"degen{E}_{k}", E=E, H=256, I=192, k=k)
    layer = synthetic.make_device_layer(cfg)
    x, logits = synthetic.inputs(cfg, M)
    if k == 1:
        logits[:, 5] += 30.0
    out, p = _forward(layer, x, logits, path)
    ref = _oracle_tokens(cfg, x, logits, np.arange(M))
    assert_close_layer(bf16_to_f64(out), ref, f"E={E} k={k} M={M} {p}")


@pytest.mark.parametrize("M", [3, 300])
def test_forward_replays_bit_identically_from_a_cuda_graph(M):
    """The header promises graph-capturable calls (no host sync, no device data
    read back): a captured forward replays to the same bits as an eager call,
    on the decode path (M = 3) and the grouped tensor-core path (M = 300)."""
    require_gpu()
    cfg = workloads.CONFIGS["tiny"]
    layer = synthetic.make_device_layer(cfg)
    x, logits = synthetic.inputs(cfg, M)
    eager, _ = _forward(layer, x, logits)
    out = torch.empty_like(eager)
    ws = e4b.workspace(e4b.e4b_moe_expert_forward_workspace_size(M, layer.stack, cfg.k))
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):   # warm the library's per-device state outside the capture
        e4b.e4b_moe_expert_forward(x, logits, cfg.k, True, layer.stack, out, ws)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        e4b.e4b_moe_expert_forward(x, logits, cfg.k, True, layer.stack, out, ws)
    out.fill_(float("nan"))
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(out.view(torch.int16), eager.view(torch.int16))


LIMITS = [
    # the largest hidden size the decode kernels take (two spans of 128 k per warp)
    ("h4096", workloads.small_config("h4096", E=8, H=4096, I=128, k=2), 8),
    # the largest expert count they take, every token routed to 8 of 512
    ("e512", workloads.small_config("e512", E=512, H=128, I=64, k=8, routing="zipf"), 8),
]


@pytest.mark.parametrize("name,cfg,M", LIMITS, ids=[c[0] for c in LIMITS])
def test_forward_decode_at_its_size_limits(name, cfg, M):
    require_gpu()
    layer = synthetic.make_device_layer(cfg)
    x, logits = synthetic.inputs(cfg, M)
    out, p = _forward(layer, x, logits, e4b.E4B_PATH_DECODE)
    assert p == "forward.decode"
    ref = _oracle_tokens(cfg, x, logits, np.arange(M))
    assert_close_layer(bf16_to_f64(out), ref, f"{name} M={M} {p}")


@pytest.mark.parametrize("name,cfg,why", [
    ("h4160", workloads.small_config("h4160", E=4, H=4160, I=64, k=2), "H <= 4096"),
    ("e513", workloads.small_config("e513", E=513, H=64, I=64, k=2), "at most 512 experts"),
], ids=["h4160", "e513"])
def test_forward_past_the_decode_limits_runs_grouped(name, cfg, why):
    """One step past a decode limit: a forced decode call is refused with the
    limit named; the automatic choice runs the grouped path and matches the oracle."""
    require_gpu()
    layer = synthetic.make_device_layer(cfg)
    x, logits = synthetic.inputs(cfg, 4)
    with pytest.raises(e4b.E4BError, match=why):
        _forward(layer, x, logits, e4b.E4B_PATH_DECODE)
    out, p = _forward(layer, x, logits)
    assert p == "forward.grouped"
    assert_close_layer(bf16_to_f64(out), _oracle_tokens(cfg, x, logits, np.arange(4)), f"{name} {p}")
