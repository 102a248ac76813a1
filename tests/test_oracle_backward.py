"""Pins of the backward oracle (oracle/backward.py): analytic gradients against
central finite differences of the forward (directional derivatives in float64),
closed forms of SiLU', the routing-weight gradient's invariants and linearity.
The finite differences share no arithmetic with the analytic derivation."""
import numpy as np
import pytest

from oracle import backward, moe, nf4, routing


def _layer(E=4, H=64, I=64, r=4, seed=0, lora=True):
    rng = np.random.default_rng(seed)
    gu = (rng.standard_normal((E, 2 * I, H)) * 0.05).astype(np.float32)
    dn = (rng.standard_normal((E, H, I)) * 0.05).astype(np.float32)
    gp, ga = nf4.quantize_stack(gu)
    dp, da = nf4.quantize_stack(dn)
    A = B = None
    if lora:
        A = rng.standard_normal((E, r, H)) * 0.1
        B = rng.standard_normal((E, 2 * I, r)) * 0.1
    return moe.ExpertStack(gp, ga, dp, da, E, H, I, A, B, lora_scale=16.0 / r if lora else 0.0)


def _with_lora(stack, A, B):
    return moe.ExpertStack(stack.gu_packed, stack.gu_absmax, stack.dn_packed, stack.dn_absmax,
                           stack.E, stack.H, stack.I, A, B, stack.lora_scale)


def _objective(x, logits, ids, stack, dout, renorm):
    w = backward.route_weights64(logits, ids, renorm)
    return float(np.sum(dout * backward.forward_with_weights(x, ids, w, stack)))


def _fd(f, eps=1e-5):
    return (f(eps) - f(-eps)) / (2 * eps)


def _case(M=3, E=4, H=64, k=2, seed=1, lora=True):
    stack = _layer(E=E, H=H, seed=seed, lora=lora)
    rng = np.random.default_rng(seed + 100)
    x = rng.standard_normal((M, H))
    logits = rng.standard_normal((M, E))
    ids = routing.topk(logits.astype(np.float32), k)
    dout = rng.standard_normal((M, H))
    return stack, x, logits, ids, dout


@pytest.mark.parametrize("renorm", [True, False])
@pytest.mark.parametrize("lora", [True, False])
def test_gradients_match_finite_differences(renorm, lora):
    stack, x, logits, ids, dout = _case(lora=lora)
    dx, dl, dA, dB = backward.layer_backward(x, logits, ids, stack, dout, renorm)
    rng = np.random.default_rng(7)
    for _ in range(3):
        v = rng.standard_normal(x.shape)
        fd = _fd(lambda e: _objective(x + e * v, logits, ids, stack, dout, renorm))
        assert fd == pytest.approx(np.sum(dx * v), rel=1e-6, abs=1e-9)
        v = rng.standard_normal(logits.shape)
        fd = _fd(lambda e: _objective(x, logits + e * v, ids, stack, dout, renorm))
        assert fd == pytest.approx(np.sum(dl * v), rel=1e-6, abs=1e-9)
        if lora:
            vA = rng.standard_normal(stack.lora_A.shape)
            fd = _fd(lambda e: _objective(x, logits, ids, _with_lora(stack, stack.lora_A + e * vA, stack.lora_B),
                                          dout, renorm))
            assert fd == pytest.approx(np.sum(dA * vA), rel=1e-6, abs=1e-9)
            vB = rng.standard_normal(stack.lora_B.shape)
            fd = _fd(lambda e: _objective(x, logits, ids, _with_lora(stack, stack.lora_A, stack.lora_B + e * vB),
                                          dout, renorm))
            assert fd == pytest.approx(np.sum(dB * vB), rel=1e-6, abs=1e-9)
    if not lora:
        assert dA is None and dB is None


def test_finite_difference_check_detects_a_planted_error():
    # Positive control: a 1e-3 relative error in dx is caught by the same check.
    stack, x, logits, ids, dout = _case()
    dx, _, _, _ = backward.layer_backward(x, logits, ids, stack, dout)
    v = np.random.default_rng(3).standard_normal(x.shape)
    fd = _fd(lambda e: _objective(x + e * v, logits, ids, stack, dout, True))
    assert fd != pytest.approx(np.sum(dx * 1.001 * v), rel=1e-6, abs=1e-9)


def test_forward_helpers_agree_with_the_forward_oracle():
    stack, x, logits, ids, _ = _case()
    l32 = logits.astype(np.float32)
    w = routing.route_weights(l32, ids, True)
    assert np.allclose(backward.route_weights64(l32, ids, True), w, rtol=0, atol=1e-15)
    assert np.allclose(backward.route_weights64(l32, ids, False), routing.route_weights(l32, ids, False),
                       rtol=0, atol=1e-15)
    assert np.allclose(backward.forward_with_weights(x, ids, w, stack),
                       moe.moe_forward_per_token(x, ids, w, stack), rtol=0, atol=1e-12)


def test_silu_grad_closed_forms():
    assert backward.silu_grad(np.array([0.0]))[0] == 0.5
    z = np.linspace(-8, 8, 33)
    fd = (moe.silu(z + 1e-6) - moe.silu(z - 1e-6)) / 2e-6
    assert np.allclose(backward.silu_grad(z), fd, rtol=0, atol=1e-8)
    # large |z|: SiLU' -> 1 for z -> +inf and -> 0 for z -> -inf
    assert backward.silu_grad(np.array([60.0]))[0] == pytest.approx(1.0)
    assert abs(backward.silu_grad(np.array([-60.0]))[0]) < 1e-20


def test_routing_gradient_invariants():
    stack, x, logits, ids, dout = _case(M=4)
    _, dl, _, _ = backward.layer_backward(x, logits, ids, stack, dout, True)
    # renormalised softmax: shift-invariant per token -> the gradient sums to zero,
    # and unselected experts receive nothing
    assert np.allclose(dl.sum(axis=1), 0.0, atol=1e-12)
    mask = np.ones_like(dl, dtype=bool)
    np.put_along_axis(mask, ids.astype(np.int64), False, axis=1)
    assert np.all(dl[mask] == 0.0)
    _, dl_full, _, _ = backward.layer_backward(x, logits, ids, stack, dout, False)
    assert np.allclose(dl_full.sum(axis=1), 0.0, atol=1e-12)


def test_gradients_are_linear_in_dout():
    stack, x, logits, ids, d1 = _case()
    d2 = np.random.default_rng(11).standard_normal(d1.shape)
    g1 = backward.layer_backward(x, logits, ids, stack, d1)
    g2 = backward.layer_backward(x, logits, ids, stack, d2)
    g = backward.layer_backward(x, logits, ids, stack, 2.0 * d1 - 3.0 * d2)
    for a, b, c in zip(g1, g2, g):
        assert np.allclose(c, 2.0 * a - 3.0 * b, rtol=1e-12, atol=1e-12)


def test_lora_gradient_closed_forms():
    # B = 0: the delta and dA vanish; dB is the outer product s * da^T (x A^T).
    stack, x, logits, ids, dout = _case()
    zero_B = _with_lora(stack, stack.lora_A, np.zeros_like(stack.lora_B))
    _, _, dA, dB = backward.layer_backward(x, logits, ids, zero_B, dout)
    assert np.all(dA == 0.0)
    assert np.any(dB != 0.0)
    # A = 0: xa = 0, so dB vanishes while dA does not.
    zero_A = _with_lora(stack, np.zeros_like(stack.lora_A), stack.lora_B)
    _, _, dA0, dB0 = backward.layer_backward(x, logits, ids, zero_A, dout)
    assert np.all(dB0 == 0.0)
    assert np.any(dA0 != 0.0)


def _gemm_case(E=3, N=64, K=128, counts=(5, 0, 7), r=4, seed=5):
    rng = np.random.default_rng(seed)
    W = (rng.standard_normal((E, N, K)) * 0.05).astype(np.float32)
    packed, absmax = nf4.quantize_stack(W)
    offsets = np.concatenate([[0], np.cumsum(counts)]).astype(np.int64)
    rows = int(offsets[-1])
    la = rng.standard_normal((E, r, K)) * 0.1
    lb = rng.standard_normal((E, N, r)) * 0.1
    return packed, absmax, offsets, rows, la, lb, rng


@pytest.mark.parametrize("lora", [False, True])
def test_grouped_dgrad_is_the_adjoint_of_the_grouped_gemm(lora):
    """<dY, gemm(A)> = <dgrad(dY), A> for every A and dY: the dgrad oracle is
    pinned to the (separately pinned) forward GEMM oracle, so a transposed
    operand or a missing LoRA term fails here."""
    E, N, K = 3, 64, 128
    packed, absmax, offsets, rows, la, lb, rng = _gemm_case(E, N, K)
    A = rng.standard_normal((rows, K))
    dY = rng.standard_normal((rows, N))
    kw = dict(lora_A=la, lora_B=lb, lora_scale=2.5) if lora else {}
    y = moe.grouped_nf4_gemm(A, None, offsets, packed, absmax, N, K, **kw)
    d = backward.grouped_nf4_gemm_dgrad(dY, None, offsets, packed, absmax, N, K, **kw)
    assert d.shape == (rows, K)
    assert np.sum(dY * y) == pytest.approx(np.sum(d * A), rel=1e-12)


def test_grouped_dgrad_brute_force_and_row_index():
    """Element by element from the codes, the codebook and absmax (no
    dequantised matrix), and the row index gathers dY rows."""
    E, N, K = 3, 64, 128
    packed, absmax, offsets, rows, _, _, rng = _gemm_case(E, N, K)
    dY = rng.standard_normal((rows + 4, N))
    idx = rng.permutation(rows + 4)[:rows]
    d = backward.grouped_nf4_gemm_dgrad(dY, idx, offsets, packed, absmax, N, K)
    cb = nf4.codebook_f64()
    for p in (0, 4, rows - 1):
        e = int(np.searchsorted(offsets, p, side="right") - 1)
        q = nf4.unpack_codes(packed[e])
        for kk in (0, 63, 64, K - 1):
            ref = sum(dY[idx[p], n] * cb[q[n * K + kk]] * float(absmax[e][(n * K + kk) // 64]) for n in range(N))
            assert d[p, kk] == pytest.approx(ref, rel=1e-12, abs=1e-12)
    assert np.array_equal(d, backward.grouped_nf4_gemm_dgrad(dY[idx], None, offsets, packed, absmax, N, K))


def test_adjoint_check_detects_a_transposed_operand():
    # Positive control: the same check fails for dY . W^T on a square stack.
    E, N, K = 2, 64, 64
    packed, absmax, offsets, rows, _, _, rng = _gemm_case(E, N, K, counts=(4, 6))
    A = rng.standard_normal((rows, K))
    dY = rng.standard_normal((rows, N))
    y = moe.grouped_nf4_gemm(A, None, offsets, packed, absmax, N, K)
    wrong = np.zeros((rows, K))
    for e in range(E):
        W = nf4.dequantize_expert(packed[e], absmax[e], (N, K))
        wrong[offsets[e]:offsets[e + 1]] = dY[offsets[e]:offsets[e + 1]] @ W.T
    assert np.sum(dY * y) != pytest.approx(np.sum(wrong * A), rel=1e-6)


@pytest.mark.parametrize("renorm", [True, False])
@pytest.mark.parametrize("lora", [True, False])
def test_grouped_backward_equals_the_per_token_backward(renorm, lora):
    """The permuted grouped form (two grouped dgrad products around the SwiGLU
    derivative, sums through the inverse permutation) gives the gradients of
    the finite-difference-pinned per-token backward."""
    stack, x, logits, ids, dout = _case(M=6, lora=lora)
    a = backward.layer_backward(x, logits, ids, stack, dout, renorm)
    b = backward.layer_backward_grouped(x, logits, ids, stack, dout, renorm)
    for u, v in zip(a, b):
        if u is None:
            assert v is None
            continue
        assert np.allclose(u, v, rtol=0, atol=1e-12 * max(1.0, np.abs(u).max()))


def test_grouped_lora_grads_brute_force_and_empty_groups():
    """Element by element over the rows of each group; an expert with no rows
    gets zero gradients; the row index gathers the input rows."""
    rng = np.random.default_rng(9)
    E, N, K, r, s = 3, 6, 5, 2, 1.5
    offsets = np.array([0, 4, 4, 7])
    x = rng.standard_normal((9, K))
    idx = np.array([8, 0, 3, 3, 1, 5, 2])
    da = rng.standard_normal((7, N))
    A = rng.standard_normal((E, r, K))
    B = rng.standard_normal((E, N, r))
    dA, dB = backward.grouped_lora_grads(x, idx, offsets, da, A, B, s)
    assert np.all(dA[1] == 0) and np.all(dB[1] == 0)
    for e, (lo, hi) in enumerate([(0, 4), (4, 4), (4, 7)]):
        for i in range(N):
            for rho in range(r):
                ref = s * sum(da[p, i] * sum(x[idx[p], kk] * A[e, rho, kk] for kk in range(K)) for p in range(lo, hi))
                assert dB[e, i, rho] == pytest.approx(ref, rel=1e-12, abs=1e-12)
        for rho in range(r):
            for kk in range(K):
                ref = s * sum(sum(da[p, i] * B[e, i, rho] for i in range(N)) * x[idx[p], kk] for p in range(lo, hi))
                assert dA[e, rho, kk] == pytest.approx(ref, rel=1e-12, abs=1e-12)
