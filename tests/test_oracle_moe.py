"""Pins for the oracle's grouped GEMM and routed SwiGLU layer (CPU only).

The matrix code is tied to scalar closed forms: with constant-code stacks every
dequantised weight is one number, so each stage of the layer collapses to a
formula that is evaluated here by hand with ``math``.  The permuted form and
the brute-force per-token form are checked against each other, and the
planted-mistake controls show each check can fail.
"""
import math

import numpy as np
import pytest
from scipy.special import expit

from oracle import moe, nf4, routing

CB = [float(c) for c in nf4.NF4_CODEBOOK]


def _const_packed(E, n, codes_per_expert):
    """Packed bytes where expert e has every code equal to codes_per_expert[e]."""
    out = np.empty((E, n // 2), dtype=np.uint8)
    for e in range(E):
        c = int(codes_per_expert[e])
        out[e] = (c << 4) | c
    return out


def _const_gate_up(E, I, H, cg, cu):
    """gate rows all code cg[e], up rows all code cu[e]."""
    out = np.empty((E, 2 * I * H // 2), dtype=np.uint8)
    for e in range(E):
        half = I * H // 2
        out[e, :half] = (cg[e] << 4) | cg[e]
        out[e, half:] = (cu[e] << 4) | cu[e]
    return out


def test_silu_against_library_and_identities():
    z = np.linspace(-30, 30, 1001)
    assert np.allclose(moe.silu(z), z * expit(z), rtol=1e-14, atol=1e-300)
    assert moe.silu(np.array([0.0]))[0] == 0.0
    assert np.allclose(moe.silu(z) - moe.silu(-z), z, rtol=1e-13, atol=1e-13)
    assert moe.silu(np.array([-800.0]))[0] == 0.0     # no overflow warning escapes


def _closed_form_layer(x, ids, w, E, H, I, cg, cu, cd, ag, au, ad, lora=None):
    """Scalar form of the layer when every weight of a region is one value."""
    M, k = ids.shape
    out = np.zeros((M, H))
    for t in range(M):
        S = math.fsum(float(v) for v in x[t])
        for j in range(k):
            e = int(ids[t, j])
            g = CB[cg[e]] * ag[e] * S
            u = CB[cu[e]] * au[e] * S
            if lora is not None:
                scale, x0 = lora, float(x[t, 0])
                g += scale * x0
                u += scale * x0
            h = (g / (1.0 + math.exp(-g))) * u
            z = I * h * CB[cd[e]] * ad[e]
            out[t, :] += w[t, j] * z
    return out


def _closed_form_setup(E=4, H=128, I=64, M=6, k=2, seed=11):
    rng = np.random.default_rng(seed)
    cg = rng.integers(8, 16, size=E)            # positive gate values
    cu = rng.integers(0, 7, size=E)             # negative up values
    cd = rng.integers(0, 16, size=E)
    ag = rng.uniform(0.001, 0.01, size=E).astype(np.float32)
    au = rng.uniform(0.001, 0.01, size=E).astype(np.float32)
    ad = (np.arange(E, dtype=np.float32) + 1) / np.float32(8)
    gu_packed = _const_gate_up(E, I, H, cg, cu)
    gu_absmax = np.concatenate([np.stack([np.full(I * H // 64, ag[e], np.float32) for e in range(E)]),
                                np.stack([np.full(I * H // 64, au[e], np.float32) for e in range(E)])], axis=1)
    dn_packed = _const_packed(E, H * I, cd)
    dn_absmax = np.stack([np.full(H * I // 64, ad[e], np.float32) for e in range(E)])
    x = rng.standard_normal((M, H)).astype(np.float32)
    logits = rng.standard_normal((M, E)).astype(np.float32)
    ids, w, offs, perm, inv = routing.route_permute(logits, k)
    return dict(E=E, H=H, I=I, cg=cg, cu=cu, cd=cd, ag=ag.astype(np.float64),
                au=au.astype(np.float64), ad=ad.astype(np.float64),
                gu_packed=gu_packed, gu_absmax=gu_absmax, dn_packed=dn_packed, dn_absmax=dn_absmax,
                x=x, ids=ids, w=w, offs=offs, perm=perm, inv=inv)


def test_layer_closed_form_constant_codes():
    d = _closed_form_setup()
    st = moe.ExpertStack(d["gu_packed"], d["gu_absmax"], d["dn_packed"], d["dn_absmax"],
                         d["E"], d["H"], d["I"])
    want = _closed_form_layer(d["x"].astype(np.float64), d["ids"], d["w"], d["E"], d["H"], d["I"],
                              d["cg"], d["cu"], d["cd"], d["ag"], d["au"], d["ad"])
    got_tok = moe.moe_forward_per_token(d["x"], d["ids"], d["w"], st)
    got_grp = moe.moe_forward_grouped(d["x"], d["ids"], d["w"], d["offs"], d["perm"], d["inv"], st)
    scale = np.abs(want).max()
    assert scale > 0
    assert np.max(np.abs(got_tok - want)) <= 1e-12 * scale
    assert np.max(np.abs(got_grp - want)) <= 1e-12 * scale


def test_layer_closed_form_with_lora():
    d = _closed_form_setup(seed=12)
    E, H, I, r = d["E"], d["H"], d["I"], 8
    A = np.zeros((E, r, H))
    for rho in range(r):
        A[:, rho, rho] = 1.0                     # x . A^T = x[:r]
    B = np.zeros((E, 2 * I, r))
    B[:, :, 0] = 1.0                             # delta[n] = scale * x[0]
    st = moe.ExpertStack(d["gu_packed"], d["gu_absmax"], d["dn_packed"], d["dn_absmax"],
                         E, H, I, lora_A=A, lora_B=B, lora_scale=16 / 8)
    want = _closed_form_layer(d["x"].astype(np.float64), d["ids"], d["w"], E, H, I,
                              d["cg"], d["cu"], d["cd"], d["ag"], d["au"], d["ad"], lora=2.0)
    got = moe.moe_forward_grouped(d["x"], d["ids"], d["w"], d["offs"], d["perm"], d["inv"], st)
    got2 = moe.moe_forward_per_token(d["x"], d["ids"], d["w"], st)
    scale = np.abs(want).max()
    assert np.max(np.abs(got - want)) <= 1e-12 * scale
    assert np.max(np.abs(got2 - want)) <= 1e-12 * scale


def test_closed_form_positive_control_swapped_halves(monkeypatch):
    """Plant a gate/up swap in the oracle: the closed-form check must fail."""
    d = _closed_form_setup(seed=13)
    st = moe.ExpertStack(d["gu_packed"], d["gu_absmax"], d["dn_packed"], d["dn_absmax"],
                         d["E"], d["H"], d["I"])
    want = _closed_form_layer(d["x"].astype(np.float64), d["ids"], d["w"], d["E"], d["H"], d["I"],
                              d["cg"], d["cu"], d["cd"], d["ag"], d["au"], d["ad"])
    real = moe.ExpertStack.gate_up

    def swapped(self, e):
        g = real(self, e)
        return np.concatenate([g[self.I:], g[:self.I]])

    monkeypatch.setattr(moe.ExpertStack, "gate_up", swapped)
    got = moe.moe_forward_per_token(d["x"], d["ids"], d["w"], st)
    assert np.max(np.abs(got - want)) > 1e-3 * np.abs(want).max()


def _random_layer(E, H, I, M, k, seed, lora=False):
    rng = np.random.default_rng(seed)
    Wgu = (rng.standard_normal((E, 2 * I, H)) * 0.02).astype(np.float32)
    Wd = (rng.standard_normal((E, H, I)) * 0.02).astype(np.float32)
    gp, ga = nf4.quantize_stack(Wgu)
    dp, da = nf4.quantize_stack(Wd)
    la = lb = None
    if lora:
        la = rng.standard_normal((E, 8, H)) * 0.01
        lb = rng.standard_normal((E, 2 * I, 8)) * 0.01
    st = moe.ExpertStack(gp, ga, dp, da, E, H, I, la, lb, 2.0 if lora else 0.0)
    x = rng.standard_normal((M, H)).astype(np.float32)
    logits = rng.standard_normal((M, E)).astype(np.float32)
    return st, x, routing.route_permute(logits, k)


@pytest.mark.parametrize("E,H,I,M,k,lora", [(8, 256, 128, 64, 2, False), (8, 128, 64, 9, 3, True),
                                            (16, 64, 192, 5, 4, False)])
def test_grouped_equals_per_token(E, H, I, M, k, lora):
    st, x, (ids, w, offs, perm, inv) = _random_layer(E, H, I, M, k, seed=E + H + M, lora=lora)
    a = moe.moe_forward_per_token(x, ids, w, st)
    b = moe.moe_forward_grouped(x, ids, w, offs, perm, inv, st)
    assert np.linalg.norm(a - b) <= 1e-12 * np.linalg.norm(a)
    # sampled-token form agrees with the full one
    c = moe.moe_forward_per_token(x, ids, w, st, tokens=np.array([M - 1, 0]))
    assert np.array_equal(c, a[[M - 1, 0]])


def test_grouped_positive_control_corrupted_inverse():
    st, x, (ids, w, offs, perm, inv) = _random_layer(8, 64, 64, 12, 2, seed=21)
    a = moe.moe_forward_per_token(x, ids, w, st)
    bad = inv.copy()
    i = int(np.argmax(ids.reshape(-1) != ids.reshape(-1)[0]))
    bad[[0, i]] = bad[[i, 0]]
    b = moe.moe_forward_grouped(x, ids, w, offs, perm, bad, st)
    assert np.linalg.norm(a - b) > 1e-3 * np.linalg.norm(a)


def test_grouped_gemm_all_ones_row_sums():
    """Codes all 15 with absmax 1: W is all ones, so y is the row sum of A."""
    E, N, K, R = 3, 48, 128, 10
    rng = np.random.default_rng(5)
    A = rng.integers(-4, 5, size=(R, K)).astype(np.float64)
    packed = np.full((E, N * K // 2), 0xFF, dtype=np.uint8)
    absmax = np.ones((E, N * K // 64), dtype=np.float32)
    offs = np.array([0, 4, 4, R])
    ridx = rng.permutation(R)
    y = moe.grouped_nf4_gemm(A, ridx, offs, packed, absmax, N, K)
    want = A[ridx].sum(axis=1)[:, None] * np.ones((1, N))
    assert np.array_equal(y, want)


def test_grouped_gemm_single_group_is_plain_gemm():
    """E = 1 with identity rows: the dense product with the dequantised matrix."""
    rng = np.random.default_rng(6)
    N, K, R = 32, 192, 7
    W = (rng.standard_normal((1, N, K)) * 0.05).astype(np.float32)
    p, a = nf4.quantize_stack(W)
    A = rng.standard_normal((R, K))
    y = moe.grouped_nf4_gemm(A, None, np.array([0, R]), p, a, N, K)
    # dequantise by hand: code -> table value, times the block's absmax
    q = np.empty(N * K, dtype=np.int64)
    q[0::2] = p[0] >> 4
    q[1::2] = p[0] & 15
    Wd = np.array([CB[c] for c in q]).reshape(N, K) * np.repeat(a[0].astype(np.float64), 64).reshape(N, K)
    assert np.allclose(y, np.einsum("rk,nk->rn", A, Wd), rtol=1e-12, atol=1e-12)
