"""Pins of the FP4 storage oracle (oracle/fp4.py) against the e2m1 format's
own definition, brute force, closed forms and the pages' fidelity ordering."""
from fractions import Fraction

import numpy as np
import pytest

from oracle import fp4, moe, nf4, routing

# The e2m1 element magnitudes as the OCP microscaling format defines them
# (codes 0-7; codes 8-15 are their negatives).
E2M1_MAGNITUDES = [Fraction(0), Fraction(1, 2), Fraction(1), Fraction(3, 2), Fraction(2), Fraction(3), Fraction(4),
                   Fraction(6)]


def _nearest_f32(r: Fraction) -> float:
    c = np.float32(float(r))
    cands = [np.nextafter(c, np.float32(-np.inf)), c, np.nextafter(c, np.float32(np.inf))]
    return float(min(cands, key=lambda x: abs(Fraction(float(x)) - r)))


def test_codebook_is_e2m1_over_six_in_float32():
    cb = fp4.codebook_f64()
    for c in range(16):
        r = E2M1_MAGNITUDES[c & 7] / 6 * (-1 if c & 8 else 1)
        assert cb[c] == _nearest_f32(r), c
    assert cb[7] == 1.0 and cb[15] == -1.0
    assert cb[0] == 0.0 and cb[8] == 0.0
    assert np.all(np.diff(cb[:8]) > 0)


def _brute_code_values(s):
    """Nearest entry by exhaustive search in exact rationals, ties to the smaller value."""
    cb = fp4.codebook_f64()
    out = []
    for v in np.asarray(s, dtype=np.float32):
        fv = Fraction(float(v))
        best = None
        for e in sorted(set(cb.tolist())):
            d = abs(Fraction(e) - fv)
            if best is None or d < best[0]:  # strict: a tie keeps the smaller value
                best = (d, e)
        out.append(best[1])
    return np.array(out)


def test_code_choice_matches_brute_force_including_midpoints():
    rng = np.random.default_rng(5)
    s = rng.uniform(-1, 1, 4000).astype(np.float32)
    mids = fp4.midpoints()
    near = []
    for m in mids:
        f = np.float32(m)
        near += [f, np.nextafter(f, np.float32(-2)), np.nextafter(f, np.float32(2))]
    s = np.concatenate([s, np.array(near, dtype=np.float32), np.float32([0.0, -0.0, 1.0, -1.0])])
    q = fp4.code_of_scaled(s)
    assert np.array_equal(fp4.codebook_f64()[q], _brute_code_values(s))
    assert not np.any(q == 8), "code 8 (-0) is never written"
    assert np.all(q[s == 0] == 0)


def test_exact_midpoints_take_the_smaller_value():
    # Of the decision points only the two around zero are float32 values:
    # +-fl32(1/12)/2.  They take the smaller neighbour: 0 (code 0) and -1/12
    # (code 9).  0.75 lies below the decision point between 2/3 and 1.
    h = np.float32(fp4.codebook_f64()[1] / 2)
    assert np.float64(h) * 2 == fp4.codebook_f64()[1]
    q = fp4.code_of_scaled(np.float32([h, -h, 0.75]))
    assert list(q) == [0, 9, 6]


def test_quantised_block_by_hand():
    a = np.float32(3.0)
    vals = np.array([1, -1, 0, 0.5, 1 / 3, -0.25, 1 / 12, -2 / 3] * 8, dtype=np.float64) * 3.0
    w = vals.astype(np.float32)
    packed, absmax = fp4.quantize_expert(w)
    assert absmax[0] == a
    # codes 7, 15, 0, 5, 4, 11, 1, 14 -> bytes 0x7F, 0x05, 0x4B, 0x1E (high nibble first)
    assert list(packed[:4]) == [0x7F, 0x05, 0x4B, 0x1E]


def test_block_invariants_and_round_trip_bound():
    rng = np.random.default_rng(6)
    W = (rng.standard_normal((3, 16, 128)) * 0.02).astype(np.float32)
    W[1, 3, :64] = 0.0  # one all-zero block
    packed, absmax = fp4.quantize_stack(W)
    assert absmax[1, 3 * 2] == 0.0
    q = nf4.unpack_codes(packed).reshape(3, -1, 64)
    assert np.all(q[1, 3 * 2] == 0)
    live = absmax > 0
    assert np.all(np.any((q == 7) | (q == 15), axis=2)[live]), "every block holds its absmax code"
    levels = np.unique(fp4.codebook_f64())
    for e in range(3):
        R = fp4.dequantize_expert(packed[e], absmax[e], (16, 128))
        a = np.repeat(absmax[e].astype(np.float64), 64).reshape(16, 128)
        s = W[e].astype(np.float64) / np.where(a == 0, 1, a)
        hi = np.searchsorted(levels, s, side="left").clip(1, levels.size - 1)
        gap = levels[hi] - levels[hi - 1]
        assert np.all(np.abs(W[e] - R) <= a * gap / 2 + a * 2.0 ** -24)
        amax_pos = np.abs(W[e]) == a
        assert np.all(np.abs(R[amax_pos]) == a[amax_pos])


def test_fidelity_ordering_nf4_below_fp4():
    """The pages pin nf4 reconstruction error below fp4's on the same stack."""
    rng = np.random.default_rng(7)
    W = (rng.standard_normal((4, 64, 256)) * 0.02).astype(np.float32)
    err = {}
    for name, mod in (("nf4", nf4), ("fp4", fp4)):
        p, a = mod.quantize_stack(W)
        R = np.stack([mod.dequantize_expert(p[e], a[e], (64, 256)) for e in range(4)])
        err[name] = np.linalg.norm(R - W) / np.linalg.norm(W)
    assert 0 < err["nf4"] < err["fp4"] < 0.2, err


def test_grouped_gemm_and_layer_with_fp4_storage():
    rng = np.random.default_rng(8)
    E, N, K = 3, 8, 128
    W = (rng.standard_normal((E, N, K)) * 0.02).astype(np.float32)
    packed, absmax = fp4.quantize_stack(W)
    A = rng.standard_normal((5, K))
    offsets = np.array([0, 2, 2, 5])
    got = moe.grouped_nf4_gemm(A, None, offsets, packed, absmax, N, K, quant="fp4")
    q = nf4.unpack_codes(packed).reshape(E, N, K)
    cb = fp4.codebook_f64()
    for p in range(5):
        e = int(np.searchsorted(offsets, p, side="right") - 1)
        for n in range(N):
            want = sum(A[p, kk] * cb[q[e, n, kk]] * float(absmax[e, (n * K + kk) // 64]) for kk in range(K))
            assert abs(got[p, n] - want) <= 1e-12 * max(1.0, abs(want))
    # the whole layer: per-token brute force == the permuted grouped form
    H, I, M, k = 128, 64, 6, 2
    gu = (rng.standard_normal((E, 2 * I, H)) * 0.02).astype(np.float32)
    dn = (rng.standard_normal((E, H, I)) * 0.02).astype(np.float32)
    st = moe.ExpertStack(*fp4.quantize_stack(gu), *fp4.quantize_stack(dn), E, H, I, quant="fp4")
    x = rng.standard_normal((M, H))
    ids, w, off, perm, inv = routing.route_permute(rng.standard_normal((M, E)), k)
    a = moe.moe_forward_per_token(x, ids, w, st)
    b = moe.moe_forward_grouped(x, ids, w, off, perm, inv, st)
    assert np.abs(a - b).max() <= 1e-12 * np.abs(a).max()
    # and it differs from reading the same bytes as NF4
    st_nf4 = moe.ExpertStack(st.gu_packed, st.gu_absmax, st.dn_packed, st.dn_absmax, E, H, I)
    assert np.abs(moe.moe_forward_per_token(x, ids, w, st_nf4) - a).max() > 1e-3 * np.abs(a).max()


def test_unknown_storage_type_is_refused():
    with pytest.raises(ValueError):
        moe.ExpertStack(np.zeros((1, 64), np.uint8), np.zeros((1, 2), np.float32), np.zeros((1, 64), np.uint8),
                        np.zeros((1, 2), np.float32), 1, 64, 1, quant="int4")
