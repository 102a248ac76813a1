"""Pins for the oracle's NF4 codebook and stack quantiser (CPU only).

Each check ties the oracle to something other than itself: the published
codebook (golden file), its construction from normal quantiles, a brute-force
nearest-code search in extended precision, a hand-worked block, and the
round-trip bound and endpoint invariants of blockwise absmax quantisation.
"""
import os

import numpy as np
import pytest

from oracle import nf4

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _read_golden(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                rows.append(line.split())
    return rows


def test_codebook_matches_published_table():
    table = np.array([float(r[0]) for r in _read_golden("nf4_codebook.txt")], dtype=np.float32)
    assert table.shape == (16,)
    assert np.array_equal(table.view(np.uint32), nf4.NF4_CODEBOOK.view(np.uint32))


def test_codebook_matches_quantile_construction():
    d = nf4.derived_codebook()
    assert np.max(np.abs(d - nf4.codebook_f64())) < 2e-7


def test_codebook_endpoints_and_order():
    cb = nf4.NF4_CODEBOOK
    assert cb[0] == np.float32(-1.0) and cb[7] == np.float32(0.0) and cb[15] == np.float32(1.0)
    assert np.all(np.diff(cb.astype(np.float64)) > 0)
    # exactly representable: the float32 values round-trip through float64
    assert np.array_equal(cb.astype(np.float64).astype(np.float32), cb)


def _brute_force_code(s32):
    """Argmin over the 16 entries of |s - c| in long double, first index on ties."""
    cb = nf4.NF4_CODEBOOK.astype(np.longdouble)
    s = np.asarray(s32, dtype=np.float32).astype(np.longdouble)
    d = np.abs(s[:, None] - cb[None, :])
    return np.argmin(d, axis=1).astype(np.uint8)     # argmin keeps the first minimum


def test_code_selection_brute_force_random():
    rng = np.random.default_rng(1)
    s = np.concatenate([
        rng.uniform(-1, 1, 400_000).astype(np.float32),
        rng.standard_normal(200_000).astype(np.float32).clip(-1, 1),
    ])
    assert np.array_equal(nf4.code_of_scaled(s), _brute_force_code(s))


def test_code_selection_at_decision_points_and_neighbours():
    cb = nf4.codebook_f64()
    pts = []
    for c in range(15):
        m = (cb[c] + cb[c + 1]) / 2
        m32 = np.float32(m)
        for v in (m32, np.nextafter(m32, np.float32(-2)), np.nextafter(m32, np.float32(2))):
            pts.append(v)
        pts.extend([np.float32(cb[c]), np.float32(cb[c + 1])])
    s = np.array(pts, dtype=np.float32)
    assert np.array_equal(nf4.code_of_scaled(s), _brute_force_code(s))
    # the two decision points that are exact float32 values resolve to the lower code
    assert nf4.code_of_scaled(np.array([np.float32(cb[8] / 2)]))[0] == 7
    assert nf4.code_of_scaled(np.array([np.float32(cb[6] / 2)]))[0] == 6


def test_hand_worked_block():
    rows = _read_golden("nf4_block_example.txt")
    w = np.zeros(64, dtype=np.float32)
    want = np.full(64, 7, dtype=np.uint8)
    for i, (wv, code) in enumerate(rows):
        w[i] = np.float32(float(wv))
        want[i] = int(code)
    packed, absmax = nf4.quantize_expert(w)
    assert absmax.tolist() == [2.0]
    assert np.array_equal(nf4.unpack_codes(packed), want)
    # first byte: codes 0 (high nibble) and 15 (low nibble)
    assert packed[0] == 0x0F
    assert packed[1] == (7 << 4) | 12


def test_pack_unpack_identity_and_nibble_order():
    rng = np.random.default_rng(2)
    q = rng.integers(0, 16, size=(3, 128), dtype=np.uint8)
    p = nf4.pack_codes(q)
    assert np.array_equal(nf4.unpack_codes(p), q)
    assert p[0, 0] == (q[0, 0] << 4) | q[0, 1]


def _random_stack(E, N, K, seed=3, scale=0.02):
    rng = np.random.default_rng(seed)
    return (rng.standard_normal((E, N, K), dtype=np.float32) * np.float32(scale))


def test_round_trip_bound_and_endpoints():
    W = _random_stack(3, 40, 192)
    packed, absmax = nf4.quantize_stack(W)
    cb = nf4.codebook_f64()
    for e in range(3):
        q = nf4.unpack_codes(packed[e]).reshape(-1, 64)
        a = absmax[e].astype(np.float64)
        blocks = W[e].reshape(-1, 64).astype(np.float64)
        # absmax is the exact block maximum
        assert np.array_equal(a, np.abs(blocks).max(axis=1))
        # every non-zero block holds code 0 or 15 at its largest element, which
        # dequantises to exactly +-absmax
        i = np.argmax(np.abs(blocks), axis=1)
        qi = q[np.arange(q.shape[0]), i]
        assert np.all((qi == 0) | (qi == 15))
        deq = cb[q] * a[:, None]
        assert np.array_equal(np.abs(deq[np.arange(q.shape[0]), i]), a)
        # round trip: within half the local codebook gap (plus the rounding of s)
        s = blocks / a[:, None]
        c = np.clip(np.searchsorted(cb, s, side="right") - 1, 0, 14)
        gap = cb[c + 1] - cb[c]
        bound = a[:, None] * gap / 2 + a[:, None] * 2.0 ** -24
        assert np.all(np.abs(blocks - deq) <= bound)


def test_zero_block_and_zero_elements():
    W = np.zeros((2, 2, 64), dtype=np.float32)
    W[1, 1, 5] = 0.5
    packed, absmax = nf4.quantize_stack(W)
    assert absmax[0].tolist() == [0.0, 0.0]
    assert np.all(nf4.unpack_codes(packed[0]) == 7)
    q = nf4.unpack_codes(packed[1]).reshape(2, 64)
    assert np.all(q[0] == 7)
    assert q[1, 5] == 15 and np.all(np.delete(q[1], 5) == 7)
    deq = nf4.dequantize_expert(packed[1], absmax[1], (2, 64))
    assert deq[1, 5] == 0.5 and np.count_nonzero(deq) == 1


def test_blocks_never_cross_experts():
    # Each expert here holds 64*3 elements, so blocks tile every expert exactly.
    # A huge expert next to a small one must not change the small one's bytes.
    W = _random_stack(2, 3, 64, seed=4)
    p_a, a_a = nf4.quantize_stack(W)
    W2 = W.copy()
    W2[1] *= np.float32(1000.0)
    p_b, a_b = nf4.quantize_stack(W2)
    assert np.array_equal(p_a[0], p_b[0]) and np.array_equal(a_a[0], a_b[0])
    # blocks of one expert span rows when K is not a multiple of 64
    W3 = _random_stack(1, 2, 96, seed=5)
    p3, a3 = nf4.quantize_stack(W3)
    assert a3.shape == (1, 3)
    flat = W3[0].reshape(-1)
    assert a3[0, 1] == np.abs(flat[64:128]).max()


def test_quantiser_scale_invariance_positive_control():
    # Scaling a block by a power of two leaves codes unchanged (s is unchanged)
    W = _random_stack(1, 4, 64, seed=6)
    p1, a1 = nf4.quantize_stack(W)
    p2, a2 = nf4.quantize_stack(W * np.float32(8.0))
    assert np.array_equal(p1, p2) and np.array_equal(a2, a1 * np.float32(8.0))
    # ... and the check is able to fail: flipping a sign changes the codes
    W3 = W.copy()
    W3[0, 0, 0] = -W3[0, 0, 0]
    p3, _ = nf4.quantize_stack(W3)
    assert not np.array_equal(p1, p3)
