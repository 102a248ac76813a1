"""Pins of the MXFP4 oracle (oracle/mxfp4.py): the e2m1 and e8m0 field
definitions, a block worked out by hand from those definitions, the packing
order and the grouped GEMM against per-element sums."""
import numpy as np
import pytest

from oracle import mxfp4


def test_e2m1_magnitudes_and_signs():
    t = mxfp4.e2m1_table()
    assert list(t[:8]) == [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    assert np.array_equal(t[8:], -t[:8])
    assert np.signbit(t[8]) and t[8] == 0.0          # code 8 is -0
    # every magnitude is exactly representable in bf16 (at most 2 significant bits)
    assert all(float(np.float32(v)) == v for v in t)


def test_e8m0_scale():
    assert mxfp4.e8m0_value(127) == 1.0
    assert mxfp4.e8m0_value(128) == 2.0 and mxfp4.e8m0_value(126) == 0.5
    assert mxfp4.e8m0_value(0) == 2.0 ** -127
    assert np.isnan(mxfp4.e8m0_value(255))


def test_hand_worked_block():
    """Scale byte 129 is 2^2 = 4.  Byte 0x10 holds code 0 (low nibble, element 0:
    +0 * 4) and code 1 (element 1: 0.5 * 4 = 2); 0x98 holds code 8 (-0) and 9
    (-0.5 * 4); the second half repeats the codes with the nibbles swapped."""
    scale = np.array([129], dtype=np.uint8)
    blk = np.array([0x10, 0x32, 0x54, 0x76, 0x98, 0xBA, 0xDC, 0xFE, 0x01, 0x23, 0x45, 0x67, 0x89, 0xAB, 0xCD, 0xEF],
                   dtype=np.uint8)
    vals = np.array([0, 2, 4, 6, 8, 12, 16, 24, -0.0, -2, -4, -6, -8, -12, -16, -24,
                     2, 0, 6, 4, 12, 8, 24, 16, -2, -0.0, -6, -4, -12, -8, -24, -16], dtype=np.float64)
    w = mxfp4.dequantize_expert(blk, scale, 1, 32)[0]
    assert np.array_equal(w, vals)
    assert np.array_equal(np.signbit(w), np.signbit(vals))   # the two -0 entries


def test_packing_is_low_nibble_first():
    codes = mxfp4.unpack_codes(np.array([0x21], dtype=np.uint8))
    assert list(codes) == [1, 2]


def test_grouped_gemm_against_per_element_sums():
    rng = np.random.default_rng(4)
    E, N, K = 3, 5, 64
    blocks = rng.integers(0, 256, size=(E, N * K // 2), dtype=np.uint8)
    scales = rng.integers(120, 132, size=(E, N * K // 32), dtype=np.uint8)
    offsets = np.array([0, 3, 3, 7])
    A = rng.standard_normal((9, K))
    idx = np.array([8, 1, 1, 0, 5, 2, 7])
    y = mxfp4.grouped_mxfp4_gemm(A, idx, offsets, blocks, scales, N, K)
    t = mxfp4.e2m1_table()
    for p in range(7):
        e = int(np.searchsorted(offsets, p, side="right") - 1)
        for n in range(N):
            ref = 0.0
            for kk in range(K):
                byte = blocks[e, (n * K + kk) // 2]
                code = (byte & 0x0F) if kk % 2 == 0 else (byte >> 4)
                ref += A[idx[p], kk] * t[code] * 2.0 ** (int(scales[e, (n * K + kk) // 32]) - 127)
            assert y[p, n] == pytest.approx(ref, rel=1e-12, abs=1e-12)
    # a planted mistake (high nibble first) changes the result
    swapped = ((blocks & 0x0F) << 4) | (blocks >> 4)
    assert not np.allclose(mxfp4.grouped_mxfp4_gemm(A, idx, offsets, swapped, scales, N, K), y)
