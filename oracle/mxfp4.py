"""MXFP4 expert weights and their grouped GEMM (oracle, float64).

TEST INFRASTRUCTURE ONLY (see the package docstring).

The pages run MoE experts natively on MXFP4 weights -- e2m1 element codes with
e8m0 block scales, multiplied straight from the released checkpoint bytes,
with no requantisation to NF4 and no bf16 copy (Solutions -- one page per
problem, the ``gemm_mxfp4_grouped`` row of grouped-nf4-gemm; the gpt-oss
entry of experts4bit-qlora 0.22.0, "Scope").  The format itself is the OCP
Microscaling (MX) one:

* e2m1 element (4 bits): sign s (bit 3), exponent e (bits 2-1, bias 1),
  mantissa m (bit 0); value (-1)^s * 2^(e-1) * (1 + m/2) for e > 0 and
  (-1)^s * m/2 for e = 0 (subnormal): magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6;
* e8m0 scale (8 bits): 2^(x - 127), with x = 255 meaning NaN;
* one scale per block of 32 consecutive elements of a row.

Layout (the released per-expert layout, as for the NF4 stacks here): an
expert's [N, K] matrix is row-major; row n holds K/2 bytes of codes and K/32
scale bytes.  Readings where the pages are silent: element 2i of a row sits
in the LOW nibble of byte i (the released-checkpoint convention; the NF4
packing of this repository is the other way round), and a NaN scale makes its
block NaN.
"""
from __future__ import annotations

from typing import Optional

import numpy as np


def e2m1_value(code: int) -> float:
    """The value of one e2m1 code, from its bit fields."""
    s = (code >> 3) & 1
    e = (code >> 1) & 3
    m = code & 1
    mag = (m / 2.0) if e == 0 else 2.0 ** (e - 1) * (1.0 + m / 2.0)
    return -mag if s else mag


def e2m1_table() -> np.ndarray:
    return np.array([e2m1_value(c) for c in range(16)], dtype=np.float64)


def e8m0_value(x: int) -> float:
    return float("nan") if x == 255 else 2.0 ** (int(x) - 127)


def unpack_codes(row_bytes: np.ndarray) -> np.ndarray:
    """Element codes of packed bytes: element 2i = low nibble of byte i."""
    b = np.asarray(row_bytes, dtype=np.uint8)
    out = np.empty(b.shape[:-1] + (2 * b.shape[-1],), dtype=np.uint8)
    out[..., 0::2] = b & 0x0F
    out[..., 1::2] = b >> 4
    return out


def dequantize_expert(blocks_e: np.ndarray, scales_e: np.ndarray, N: int, K: int) -> np.ndarray:
    """[N, K] float64 weights of one expert from its K/2 code bytes and K/32
    scale bytes per row."""
    codes = unpack_codes(np.asarray(blocks_e, dtype=np.uint8).reshape(N, K // 2))
    table = e2m1_table()
    sc = np.array([e8m0_value(x) for x in np.asarray(scales_e, dtype=np.uint8).reshape(-1)]).reshape(N, K // 32)
    return table[codes] * np.repeat(sc, 32, axis=1)


def grouped_mxfp4_gemm(A: np.ndarray, row_index: Optional[np.ndarray], offsets: np.ndarray, blocks: np.ndarray,
                       scales: np.ndarray, N: int, K: int) -> np.ndarray:
    """Row p of group e: A[row_index[p]] . W_e^T with W_e the MXFP4 expert."""
    A = np.asarray(A, dtype=np.float64)
    offsets = np.asarray(offsets, dtype=np.int64)
    E = offsets.size - 1
    rows = offsets[-1]
    idx = np.arange(rows) if row_index is None else np.asarray(row_index, dtype=np.int64)
    blocks = np.asarray(blocks, dtype=np.uint8).reshape(E, -1)
    scales = np.asarray(scales, dtype=np.uint8).reshape(E, -1)
    out = np.zeros((rows, N), dtype=np.float64)
    for e in range(E):
        lo, hi = offsets[e], offsets[e + 1]
        if hi == lo:
            continue
        out[lo:hi] = A[idx[lo:hi]] @ dequantize_expert(blocks[e], scales[e], N, K).T
    return out
