"""FP4 blockwise storage of a fused expert stack (oracle).

TEST INFRASTRUCTURE ONLY (see the package docstring).

What the pages fix
------------------
* The same fused stack can be stored at a selectable precision, among them
  the two 4-bit packed modes ``nf4`` and ``fp4``, with a fidelity ordering
  pinned by tests in which the NF4 reconstruction error is below the FP4 one
  (experts4bit-qlora 0.22.0, opening section; "Scope", storage modes).
* The pages call the 4-bit elements of MXFP4 checkpoints "fp4" ("Why does
  load_in_4bit still OOM on a Mixture-of-Experts model?", section "Why it
  happens"), and name their format e2m1 (Solutions -- one page per problem,
  the ``gemm_mxfp4_grouped`` row).

Readings where the pages are silent (each listed in the design notes)
--------------------------------------------------------------------
* Codebook: code c is an e2m1 element -- sign bit 3, exponent bits 2-1 (bias
  1), mantissa bit 0, magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6 -- divided by the
  largest magnitude 6, so that the block's absmax maps to code 7 (+1) or 15
  (-1); each entry is stored as the float32 nearest to that rational.
* Everything else is the NF4 storage of this repository: blocks of 64
  consecutive elements of an expert's row-major flattening, fp32 absmax,
  ``s = fl32(w / a)``, two codes per byte with the lower-index element in the
  high nibble.
* Code choice: the nearest entry to ``s`` in exact arithmetic; a value exactly
  halfway between two entries takes the smaller one; zero is code 0, so code
  8 (-0) is never written.  An all-zero block stores ``a = 0`` and code 0.
"""
from __future__ import annotations

import numpy as np

from . import mxfp4, nf4

BLOCKSIZE = nf4.BLOCKSIZE
ZERO_CODE = 0


def codebook_f64() -> np.ndarray:
    """Entry c = fl32(e2m1(c) / 6), in code order, as float64."""
    v = np.array([mxfp4.e2m1_value(c) / 6.0 for c in range(16)], dtype=np.float64)
    return v.astype(np.float32).astype(np.float64)


def _levels():
    """The distinct entries in ascending order and, for each, its code (the
    lowest code holding that value: +0 for zero)."""
    cb = codebook_f64()
    values = np.unique(cb)
    codes = np.array([int(np.flatnonzero(cb == v)[0]) for v in values], dtype=np.uint8)
    return values, codes


def midpoints() -> np.ndarray:
    """Decision points between neighbouring distinct entries, exact in float64."""
    values, _ = _levels()
    return (values[:-1] + values[1:]) / 2.0


def code_of_scaled(s: np.ndarray) -> np.ndarray:
    """The code of each float32 ``s``: the level index is the number of decision
    points strictly below ``s`` (a value on a decision point takes the smaller
    level); the code is that level's code."""
    s64 = np.asarray(s, dtype=np.float32).astype(np.float64)
    rank = np.zeros(s64.shape, dtype=np.int64)
    for m in midpoints():
        rank += (s64 > m)
    _, codes = _levels()
    return codes[rank]


def quantize_expert(w: np.ndarray):
    """Quantise one expert (any shape, row-major flattened) ->
    ``(packed uint8 [n/2], absmax float32 [n/64])``."""
    flat = np.ascontiguousarray(w, dtype=np.float32).reshape(-1)
    n = flat.size
    if n % BLOCKSIZE != 0:
        raise ValueError("expert size must be a multiple of the block size 64")
    blocks = flat.reshape(n // BLOCKSIZE, BLOCKSIZE)
    absmax = np.max(np.abs(blocks), axis=1).astype(np.float32)
    zero = absmax == 0
    safe = np.where(zero, np.float32(1.0), absmax).astype(np.float32)
    s = (blocks / safe[:, None]).astype(np.float32)   # IEEE float32 division
    q = code_of_scaled(s)
    q[zero, :] = ZERO_CODE
    return nf4.pack_codes(q.reshape(-1)), absmax


def quantize_stack(W: np.ndarray):
    """Quantise a fused stack ``W [E, ...]`` expert by expert."""
    W = np.asarray(W)
    E = W.shape[0]
    n = int(np.prod(W.shape[1:]))
    packed = np.empty((E, n // 2), dtype=np.uint8)
    absmax = np.empty((E, n // BLOCKSIZE), dtype=np.float32)
    for e in range(E):
        packed[e], absmax[e] = quantize_expert(W[e])
    return packed, absmax


def dequantize_expert(packed_e: np.ndarray, absmax_e: np.ndarray, shape) -> np.ndarray:
    """``codebook[q] * absmax`` in float64 (exact: a product of two float32)."""
    q = nf4.unpack_codes(np.asarray(packed_e).reshape(-1))
    a = np.repeat(np.asarray(absmax_e, dtype=np.float32).astype(np.float64), BLOCKSIZE)
    return (codebook_f64()[q] * a).reshape(shape)
