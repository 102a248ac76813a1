"""NF4 blockwise quantisation of a fused 3-D expert stack (oracle).

TEST INFRASTRUCTURE ONLY (see the package docstring).

What the pages fix
------------------
* Fused stacks ``gate_up_proj [E, 2I, H]`` and ``down_proj [E, H, I]`` --
  "Why does load_in_4bit still OOM on a Mixture-of-Experts model?", section
  "Why it happens".
* Quantisation blocks "never cross an expert boundary" -- same page, section
  "Which project solves it".
* One fixed 16-entry codebook with a per-block absmax ("same codebook, same
  per-expert absmax") -- experts4bit-qlora 0.22.0, section "Inference: serve
  the fine-tune you just made"; the fast path accepts only NF4 with blocksize
  64 -- same page, section "Install".

Readings where the pages are silent (each listed in the design notes)
--------------------------------------------------------------------
* Codebook values: the NF4 table of the QLoRA paper (Dettmers et al. 2023,
  Appendix E), which bitsandbytes ships.  The pages never print it.
* Quantiser: per block of 64 consecutive elements of one expert's row-major
  flattening, ``a = max |w|`` (float32, exact); ``s = fl32(w / a)`` (one IEEE
  float32 division, round to nearest even); code = the nearest codebook entry
  in exact arithmetic, ties to the lower index; an all-zero block stores
  ``a = 0`` and code 7 (the entry 0.0) everywhere.
* Packing: two codes per byte, the element with the lower index in the high
  nibble.
* Parity unpinned: byte compatibility with the bitsandbytes library itself.
"""
from __future__ import annotations

import numpy as np

BLOCKSIZE = 64

# NF4 codebook, QLoRA paper Appendix E, as float32 (ascending; entry 7 is 0.0).
NF4_CODEBOOK = np.array(
    [
        -1.0,
        -0.6961928009986877,
        -0.5250730514526367,
        -0.39491748809814453,
        -0.28444138169288635,
        -0.18477343022823334,
        -0.09105003625154495,
        0.0,
        0.07958029955625534,
        0.16093020141124725,
        0.24611230194568634,
        0.33791524171829224,
        0.44070982933044434,
        0.5626170039176941,
        0.7229568362236023,
        1.0,
    ],
    dtype=np.float32,
)


def codebook_f64() -> np.ndarray:
    return NF4_CODEBOOK.astype(np.float64)


def derived_codebook() -> np.ndarray:
    """The NF4 construction of the QLoRA paper, in float64.

    Eight positive normal quantiles at ``linspace(0.9677083, 0.5, 9)[:-1]``,
    seven negated quantiles at ``linspace(0.9677083, 0.5, 8)[:-1]``, and 0;
    sorted and divided by the largest.  Used only to pin the stored table.
    """
    from scipy.stats import norm

    offset = 0.9677083
    pos = norm.ppf(np.linspace(offset, 0.5, 9)[:-1])
    neg = -norm.ppf(np.linspace(offset, 0.5, 8)[:-1])
    v = np.sort(np.concatenate([pos, [0.0], neg]))
    return v / v.max()


def midpoints() -> np.ndarray:
    """The 15 decision points between neighbouring codes, exact in float64.

    The sum of two float32 values is exact in float64 and halving is exact.
    """
    cb = codebook_f64()
    return (cb[:-1] + cb[1:]) / 2.0


def code_of_scaled(s: np.ndarray) -> np.ndarray:
    """Nearest code to each float32 ``s`` in exact arithmetic, ties to the lower.

    The code is the number of decision points strictly below ``s``: a value
    exactly on a decision point therefore takes the lower of the two codes.
    """
    s64 = np.asarray(s, dtype=np.float32).astype(np.float64)
    q = np.zeros(s64.shape, dtype=np.uint8)
    for m in midpoints():
        q += (s64 > m).astype(np.uint8)
    return q


def pack_codes(q: np.ndarray) -> np.ndarray:
    """Pack codes along the last axis, two per byte, lower index in the high nibble."""
    q = np.asarray(q, dtype=np.uint8)
    assert q.shape[-1] % 2 == 0
    return ((q[..., 0::2] << 4) | q[..., 1::2]).astype(np.uint8)


def unpack_codes(packed: np.ndarray) -> np.ndarray:
    """Inverse of :func:`pack_codes`."""
    p = np.asarray(packed, dtype=np.uint8)
    out = np.empty(p.shape[:-1] + (p.shape[-1] * 2,), dtype=np.uint8)
    out[..., 0::2] = p >> 4
    out[..., 1::2] = p & 0x0F
    return out


def quantize_expert(w: np.ndarray):
    """Quantise one expert's weights (any shape, row-major flattened).

    Returns ``(packed uint8 [n/2], absmax float32 [n/64])``.
    """
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
    q[zero, :] = 7
    return pack_codes(q.reshape(-1)), absmax


def quantize_stack(W: np.ndarray):
    """Quantise a fused stack ``W [E, ...]`` expert by expert.

    Blocks are formed inside each expert's own flattening, so none crosses an
    expert boundary.  Returns ``(packed [E, n/2] uint8, absmax [E, n/64] f32)``.
    """
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
    q = unpack_codes(np.asarray(packed_e).reshape(-1))
    a = np.repeat(np.asarray(absmax_e, dtype=np.float32).astype(np.float64), BLOCKSIZE)
    return (codebook_f64()[q] * a).reshape(shape)
