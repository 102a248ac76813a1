"""Grouped NF4 GEMM and the routed SwiGLU expert layer (oracle, float64).

TEST INFRASTRUCTURE ONLY (see the package docstring).

What the layer computes, per token t and slot j with expert e = ids[t, j]:

    g_u   = x_t . Wgu_e^T                         (length 2I)
    g_u  += (alpha / r) * ((x_t . A_e^T) . B_e^T)  (only with a LoRA adapter)
    h     = SiLU(g_u[:I]) * g_u[I:]               SiLU(z) = z / (1 + exp(-z))
    z_j   = h . Wd_e^T                            (length H)
    out_t = sum_j w[t, j] * z_j                   (j ascending)

Sources: the expert MLP is SwiGLU ("supports SwiGLU fused-MoE architectures",
experts4bit-qlora 0.22.0, section "Scope"); the adapter is a "per-expert
low-rank delta before each routed expert's activation" over the frozen NF4
stack (Solutions -- one page per problem, the ExpertsLoRA row) with r=8,
alpha=16 (experts4bit-qlora 0.22.0, "Quickstart"); the GEMM runs on the NF4
bytes with float32 accumulation and no bf16 expert tensor (same Solutions page,
the grouped-nf4-gemm ``gemm_4bit_grouped`` row); the weighted sum over the
experts of a token (experts4bit-qlora 0.22.0, "Which training path?",
numerics paragraph).

Readings where the pages are silent:
* gate/up are the two halves of ``gate_up_proj[e]``: rows [0, I) gate, rows
  [I, 2I) up (not interleaved); no biases;
* LoRA scale alpha/r; A is [E, r, H], B is [E, 2I, r]; the delta applies to
  gate_up only;
* the oracle sums the k expert outputs in slot order j (the pages sum in
  group-sorted order; both are correct results of the same sum);
* every step here is exact float64 with no intermediate rounding; the
  tolerance of the parity tests covers the bf16 roundings of the GPU path.
"""
from __future__ import annotations

from typing import Optional

import numpy as np

from . import fp4, nf4

QUANT_TYPES = {"nf4": nf4, "fp4": fp4}


def dequantize(quant: str, packed_e, absmax_e, shape) -> np.ndarray:
    """One expert's weights in float64 from its 4-bit storage (``nf4`` or ``fp4``)."""
    return QUANT_TYPES[quant].dequantize_expert(packed_e, absmax_e, shape)


def silu(z: np.ndarray) -> np.ndarray:
    z = np.asarray(z, dtype=np.float64)
    with np.errstate(over="ignore"):
        return z / (1.0 + np.exp(-z))


class ExpertStack:
    """A 4-bit fused stack pair (NF4, or FP4 with ``quant="fp4"``) with lazily
    dequantised float64 experts."""

    def __init__(self, gu_packed, gu_absmax, dn_packed, dn_absmax, E, H, I,
                 lora_A=None, lora_B=None, lora_scale=0.0, quant="nf4"):
        self.gu_packed = np.asarray(gu_packed, dtype=np.uint8).reshape(E, -1)
        self.gu_absmax = np.asarray(gu_absmax, dtype=np.float32).reshape(E, -1)
        self.dn_packed = np.asarray(dn_packed, dtype=np.uint8).reshape(E, -1)
        self.dn_absmax = np.asarray(dn_absmax, dtype=np.float32).reshape(E, -1)
        self.E, self.H, self.I = int(E), int(H), int(I)
        self.lora_A = None if lora_A is None else np.asarray(lora_A, dtype=np.float64)
        self.lora_B = None if lora_B is None else np.asarray(lora_B, dtype=np.float64)
        self.lora_scale = float(lora_scale)
        if quant not in QUANT_TYPES:
            raise ValueError(f"unknown storage type {quant!r}")
        self.quant = quant
        self._gu = {}
        self._dn = {}

    def gate_up(self, e: int) -> np.ndarray:
        """Dequantised ``[2I, H]`` float64."""
        if e not in self._gu:
            self._gu[e] = dequantize(self.quant, self.gu_packed[e], self.gu_absmax[e],
                                     (2 * self.I, self.H))
        return self._gu[e]

    def down(self, e: int) -> np.ndarray:
        """Dequantised ``[H, I]`` float64."""
        if e not in self._dn:
            self._dn[e] = dequantize(self.quant, self.dn_packed[e], self.dn_absmax[e],
                                     (self.H, self.I))
        return self._dn[e]

    def has_lora(self) -> bool:
        return self.lora_A is not None and self.lora_B is not None


def expert_mlp(stack: ExpertStack, e: int, xrows: np.ndarray) -> np.ndarray:
    """The SwiGLU MLP of expert e on rows ``xrows [R, H]`` (float64) -> ``[R, H]``."""
    I = stack.I
    gu = xrows @ stack.gate_up(e).T
    if stack.has_lora():
        gu = gu + stack.lora_scale * ((xrows @ stack.lora_A[e].T) @ stack.lora_B[e].T)
    h = silu(gu[:, :I]) * gu[:, I:]
    return h @ stack.down(e).T


def moe_forward_per_token(x: np.ndarray, ids: np.ndarray, w: np.ndarray,
                          stack: ExpertStack, tokens: Optional[np.ndarray] = None) -> np.ndarray:
    """Brute-force dense loop: every token, every slot, one expert at a time.

    ``tokens`` (optional) restricts the computation to those token indices;
    the result then has one row per listed token.
    """
    x = np.asarray(x, dtype=np.float64)
    ids = np.asarray(ids)
    w = np.asarray(w, dtype=np.float64)
    rows = np.arange(x.shape[0]) if tokens is None else np.asarray(tokens)
    out = np.zeros((rows.size, stack.H), dtype=np.float64)
    for i, t in enumerate(rows):
        for j in range(ids.shape[1]):
            z = expert_mlp(stack, int(ids[t, j]), x[t:t + 1])[0]
            out[i] += w[t, j] * z
    return out


def grouped_nf4_gemm(A: np.ndarray, row_index: Optional[np.ndarray], offsets: np.ndarray,
                     packed: np.ndarray, absmax: np.ndarray, N: int, K: int,
                     lora_A=None, lora_B=None, lora_scale: float = 0.0,
                     swiglu: bool = False, quant: str = "nf4") -> np.ndarray:
    """One grouped GEMM over the groups ``[offsets[e], offsets[e+1])``.

    Row p of the result is ``A[row_index[p]] . W_e^T`` (plus the LoRA delta)
    for the group e holding p; with ``swiglu`` the result is
    ``SiLU(y[:, :N/2]) * y[:, N/2:]``.  ``row_index=None`` means identity;
    ``quant`` names the storage of ``packed`` (``nf4`` or ``fp4``).
    """
    A = np.asarray(A, dtype=np.float64)
    offsets = np.asarray(offsets, dtype=np.int64)
    E = offsets.size - 1
    rows = offsets[-1]
    idx = np.arange(rows) if row_index is None else np.asarray(row_index, dtype=np.int64)
    packed = np.asarray(packed, dtype=np.uint8).reshape(E, -1)
    absmax = np.asarray(absmax, dtype=np.float32).reshape(E, -1)
    out = np.zeros((rows, N // 2 if swiglu else N), dtype=np.float64)
    for e in range(E):
        lo, hi = offsets[e], offsets[e + 1]
        if hi == lo:
            continue
        W = dequantize(quant, packed[e], absmax[e], (N, K))
        Xe = A[idx[lo:hi]]
        y = Xe @ W.T
        if lora_A is not None and lora_B is not None:
            la = np.asarray(lora_A, dtype=np.float64)[e]
            lb = np.asarray(lora_B, dtype=np.float64)[e]
            y = y + lora_scale * ((Xe @ la.T) @ lb.T)
        if swiglu:
            y = silu(y[:, :N // 2]) * y[:, N // 2:]
        out[lo:hi] = y
    return out


def moe_forward_grouped(x: np.ndarray, ids: np.ndarray, w: np.ndarray, offsets: np.ndarray,
                        perm: np.ndarray, inv: np.ndarray, stack: ExpertStack) -> np.ndarray:
    """The permuted form: gather by perm, one GEMM per expert group, combine via inv."""
    x = np.asarray(x, dtype=np.float64)
    M, k = np.asarray(ids).shape
    perm = np.asarray(perm, dtype=np.int64)
    h = grouped_nf4_gemm(x, perm // k, offsets, stack.gu_packed, stack.gu_absmax,
                         2 * stack.I, stack.H,
                         stack.lora_A if stack.has_lora() else None,
                         stack.lora_B if stack.has_lora() else None,
                         stack.lora_scale, swiglu=True, quant=stack.quant)
    z = grouped_nf4_gemm(h, None, offsets, stack.dn_packed, stack.dn_absmax,
                         stack.H, stack.I, quant=stack.quant)
    zs = z[np.asarray(inv, dtype=np.int64)].reshape(M, k, stack.H)
    out = np.zeros((M, stack.H), dtype=np.float64)
    w = np.asarray(w, dtype=np.float64)
    for j in range(k):
        out += w[:, j:j + 1] * zs[:, j, :]
    return out
