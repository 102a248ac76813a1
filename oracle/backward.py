"""Backward of the routed SwiGLU expert layer through frozen NF4 experts (oracle, float64).

TEST INFRASTRUCTURE ONLY (see the package docstring).

The pages fine-tune per-expert LoRA adapters over a frozen NF4 stack: the
frozen base projections are dequantised again from the packed bytes inside
backward, so no dequantised expert is kept between passes (experts4bit-qlora
0.22.0, the training notes under "Inference: serve the fine-tune you just
made"), and the fast lane sends that backward through one dgrad launch instead
of a per-expert decode loop (same page, "Which training path?").  This module
states what such a backward computes, for the forward of ``moe.py`` with the
routing ids held fixed (top-k selection is piecewise constant in the logits).

For an upstream gradient ``dout [M, H]`` it returns

    dx       [M, H]        the input gradient through gate_up and the LoRA path
    dlogits  [M, E]        through the routing weights
    dA, dB   [E, r, H], [E, 2I, r]   the LoRA adapter gradients (s = alpha / r)

Per slot (t, j) with e = ids[t, j] and w = w[t, j]:

    a  = x_t Wgu_e^T + s (x_t A_e^T) B_e^T         a = [g | u]
    h  = SiLU(g) * u ;  z = h Wd_e^T ;  out_t += w z
    dz = w dout_t ;  dw = dout_t . z
    dh = dz Wd_e
    dg = dh * u * SiLU'(g) ;  du = dh * SiLU(g)
         SiLU'(g) = sig(g) (1 + g (1 - sig(g))),  sig = logistic function
    da = [dg | du]
    dx_t += da Wgu_e + s (da B_e) A_e
    dB_e += s da^T (x_t A_e^T)          (outer product, 2I x r)
    dA_e += s (da B_e)^T x_t            (outer product, r x H)

Routing weights: with renormalisation, w is the softmax over the k selected
logits, so dl_(ids_j) = w_j (dw_j - sum_i w_i dw_i) and unselected logits get
zero; without it, w_j = p_(ids_j) with p the softmax over all E logits, so
dl_e = sum_j dw_j p_(ids_j) (delta(e, ids_j) - p_e).

Readings where the pages are silent: the router's logits receive the gradient
through the weights (the pages do not say whether the router trains; the
gradient is reported and a caller may ignore it); the frozen NF4 weights
receive none; the order of the sums over slots is slot order (exact float64).
"""
from __future__ import annotations

import numpy as np

from .moe import ExpertStack, silu


def _sigmoid(z: np.ndarray) -> np.ndarray:
    with np.errstate(over="ignore"):
        return 1.0 / (1.0 + np.exp(-z))


def silu_grad(z: np.ndarray) -> np.ndarray:
    """d SiLU / dz = sig(z) (1 + z (1 - sig(z)))."""
    z = np.asarray(z, dtype=np.float64)
    s = _sigmoid(z)
    return s * (1.0 + z * (1.0 - s))


def route_weights64(logits: np.ndarray, ids: np.ndarray, renormalize: bool = True) -> np.ndarray:
    """Routing weights of the selected experts from float64 logits (no float32
    rounding of the input), for differentiation; equal to
    ``routing.route_weights`` on logits that are float32 values."""
    l = np.asarray(logits, dtype=np.float64)
    sel = np.take_along_axis(l, np.asarray(ids, dtype=np.int64), axis=1)
    if renormalize:
        num = np.exp(sel - sel.max(axis=1, keepdims=True))
        return num / num.sum(axis=1, keepdims=True)
    ref = l.max(axis=1, keepdims=True)
    return np.exp(sel - ref) / np.exp(l - ref).sum(axis=1, keepdims=True)


def forward_with_weights(x: np.ndarray, ids: np.ndarray, w: np.ndarray, stack: ExpertStack) -> np.ndarray:
    """The layer output for given routing weights (slot order), float64."""
    x = np.asarray(x, dtype=np.float64)
    M, k = np.asarray(ids).shape
    out = np.zeros((M, stack.H), dtype=np.float64)
    for t in range(M):
        for j in range(k):
            e = int(ids[t, j])
            a = x[t] @ stack.gate_up(e).T
            if stack.has_lora():
                a = a + stack.lora_scale * ((x[t] @ stack.lora_A[e].T) @ stack.lora_B[e].T)
            h = silu(a[:stack.I]) * a[stack.I:]
            out[t] += w[t, j] * (h @ stack.down(e).T)
    return out


def layer_backward(x: np.ndarray, logits: np.ndarray, ids: np.ndarray, stack: ExpertStack, dout: np.ndarray,
                   renormalize: bool = True):
    """Gradients ``(dx, dlogits, dA, dB)`` of ``sum(dout * out)`` (dA, dB are
    None without an adapter), with the routing ids held fixed."""
    x = np.asarray(x, dtype=np.float64)
    dout = np.asarray(dout, dtype=np.float64)
    ids = np.asarray(ids, dtype=np.int64)
    M, k = ids.shape
    I = stack.I
    s = stack.lora_scale
    w = route_weights64(logits, ids, renormalize)
    dx = np.zeros_like(x)
    dw = np.zeros((M, k), dtype=np.float64)
    lora = stack.has_lora()
    dA = np.zeros_like(stack.lora_A) if lora else None
    dB = np.zeros_like(stack.lora_B) if lora else None
    for t in range(M):
        for j in range(k):
            e = int(ids[t, j])
            Wgu, Wd = stack.gate_up(e), stack.down(e)
            xa = x[t] @ stack.lora_A[e].T if lora else None
            a = x[t] @ Wgu.T
            if lora:
                a = a + s * (xa @ stack.lora_B[e].T)
            g, u = a[:I], a[I:]
            h = silu(g) * u
            z = h @ Wd.T
            dw[t, j] = dout[t] @ z
            dh = (w[t, j] * dout[t]) @ Wd
            da = np.concatenate([dh * u * silu_grad(g), dh * silu(g)])
            dx[t] += da @ Wgu
            if lora:
                daB = da @ stack.lora_B[e]            # [r]
                dx[t] += s * (daB @ stack.lora_A[e])
                dB[e] += s * np.outer(da, xa)
                dA[e] += s * np.outer(daB, x[t])
    # Through the routing weights.
    l = np.asarray(logits, dtype=np.float64)
    dlogits = np.zeros_like(l)
    if renormalize:
        inner = (w * dw).sum(axis=1, keepdims=True)
        np.put_along_axis(dlogits, ids, w * (dw - inner), axis=1)
    else:
        p = np.exp(l - l.max(axis=1, keepdims=True))
        p /= p.sum(axis=1, keepdims=True)
        for t in range(M):
            for j in range(k):
                e = int(ids[t, j])
                coef = dw[t, j] * p[t, e]
                dlogits[t] -= coef * p[t]
                dlogits[t, e] += coef
    return dx, dlogits, dA, dB


def grouped_nf4_gemm_dgrad(dY: np.ndarray, row_index, offsets: np.ndarray, packed: np.ndarray,
                           absmax: np.ndarray, N: int, K: int, lora_A=None, lora_B=None,
                           lora_scale: float = 0.0, quant: str = "nf4") -> np.ndarray:
    """The input gradient of the grouped NF4 GEMM, in one call over all groups.

    The forward row p is ``y_p = a_p . W_e^T (+ s (a_p . A_e^T) . B_e^T)``; for
    an upstream gradient ``dY`` the result row p is

        da_p = dY[row_index[p]] . W_e  (+ s (dY[row_index[p]] . B_e) . A_e)

    with W_e the dequantised [N, K] expert of the group e holding p (the
    frozen base is decoded again from the packed bytes, never kept), so the
    result has K columns.  ``row_index=None`` means identity; ``quant`` names
    the storage of ``packed`` (``nf4`` or ``fp4``).  This is the
    single grouped dgrad launch the pages put in place of a per-expert decode
    loop (experts4bit-qlora 0.22.0, "Which training path?").
    """
    from . import moe
    dY = np.asarray(dY, dtype=np.float64)
    offsets = np.asarray(offsets, dtype=np.int64)
    E = offsets.size - 1
    rows = offsets[-1]
    idx = np.arange(rows) if row_index is None else np.asarray(row_index, dtype=np.int64)
    packed = np.asarray(packed, dtype=np.uint8).reshape(E, -1)
    absmax = np.asarray(absmax, dtype=np.float32).reshape(E, -1)
    out = np.zeros((rows, K), dtype=np.float64)
    for e in range(E):
        lo, hi = offsets[e], offsets[e + 1]
        if hi == lo:
            continue
        W = moe.dequantize(quant, packed[e], absmax[e], (N, K))
        G = dY[idx[lo:hi]]
        d = G @ W
        if lora_A is not None and lora_B is not None:
            la = np.asarray(lora_A, dtype=np.float64)[e]
            lb = np.asarray(lora_B, dtype=np.float64)[e]
            d = d + lora_scale * ((G @ lb) @ la)
        out[lo:hi] = d
    return out


def grouped_lora_grads(x: np.ndarray, row_index, offsets: np.ndarray, da: np.ndarray, lora_A: np.ndarray,
                       lora_B: np.ndarray, lora_scale: float):
    """The adapter gradients of one grouped projection, from the gradient ``da``
    of its output rows (group order) and its input rows ``x[row_index[p]]``:

        dB_e = s * sum_{p in e} da_p^T (x_p . A_e^T)        [N, r]
        dA_e = s * sum_{p in e} (da_p . B_e)^T x_p          [r, K]

    (the per-slot outer products of ``layer_backward`` summed over a group).
    Experts without rows get zero gradients."""
    x = np.asarray(x, dtype=np.float64)
    da = np.asarray(da, dtype=np.float64)
    lora_A = np.asarray(lora_A, dtype=np.float64)
    lora_B = np.asarray(lora_B, dtype=np.float64)
    off = np.asarray(offsets, dtype=np.int64)
    rows = off[-1]
    idx = np.arange(rows) if row_index is None else np.asarray(row_index, dtype=np.int64)
    dA = np.zeros_like(lora_A)
    dB = np.zeros_like(lora_B)
    for e in range(off.size - 1):
        lo, hi = off[e], off[e + 1]
        if hi == lo:
            continue
        xe = x[idx[lo:hi]]
        dae = da[lo:hi]
        dB[e] = lora_scale * dae.T @ (xe @ lora_A[e].T)
        dA[e] = lora_scale * (dae @ lora_B[e]).T @ xe
    return dA, dB


def layer_backward_grouped(x: np.ndarray, logits: np.ndarray, ids: np.ndarray, stack: ExpertStack,
                           dout: np.ndarray, renormalize: bool = True):
    """``layer_backward`` restated in the permuted, grouped form a GPU runs:
    gather by the permutation, recompute the gate_up output and z per group,
    two grouped dgrad products (down, then gate_up with its LoRA term), the
    SwiGLU derivative in between, and the per-token sum through the inverse
    permutation.  Returns the same ``(dx, dlogits, dA, dB)``."""
    from . import moe, routing
    x = np.asarray(x, dtype=np.float64)
    dout = np.asarray(dout, dtype=np.float64)
    ids = np.asarray(ids, dtype=np.int64)
    M, k = ids.shape
    I, H = stack.I, stack.H
    s = stack.lora_scale
    lora = stack.has_lora()
    w = route_weights64(logits, ids, renormalize)
    offsets, perm, inv = routing.permute(ids.astype(np.int32), stack.E)
    perm = np.asarray(perm, dtype=np.int64)
    tok = perm // k
    a = moe.grouped_nf4_gemm(x, tok, offsets, stack.gu_packed, stack.gu_absmax, 2 * I, H,
                             stack.lora_A if lora else None, stack.lora_B if lora else None, s,
                             quant=stack.quant)
    g, u = a[:, :I], a[:, I:]
    h = silu(g) * u
    z = moe.grouped_nf4_gemm(h, None, offsets, stack.dn_packed, stack.dn_absmax, H, I, quant=stack.quant)
    wp = w.reshape(-1)[perm]                       # routing weight of each grouped row
    dz = wp[:, None] * dout[tok]
    dh = grouped_nf4_gemm_dgrad(dz, None, offsets, stack.dn_packed, stack.dn_absmax, H, I, quant=stack.quant)
    da = np.concatenate([dh * u * silu_grad(g), dh * silu(g)], axis=1)
    dxg = grouped_nf4_gemm_dgrad(da, None, offsets, stack.gu_packed, stack.gu_absmax, 2 * I, H,
                                 stack.lora_A if lora else None, stack.lora_B if lora else None, s,
                                 quant=stack.quant)
    dx = dxg[np.asarray(inv, dtype=np.int64)].reshape(M, k, H).sum(axis=1)
    dw = np.zeros(M * k, dtype=np.float64)
    dw[perm] = np.sum(dout[tok] * z, axis=1)
    dw = dw.reshape(M, k)
    dA = dB = None
    if lora:
        dA, dB = grouped_lora_grads(x, tok, offsets, da, stack.lora_A, stack.lora_B, s)
    l = np.asarray(logits, dtype=np.float64)
    dlogits = np.zeros_like(l)
    if renormalize:
        inner = (w * dw).sum(axis=1, keepdims=True)
        np.put_along_axis(dlogits, ids, w * (dw - inner), axis=1)
    else:
        p = np.exp(l - l.max(axis=1, keepdims=True))
        p /= p.sum(axis=1, keepdims=True)
        for j in range(k):
            coef = dw[:, j] * p[np.arange(M), ids[:, j]]
            dlogits -= coef[:, None] * p
            dlogits[np.arange(M), ids[:, j]] += coef
    return dx, dlogits, dA, dB
