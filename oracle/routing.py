"""Router top-k and the token/expert permutation (oracle).

TEST INFRASTRUCTURE ONLY (see the package docstring).

The pages describe the batched path as "sort token/expert pairs, run the
groups as bmms" (experts4bit-qlora 0.22.0, section "Which training path?") and
the fused path as one grouped launch over the routed experts (Solutions -- one
page per problem, the grouped-nf4-gemm row on ``gemm_4bit_grouped``).  The
routing itself ("softmax top-k renormalised") comes from the layer shapes the
measurements use.

Readings where the pages are silent:
* Top-k order: experts sorted by (logit descending, expert index ascending);
  slot j of a token holds the j-th expert in that order, so equal logits go to
  the lower index.
* Weights with renormalisation: the softmax restricted to the k selected
  logits, ``w_j = exp(l_j - l_0) / sum_{i<k} exp(l_i - l_0)``; without it, the
  full softmax over all E experts evaluated at the selected ones.
* Permutation: flat slot ``f = t*k + j``; ``perm`` lists the slots in a stable
  sort by expert id (ties keep ascending f); ``inv[perm[p]] = p``;
  ``offsets[e]`` is the first permuted position of expert e, ``offsets[E] = S``.
"""
from __future__ import annotations

import numpy as np


def topk(logits: np.ndarray, k: int):
    """Indices ``[M, k]`` (int32) of the k largest logits per row, ties to the lower index."""
    logits = np.asarray(logits, dtype=np.float32)
    M, E = logits.shape
    if not 1 <= k <= E:
        raise ValueError("k must be in [1, E]")
    ids = np.empty((M, k), dtype=np.int32)
    idx = np.arange(E)
    for t in range(M):
        # Primary key: logit descending; secondary: index ascending.
        order = np.lexsort((idx, -logits[t].astype(np.float64)))
        ids[t] = order[:k]
    return ids


def route_weights(logits: np.ndarray, ids: np.ndarray, renormalize: bool = True) -> np.ndarray:
    """Routing weights ``[M, k]`` in float64 for the selected experts."""
    l = np.asarray(logits, dtype=np.float32).astype(np.float64)
    sel = np.take_along_axis(l, np.asarray(ids, dtype=np.int64), axis=1)
    if renormalize:
        ref = sel[:, :1]                      # the largest selected logit
        num = np.exp(sel - ref)
        return num / num.sum(axis=1, keepdims=True)
    ref = l.max(axis=1, keepdims=True)
    return np.exp(sel - ref) / np.exp(l - ref).sum(axis=1, keepdims=True)


def permute(ids: np.ndarray, E: int):
    """Group the ``S = M*k`` flat slots by expert.

    Returns ``(offsets [E+1], perm [S], inv [S])`` as int32.
    """
    flat = np.asarray(ids, dtype=np.int64).reshape(-1)
    S = flat.size
    counts = np.bincount(flat, minlength=E)
    offsets = np.zeros(E + 1, dtype=np.int64)
    offsets[1:] = np.cumsum(counts)
    perm = np.argsort(flat, kind="stable")
    inv = np.empty(S, dtype=np.int64)
    inv[perm] = np.arange(S)
    return offsets.astype(np.int32), perm.astype(np.int32), inv.astype(np.int32)


def route_permute(logits: np.ndarray, k: int, renormalize: bool = True):
    """Router top-k + permutation.  Returns ``(ids, w, offsets, perm, inv)``."""
    E = np.asarray(logits).shape[1]
    ids = topk(logits, k)
    w = route_weights(logits, ids, renormalize)
    offsets, perm, inv = permute(ids, E)
    return ids, w, offsets, perm, inv
