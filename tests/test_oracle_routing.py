"""Pins for the oracle's router top-k, weights and permutation (CPU only)."""
import math

import numpy as np
import pytest

from oracle import routing


def _selection_loop_topk(logits, k):
    """Plain selection: k passes, each keeping the first strict maximum."""
    M, E = logits.shape
    out = np.zeros((M, k), dtype=np.int32)
    for t in range(M):
        used = [False] * E
        for j in range(k):
            best = -1
            for e in range(E):
                if used[e]:
                    continue
                if best < 0 or logits[t, e] > logits[t, best]:
                    best = e
            used[best] = True
            out[t, j] = best
    return out


def _counting_sort(ids, E):
    flat = ids.reshape(-1).tolist()
    buckets = [[] for _ in range(E)]
    for f, e in enumerate(flat):
        buckets[e].append(f)
    perm = [f for b in buckets for f in b]
    offs = [0]
    for b in buckets:
        offs.append(offs[-1] + len(b))
    return np.array(offs), np.array(perm)


@pytest.mark.parametrize("M,E,k", [(1, 8, 2), (17, 8, 2), (33, 64, 8), (5, 32, 4), (9, 128, 8)])
def test_topk_matches_selection_loop(M, E, k):
    rng = np.random.default_rng(M * 1000 + E)
    logits = rng.standard_normal((M, E)).astype(np.float32)
    assert np.array_equal(routing.topk(logits, k), _selection_loop_topk(logits, k))


def test_topk_ties_go_to_lower_index():
    rng = np.random.default_rng(7)
    logits = rng.integers(-2, 3, size=(40, 16)).astype(np.float32)   # many ties
    assert np.array_equal(routing.topk(logits, 5), _selection_loop_topk(logits, 5))
    assert routing.topk(np.zeros((1, 6), np.float32), 3).tolist() == [[0, 1, 2]]
    # -0.0 and +0.0 compare equal: index order decides
    z = np.array([[0.0, -0.0, 0.0]], dtype=np.float32)
    assert routing.topk(z, 3).tolist() == [[0, 1, 2]]


def test_renormalised_weights_closed_form():
    # logits log(c): the renormalised weights are c_j / sum of selected c
    c = np.array([1.0, 4.0, 2.0, 8.0, 3.0], dtype=np.float64)
    logits = np.log(c).astype(np.float32)[None, :]
    ids = routing.topk(logits, 3)
    assert ids.tolist() == [[3, 1, 4]]
    w = routing.route_weights(logits, ids, renormalize=True)
    cs = np.exp(np.log(c).astype(np.float32).astype(np.float64))[[3, 1, 4]]
    assert np.allclose(w[0], cs / cs.sum(), rtol=1e-15, atol=0)
    assert abs(w.sum() - 1.0) < 1e-15
    # without renormalisation: divided by the full sum over all experts
    w0 = routing.route_weights(logits, ids, renormalize=False)
    call = np.exp(np.log(c).astype(np.float32).astype(np.float64))
    assert np.allclose(w0[0], cs / call.sum(), rtol=1e-15, atol=0)


def test_weights_are_shift_invariant_and_ordered():
    rng = np.random.default_rng(8)
    # multiples of 2^-10, so adding 64 is exact in float32
    logits = (np.round(rng.standard_normal((20, 16)) * 1024) / 1024).astype(np.float32)
    ids = routing.topk(logits, 4)
    w = routing.route_weights(logits, ids)
    w2 = routing.route_weights(logits + np.float32(64.0), ids)
    assert np.array_equal(routing.topk(logits + np.float32(64.0), 4), ids)
    assert np.allclose(w, w2, rtol=1e-13)
    assert np.all(np.diff(w, axis=1) <= 0)           # slot 0 is the heaviest
    assert np.allclose(w.sum(axis=1), 1.0, rtol=1e-14)


def test_k_equals_E_and_k_one():
    logits = np.array([[0.5, -1.0, 2.0]], dtype=np.float32)
    ids = routing.topk(logits, 3)
    assert ids.tolist() == [[2, 0, 1]]
    w = routing.route_weights(logits, ids, renormalize=True)
    sm = np.exp(logits[0].astype(np.float64))
    sm /= sm.sum()
    assert np.allclose(w[0], sm[[2, 0, 1]], rtol=1e-15)
    ids1 = routing.topk(logits, 1)
    assert routing.route_weights(logits, ids1).tolist() == [[1.0]]


@pytest.mark.parametrize("M,E,k", [(1, 8, 2), (64, 8, 2), (3, 64, 8), (50, 128, 8), (200, 32, 4)])
def test_permutation_invariants_and_counting_sort(M, E, k):
    rng = np.random.default_rng(M + E + k)
    logits = rng.standard_normal((M, E)).astype(np.float32)
    ids = routing.topk(logits, k)
    offsets, perm, inv = routing.permute(ids, E)
    S = M * k
    assert offsets[0] == 0 and offsets[-1] == S and np.all(np.diff(offsets) >= 0)
    assert np.array_equal(np.sort(perm), np.arange(S))              # bijection
    assert np.array_equal(inv[perm], np.arange(S))                  # inv o perm = id
    assert np.array_equal(perm[inv], np.arange(S))
    flat = ids.reshape(-1)
    assert np.all(np.diff(flat[perm]) >= 0)                          # grouped by expert
    for e in range(E):
        g = perm[offsets[e]:offsets[e + 1]]
        assert np.all(flat[g] == e) and np.all(np.diff(g) > 0)      # stable
    co, cp = _counting_sort(ids, E)
    assert np.array_equal(co, offsets) and np.array_equal(cp, perm)


def test_permutation_positive_control():
    ids = np.array([[1, 0], [0, 1]], dtype=np.int32)
    offsets, perm, inv = routing.permute(ids, 2)
    assert perm.tolist() == [1, 2, 0, 3] and offsets.tolist() == [0, 2, 4]
    bad = perm.copy()
    bad[[0, 1]] = bad[[1, 0]]
    flat = ids.reshape(-1)
    g = bad[offsets[0]:offsets[1]]
    assert not np.all(np.diff(g) > 0)      # the stability check can fail
