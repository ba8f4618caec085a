"""Pins for the oracle's router (softmax + top-k) and token-to-expert alignment.

Expected values come from brute force (numpy lexsort, Python sorted()), from library
softmax (torch, float64) in the special cases where the routed weights reduce to it, from
hand-made tie cases, and from invariants; never from the oracle itself.
"""
import numpy as np
import pytest
import torch

import oracle
import synth


@pytest.mark.parametrize("T,E,k,seed", [(16, 8, 2, 0), (64, 384, 8, 0), (64, 384, 8, 1), (33, 256, 8, 2),
                                        (5, 1, 1, 0), (7, 12, 12, 3)])
def test_route_topk_matches_bruteforce_and_invariants(T, E, k, seed):
    lg = synth.logits(seed, T, E)
    ids, w32, w64 = oracle.route(lg, k)
    for t in range(T):
        order = np.lexsort((np.arange(E), -lg[t].astype(np.float64)))  # logit desc, index asc
        assert list(ids[t]) == list(order[:k])
    assert np.all((ids >= 0) & (ids < E))
    for t in range(T):
        assert len(set(ids[t])) == k
    assert np.allclose(w64.sum(1), 1.0, atol=1e-12, rtol=0)
    assert np.allclose(w32.astype(np.float64).sum(1), 1.0, atol=1e-6, rtol=0)
    assert np.all(np.diff(w64, axis=1) <= 0)  # descending with the logits
    assert np.array_equal(w32, w64.astype(np.float32))


def test_route_k_equals_E_is_full_softmax():
    lg = synth.logits(5, 9, 12)
    ids, _, w64 = oracle.route(lg, 12)
    p = torch.softmax(torch.from_numpy(lg).double(), dim=1).numpy()
    for t in range(9):
        np.testing.assert_allclose(w64[t], p[t, ids[t]], rtol=1e-13, atol=0)


def test_route_without_renormalisation_is_softmax_probability():
    lg = synth.logits(6, 10, 64, zipf_s=1.1)
    ids, _, w64 = oracle.route(lg, 4, renormalize=False)
    p = torch.softmax(torch.from_numpy(lg).double(), dim=1).numpy()
    for t in range(10):
        np.testing.assert_allclose(w64[t], p[t, ids[t]], rtol=1e-13, atol=0)


def test_route_ties_lower_index_wins():
    lg = np.array([[1.0, 3.0, 3.0, 2.0, 3.0],
                   [0.5, 0.5, 0.5, 0.5, 0.5],
                   [-1.0, -2.0, -1.0, -2.0, -3.0]], np.float32)
    ids, _, w = oracle.route(lg, 3)
    assert ids.tolist() == [[1, 2, 4], [0, 1, 2], [0, 2, 1]]
    np.testing.assert_allclose(w[1], [1 / 3] * 3, rtol=1e-15)


def test_route_renormalised_weights_closed_form():
    # two winners with logits l and l-ln(3): weights 3/4 and 1/4 whatever the others are
    lg = np.array([[0.0, np.log(3.0), -5.0, -7.0]], np.float32)
    _, _, w = oracle.route(lg, 2)
    d = float(np.float32(np.log(3.0)))  # the logit actually stored
    np.testing.assert_allclose(w[0], [np.exp(d) / (1 + np.exp(d)), 1 / (1 + np.exp(d))], rtol=1e-14)
    assert abs(w[0, 0] - 0.75) < 1e-7


def test_route_token_permutation_equivariance():
    lg = synth.logits(2, 40, 64)
    perm = np.random.default_rng(0).permutation(40)
    a = oracle.route(lg, 6)
    b = oracle.route(lg[perm], 6)
    for x, y in zip(a, b):
        assert np.array_equal(x[perm], y)


def _bruteforce_align(ids, E, A):
    T, k = ids.shape
    P = T * k
    flat = ids.reshape(-1)
    order = sorted(range(P), key=lambda p: (int(flat[p]), p))
    counts = np.bincount(flat, minlength=E).astype(np.int32)
    padded = (counts + A - 1) // A * A
    offsets = np.concatenate([[0], np.cumsum(padded)]).astype(np.int32)
    sorted_ids = np.full(offsets[-1], P, np.int32)
    inv = np.empty(P, np.int32)
    fill = offsets[:-1].copy()
    cursor = {e: 0 for e in range(E)}
    for p in order:
        e = int(flat[p])
        sorted_ids[offsets[e] + cursor[e]] = p
        inv[p] = offsets[e] + cursor[e]
        cursor[e] += 1
    return counts, offsets, sorted_ids, inv


@pytest.mark.parametrize("A", [1, 8, 16, 128])
@pytest.mark.parametrize("T,E,k,seed", [(16, 8, 2, 0), (64, 384, 8, 0), (100, 64, 6, 4), (1, 4, 4, 1),
                                        (257, 32, 8, 7)])
def test_align_matches_bruteforce(T, E, k, seed, A):
    rng = np.random.default_rng(seed)
    # distinct experts per token, as top-k produces; a skewed choice so some experts get 0
    p = 1.0 / np.arange(1, E + 1) ** 1.1
    p /= p.sum()
    ids = np.stack([rng.choice(E, size=k, replace=False, p=p) for _ in range(T)]).astype(np.int32)
    r = oracle.align(ids, E, A)
    c, o, s, inv = _bruteforce_align(ids, E, A)
    assert np.array_equal(r["counts"], c)
    assert np.array_equal(r["offsets"], o)
    assert np.array_equal(r["sorted_ids"], s)
    assert np.array_equal(r["inv_pos"], inv)
    assert r["bad"] == 0
    assert r["counts"].sum() == T * k and np.all(r["offsets"] % A == 0)
    assert np.all(r["sorted_ids"][r["inv_pos"]] == np.arange(T * k))


def test_align_flags_out_of_range_ids():
    ids = np.array([[0, 5], [1, -1], [2, 1]], np.int32)
    r = oracle.align(ids, 4, 1)
    assert r["bad"] == 2
    assert r["counts"].tolist() == [1, 2, 1, 0]
    assert r["sorted_ids"].tolist() == [0, 2, 5, 4]
    assert r["inv_pos"][1] == -1 and r["inv_pos"][3] == -1
