"""Pins of the oracle's routing and permutation: closed forms, brute force, invariants."""
import itertools

import numpy as np
import pytest

from oracle import moe
from tests.golden import load


def test_route_closed_form():
    g = load("route_closed_form.txt")
    logits = np.log(np.array([[1.0, 2.0, 3.0, 4.0]]))
    idx, prob = moe.route(logits, g["k"], renorm=False)
    assert list(idx[0]) == g["idx"]
    np.testing.assert_allclose(prob[0], g["prob_raw"], rtol=0, atol=1e-15)
    idx, prob = moe.route(logits, g["k"], renorm=True)
    assert list(idx[0]) == g["idx"]
    np.testing.assert_allclose(prob[0], g["prob_renorm"], rtol=0, atol=1e-15)


def _brute_route(lg, k, renorm):
    """Full enumeration: the selected set maximises the sum of logits (lexicographic
    tie-break on lower indices), ordered by descending logit then index."""
    T, E = lg.shape
    idx = np.zeros((T, k), dtype=np.int64)
    prob = np.zeros((T, k))
    for t in range(T):
        keyed = sorted(range(E), key=lambda e: (-lg[t, e], e))
        sel = keyed[:k]
        # the chosen set is a maximum-sum k-subset
        best = max(sum(lg[t, list(c)]) for c in itertools.combinations(range(E), k))
        assert sum(lg[t, sel]) == best
        z = sum(np.exp(lg[t, e]) for e in range(E))
        p = [np.exp(lg[t, e]) / z for e in sel]
        if renorm:
            s = sum(p)
            p = [q / s for q in p]
        idx[t] = sel
        prob[t] = p
    return idx, prob


@pytest.mark.parametrize("renorm", [True, False])
@pytest.mark.parametrize("E,k", [(4, 1), (4, 2), (6, 3), (5, 5)])
def test_route_brute_force_with_ties(E, k, renorm):
    rng = np.random.default_rng(E * 10 + k)
    lg = rng.integers(-2, 3, size=(40, E)).astype(np.float64)   # many exact ties
    idx, prob = moe.route(lg, k, renorm)
    bidx, bprob = _brute_route(lg, k, renorm)
    assert np.array_equal(idx, bidx)
    np.testing.assert_allclose(prob, bprob, rtol=1e-13, atol=0)


def test_route_invariants():
    rng = np.random.default_rng(5)
    lg = rng.normal(size=(300, 16)).astype(np.float32)
    idx, prob = moe.route(lg, 4, True)
    assert idx.dtype == np.int32
    assert np.all((idx >= 0) & (idx < 16))
    assert all(len(set(r)) == 4 for r in idx)
    np.testing.assert_allclose(prob.sum(axis=1), 1.0, rtol=0, atol=1e-14)
    assert np.all(np.diff(np.take_along_axis(lg, idx, 1), axis=1) <= 0)


def test_permute_golden():
    g = load("permute_tiny.txt")
    idx = np.array(g["idx"]).reshape(g["T"], g["k"])
    row_map, split_sizes, offsets = moe.permute_index(idx, g["E"])
    assert list(row_map) == g["row_map"]
    assert list(split_sizes) == g["split_sizes"]
    assert list(offsets) == g["offsets"]


@pytest.mark.parametrize("T,E,k", [(1, 1, 1), (7, 3, 2), (64, 8, 2), (100, 16, 8), (33, 128, 8)])
def test_permute_invariants(T, E, k):
    rng = np.random.default_rng(T + E + k)
    lg = rng.normal(size=(T, E))
    lg[:, E // 2:] -= 50.0 if E > 2 * k else 0.0                 # some empty experts
    idx, _ = moe.route(lg, k)
    row_map, split_sizes, offsets = moe.permute_index(idx, E)
    R = T * k
    assert np.array_equal(np.sort(row_map), np.arange(R))           # bijection onto [0, R)
    assert np.array_equal(split_sizes, np.bincount(idx.reshape(-1), minlength=E))
    assert split_sizes.sum() == R and offsets[-1] == R and offsets[0] == 0
    flat = idx.reshape(-1)
    for s in range(R):                                              # row lies in its expert's range
        e = flat[s]
        assert offsets[e] <= row_map[s] < offsets[e + 1]
    for e in range(E):                                              # stable: ascending slot order
        slots = np.nonzero(flat == e)[0]
        assert np.all(np.diff(row_map[slots]) == 1)


@pytest.mark.parametrize("k", [1, 2, 8])
def test_unpermute_of_permute_is_identity(k):
    rng = np.random.default_rng(k)
    T, H, E = 50, 24, 9
    x = moe.round_to_bf16(rng.normal(size=(T, H)))   # 8 significant bits: partial sums exact
    idx, _ = moe.route(rng.normal(size=(T, E)), k)
    row_map, _, _ = moe.permute_index(idx, E)
    xp = moe.permute_rows(x, row_map, k)
    for t in range(T):
        for j in range(k):
            assert np.array_equal(xp[row_map[t * k + j]], x[t])
    w = np.full((T, k), 1.0 / k)                                    # power of two for k in {1,2,8}
    assert np.array_equal(moe.unpermute(xp, row_map, T, k, prob=w), x)
    assert np.array_equal(moe.unpermute(xp, row_map, T, k), k * x)


def test_permute_rejects_out_of_range():
    with pytest.raises(ValueError):
        moe.permute_index(np.array([[0, 3]]), 3)
