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


# ------------------------------------------------------------------ router backward
def _torch_route_grad(lg, idx, dprob, renorm):
    """dL/dlogits by torch fp64 autograd of softmax -> gather -> renormalise."""
    import torch
    lt = torch.tensor(lg, dtype=torch.float64, requires_grad=True)
    q = torch.gather(torch.softmax(lt, dim=1), 1, torch.tensor(idx, dtype=torch.int64))
    p = q / q.sum(dim=1, keepdim=True) if renorm else q
    (p * torch.tensor(dprob)).sum().backward()
    return lt.grad.numpy()


@pytest.mark.parametrize("renorm", [True, False])
@pytest.mark.parametrize("E,k", [(4, 1), (8, 2), (16, 5), (7, 7), (128, 8)])
def test_route_bwd_matches_torch_autograd(E, k, renorm):
    rng = np.random.default_rng(E + 100 * k)
    lg = rng.normal(size=(50, E)) * 2.0
    idx, _ = moe.route(lg, k, renorm)
    dprob = rng.normal(size=(50, k))
    got = moe.route_bwd(lg, idx, dprob, renorm)
    ref = _torch_route_grad(lg, idx, dprob, renorm)
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-14)


@pytest.mark.parametrize("renorm", [True, False])
def test_route_bwd_matches_finite_differences(renorm):
    # logits with gaps of at least 0.5 between sorted values: the selection does not
    # change under the perturbation, so the probabilities are smooth there
    rng = np.random.default_rng(7)
    T, E, k = 6, 9, 3
    lg = np.stack([rng.permutation(E) * 0.5 + rng.uniform(0, 0.1) for _ in range(T)])
    idx, _ = moe.route(lg, k, renorm)
    dprob = rng.normal(size=(T, k))
    got = moe.route_bwd(lg, idx, dprob, renorm)
    eps = 1e-6
    for t, b in [(0, 0), (1, 4), (3, 8), (5, 2), (2, 6)]:
        lp, lm = lg.copy(), lg.copy()
        lp[t, b] += eps
        lm[t, b] -= eps
        ip, pp = moe.route(lp, k, renorm)
        im, pm = moe.route(lm, k, renorm)
        assert np.array_equal(ip, idx) and np.array_equal(im, idx)
        fd = (np.sum(pp * dprob) - np.sum(pm * dprob)) / (2 * eps)
        assert abs(fd - got[t, b]) <= 1e-8 * max(1.0, abs(fd))


def test_route_bwd_invariants_and_special_cases():
    rng = np.random.default_rng(11)
    T, E, k = 40, 12, 4
    lg = rng.normal(size=(T, E))
    idx, prob = moe.route(lg, k, True)
    dprob = rng.normal(size=(T, k))
    # shifting every logit of a token leaves the probabilities unchanged: rows sum to 0
    for renorm in (True, False):
        g = moe.route_bwd(lg, idx, dprob, renorm)
        assert np.max(np.abs(g.sum(axis=1))) <= 1e-14
    # with renormalisation the probabilities are the softmax over the selected logits
    # only: no gradient reaches the others (zero up to fp64 rounding of <ds, s> = 0)
    g = moe.route_bwd(lg, idx, dprob, True)
    mask = np.ones((T, E), dtype=bool)
    mask[np.arange(T)[:, None], idx] = False
    assert np.max(np.abs(g[mask])) <= 1e-15
    # constant upstream gradient with renormalisation: sum_j p_j = 1, so dlogits = 0
    assert np.max(np.abs(moe.route_bwd(lg, idx, np.ones((T, k)), True))) <= 1e-15
    # k = E with renorm is the plain softmax: the textbook Jacobian p * (d - <d, p>)
    idx_all, p_all = moe.route(lg, E, True)
    d = rng.normal(size=(T, E))
    g = moe.route_bwd(lg, idx_all, d, True)
    ref = np.zeros((T, E))
    np.put_along_axis(ref, idx_all, p_all * (d - np.sum(d * p_all, axis=1, keepdims=True)), axis=1)
    np.testing.assert_allclose(g, ref, rtol=1e-12, atol=1e-15)
