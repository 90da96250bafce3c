"""Pins of the oracle's group-limited top-k routing: a numpy restatement with
stable sorts (ties to the lower index), brute force over every subset of
groups on small cases, the special case of one group (plain top-k), and
the softmax against scipy in float64."""

import itertools

import numpy as np
import pytest
from scipy.special import softmax

import oracle


def numpy_route(scores, k, n_groups, topk_groups):
    T, E = scores.shape
    per = E // n_groups
    gscore = scores.reshape(T, n_groups, per).max(axis=2)
    # descending, ties to the lower index: stable sort of the negated scores
    groups = np.argsort(-gscore, axis=1, kind="stable")[:, :topk_groups]
    allowed = np.zeros((T, n_groups), bool)
    np.put_along_axis(allowed, groups, True, axis=1)
    masked = np.where(np.repeat(allowed, per, axis=1), scores, -np.inf)
    idx = np.argsort(-masked, axis=1, kind="stable")[:, :k]
    sel = np.take_along_axis(scores, idx, axis=1).astype(np.float64)
    return idx, softmax(sel, axis=1)


@pytest.mark.parametrize("T,E,k,ng,tg", [(200, 256, 8, 8, 4), (100, 64, 6, 4, 2), (50, 16, 3, 1, 1),
                                         (50, 12, 12, 3, 3), (30, 32, 1, 8, 1)])
def test_router_matches_numpy_restatement(T, E, k, ng, tg):
    rng = np.random.default_rng(T + E)
    scores = rng.standard_normal((T, E)).astype(np.float32)
    scores[: T // 2] = np.round(scores[: T // 2] * 2) / 2  # many exact ties
    idx, w = oracle.route_group_limited(scores, k, ng, tg)
    ridx, rw = numpy_route(scores, k, ng, tg)
    assert np.array_equal(idx, ridx)
    assert np.allclose(w, rw, rtol=1e-6, atol=0)
    assert np.allclose(w.sum(1), 1.0, atol=1e-6)


def test_router_brute_force_group_choice():
    """The kept groups maximise the sum of group maxima over all subsets of
    that size (distinct scores), and the experts are the k best inside them."""
    rng = np.random.default_rng(1)
    E, ng, tg, k = 12, 4, 2, 3
    per = E // ng
    for _ in range(200):
        s = rng.permutation(E).astype(np.float32)  # distinct
        idx, _ = oracle.route_group_limited(s[None, :], k, ng, tg)
        gmax = s.reshape(ng, per).max(1)
        best = max(itertools.combinations(range(ng), tg), key=lambda c: sorted(gmax[list(c)], reverse=True))
        cand = [e for e in range(E) if e // per in best]
        expect = sorted(cand, key=lambda e: -s[e])[:k]
        assert list(idx[0]) == expect


def test_router_one_group_is_plain_topk():
    rng = np.random.default_rng(2)
    s = rng.standard_normal((40, 32)).astype(np.float32)
    idx, w = oracle.route_group_limited(s, 5, 1, 1)
    assert np.array_equal(idx, np.argsort(-s, axis=1, kind="stable")[:, :5])


def test_router_rejects_bad_arguments():
    s = np.zeros((2, 16), np.float32)
    for args in ((4, 3, 2), (4, 4, 5), (9, 4, 2), (0, 4, 2)):
        with pytest.raises(ValueError):
            oracle.route_group_limited(s, *args)
