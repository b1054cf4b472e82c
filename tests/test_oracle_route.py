"""Pins for the oracle's top-k routing and grouping (no GPU).

Brute force over every k-subset on tiny inputs, closed-form softmax values,
k = E reducing to a plain softmax, hand-made tie cases, and planted mistakes.
"""
import itertools
import math

import numpy as np
import pytest

from oracle import route


def _brute_force_set(l, k):
    """The unique k-subset whose smallest logit exceeds the largest unselected one."""
    E = len(l)
    found = []
    for s in itertools.combinations(range(E), k):
        rest = [l[i] for i in range(E) if i not in s]
        if not rest or min(l[i] for i in s) > max(rest):
            found.append(set(s))
    assert len(found) == 1
    return found[0]


@pytest.mark.parametrize("E,k", [(16, 4), (10, 3), (8, 8), (12, 1), (9, 5)])
def test_topk_matches_brute_force(E, k):
    rng = np.random.default_rng(E * 100 + k)
    for _ in range(20):
        l = rng.standard_normal((1, E)).astype(np.float32)
        idx, w = route.route(l, k)
        assert set(idx[0].tolist()) == _brute_force_set(l[0].tolist(), k)
        # slots are in descending logit order
        assert all(l[0, idx[0, j]] > l[0, idx[0, j + 1]] for j in range(k - 1))


def test_softmax_closed_form():
    l = np.array([[0.0, math.log(2.0), math.log(3.0)]])
    np.testing.assert_allclose(route.softmax(l), [[1 / 6, 2 / 6, 3 / 6]], rtol=1e-15)


def test_k_equals_E_is_full_softmax():
    l = np.random.default_rng(1).standard_normal((3, 7)).astype(np.float32)
    idx, w = route.route(l, 7)
    p = np.exp(l.astype(np.float64))
    p /= p.sum(axis=1, keepdims=True)
    np.testing.assert_allclose(w, np.take_along_axis(p, idx.astype(np.int64), axis=1), rtol=1e-14)


def test_weights_are_softmax_over_selected_and_sum_to_one():
    l = np.random.default_rng(2).standard_normal((5, 16)).astype(np.float32)
    idx, w = route.route(l, 4)
    np.testing.assert_allclose(w.sum(axis=1), 1.0, rtol=0, atol=1e-15)
    for t in range(5):
        s = l[t, idx[t]].astype(np.float64)
        ref = np.exp(s - s.max()) / np.exp(s - s.max()).sum()
        np.testing.assert_allclose(w[t], ref, rtol=1e-14)


def test_ties_go_to_lower_index():
    l = np.array([[1.0, 2.0, 2.0, 0.0]], dtype=np.float32)
    assert route.select_topk(l, 1).tolist() == [[1]]
    assert route.select_topk(l, 2).tolist() == [[1, 2]]
    l = np.array([[0.5, 0.5, 0.5, 0.5]], dtype=np.float32)
    assert route.select_topk(l, 3).tolist() == [[0, 1, 2]]
    idx, w = route.route(l, 3)
    np.testing.assert_allclose(w, [[1 / 3, 1 / 3, 1 / 3]], rtol=1e-15)


def test_large_logits_do_not_overflow():
    l = np.array([[1000.0, 999.0, -1000.0]], dtype=np.float32)
    idx, w = route.route(l, 2)
    assert idx.tolist() == [[0, 1]]
    e = math.exp(-1.0)
    np.testing.assert_allclose(w, [[1 / (1 + e), e / (1 + e)]], rtol=1e-15)


def test_group_by_expert():
    idx = np.array([[3, 0], [0, 2], [3, 1]], dtype=np.int32)
    cnt, off, perm = route.group_by_expert(idx, 5)
    assert cnt.tolist() == [2, 1, 1, 2, 0]
    assert off.tolist() == [0, 2, 3, 4, 6, 6]
    assert perm.tolist() == [1, 2, 5, 3, 0, 4]
    # every pair appears once and maps back to its expert
    flat = idx.reshape(-1)
    for e in range(5):
        assert all(flat[p] == e for p in perm[off[e]:off[e + 1]])
    assert sorted(perm.tolist()) == list(range(6))


def test_planted_reverse_order_is_caught(monkeypatch):
    orig = route.select_topk

    def ascending(l, k):
        return orig(l, k)[:, ::-1]
    monkeypatch.setattr(route, "select_topk", ascending)
    l = np.array([[0.1, 0.9, 0.5, 0.3]], dtype=np.float32)
    idx, _ = route.route(l, 2)
    assert idx.tolist() != [[1, 2]]


def test_planted_unnormalised_weights_are_caught():
    l = np.random.default_rng(3).standard_normal((2, 16)).astype(np.float32)
    idx = route.select_topk(l, 4)
    p = route.softmax(l)
    raw = np.take_along_axis(p, idx.astype(np.int64), axis=1)
    assert not np.allclose(raw.sum(axis=1), 1.0)     # the renormalisation is load-bearing


def test_router_logits_hand_case():
    """x = [[1, 2], [-1, 0.5]], Wr rows [1, 0], [0.5, -1], [0.25, 0.25]:
    logits row 0 = [1, 0.5 - 2, 0.25 + 0.5] = [1, -1.5, 0.75],
    row 1 = [-1, -0.5 - 0.5, -0.25 + 0.125] = [-1, -1, -0.125]."""
    from oracle.route import router_logits
    x = np.array([[1.0, 2.0], [-1.0, 0.5]])
    wr = np.array([[1.0, 0.0], [0.5, -1.0], [0.25, 0.25]])
    np.testing.assert_array_equal(router_logits(x, wr), [[1.0, -1.5, 0.75], [-1.0, -1.0, -0.125]])
    idx, _ = route.route(router_logits(x, wr), 2)
    np.testing.assert_array_equal(idx, [[0, 2], [2, 0]])   # row 1: tie of -1 to the lower index


def test_near_ties_flags_the_boundary():
    from oracle.route import near_ties
    l = np.array([[3.0, 1.0, 1.0 + 1e-9, 0.0], [3.0, 2.0, 1.0, 0.0]])
    np.testing.assert_array_equal(near_ties(l, 2, 1e-6), [True, False])
    np.testing.assert_array_equal(near_ties(l, 4, 1e-6), [False, False])
