"""Pins for the oracle's expert placement (no GPU).

Brute force over every split on tiny models, hand-made hot-set ties, the
refusal with its byte deficit, and slot numbering.
"""
import numpy as np

from oracle import placement as P


def test_manual_layer_split_without_hot_set():
    counts = np.zeros((4, 3), dtype=np.uint32)
    p = P.place(counts, 100, 1, 0, 10**9)
    assert p.ok and p.resident_layers == 1
    assert p.loc.tolist() == [[0, 0, 0], [1, 1, 1], [1, 1, 1], [1, 1, 1]]
    assert p.slot.tolist() == [[0, 1, 2], [0, 1, 2], [3, 4, 5], [6, 7, 8]]
    assert p.hbm_needed == 300 and p.host_needed == 900


def test_hot_set_ranks_by_count_then_index():
    counts = np.array([[5, 9, 9, 1, 7]], dtype=np.uint32)
    assert P.hot_experts(counts[0], 2).tolist() == [1, 2]
    assert P.hot_experts(counts[0], 3).tolist() == [1, 2, 4]
    counts = np.array([[3, 3, 3, 3]], dtype=np.uint32)
    assert P.hot_experts(counts[0], 2).tolist() == [0, 1]
    p = P.place(np.array([[5, 9, 9, 1, 7]], np.uint32), 10, 0, 2, 10**6)
    assert p.loc.tolist() == [[1, 0, 0, 1, 1]]


def test_auto_is_largest_fitting_split_brute_force():
    rng = np.random.default_rng(0)
    for L, E in [(3, 4), (5, 2), (4, 6)]:
        counts = rng.integers(0, 50, (L, E)).astype(np.uint32)
        eb = 7
        for h in range(0, E + 1):
            for budget in range(0, L * E * eb + 10, 5):
                p = P.place(counts, eb, -1, h, budget)
                fits = [n for n in range(L + 1) if (n * E + (L - n) * h) * eb <= budget]
                if not fits:
                    assert not p.ok and p.deficit == (L * h) * eb - budget
                else:
                    assert p.ok and p.resident_layers == max(fits)
                    assert p.hbm_needed == (max(fits) * E + (L - max(fits)) * h) * eb
                    assert int((p.loc == 0).sum()) * eb == p.hbm_needed


def test_refusal_names_the_deficit():
    counts = np.zeros((48, 512), dtype=np.uint32)
    eb = 1_671_168
    p = P.place(counts, eb, 48, 0, 30 * 2**30)
    assert not p.ok
    assert p.hbm_needed == 48 * 512 * eb
    assert p.deficit == 48 * 512 * eb - 30 * 2**30


def test_slots_are_dense_per_location():
    counts = np.random.default_rng(1).integers(0, 9, (6, 8)).astype(np.uint32)
    p = P.place(counts, 3, 2, 3, 10**9)
    for where in (0, 1):
        s = sorted(p.slot[p.loc == where].tolist())
        assert s == list(range(len(s)))


def test_hand_worked_auto_placement_of_the_explainers_40_layer_model():
    """tests/golden/placement_auto.txt: the 40-layer, 408 MiB-per-layer model
    of the explainer's measurements, worked out by hand (auto with and without
    hot sets, and both refusals)."""
    from tests.golden_io import load_placement_cases
    L, E, eb = 40, 256, 1_671_168
    counts = np.tile(np.arange(E, dtype=np.uint32), (L, 1))      # c[l][e] = e
    cases = load_placement_cases()
    assert len(cases) == 4
    for c in cases:
        p = P.place(counts, eb, c["resident"], c["hot"], c["budget"])
        assert p.ok == c["ok"], c["name"]
        assert p.resident_layers == c["N"], c["name"]
        assert (p.hbm_needed, p.host_needed, p.deficit) == (c["hbm"], c["host"], c["deficit"]), c["name"]
        if c["ok"]:
            N, h = c["N"], c["hot"]
            assert np.all(p.loc[:N] == P.HBM)
            for l in range(N, L):
                assert np.nonzero(p.loc[l] == P.HBM)[0].tolist() == list(range(E - h, E))
