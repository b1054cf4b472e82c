"""The expert cache's policy without a GPU (hfq_cache with no device tables
keeps the bookkeeping only): a hand-worked sequence of observations, and
invariants on a long skewed stream of routings (Strata report, "model and
engine": a VRAM cache of hot experts in front of the pinned host arena)."""
import numpy as np
import pytest

import expert_offload_b200 as eo


@pytest.fixture(scope="module", autouse=True)
def built():
    from expert_offload_b200 import build
    build.build()


def _cache(L, E, slots, home_loc):
    home_loc = np.asarray(home_loc, np.uint8).reshape(L, E)
    home = np.arange(L * E, dtype=np.uint64).reshape(L, E) * 4096 + 0x10000
    host_src = np.where(home_loc == 1, home + 0x100000000, 0).astype(np.uint64)
    return eo.ExpertCache(L, E, 4096, slots, home, host_src, home_loc)


def _slots(c, E):
    return [c.slot_of(0, e) for e in range(E)]


def test_hand_worked_sequence():
    """One layer, 6 host experts, 2 slots.  Frequencies count selections;
    ties go to the lower expert id, for admission and for eviction alike."""
    c = _cache(1, 6, 2, [1] * 6)
    c.observe(0, [0, 1], 2)           # two misses, two free slots
    assert _slots(c, 6) == [0, 1, -1, -1, -1, -1]
    c.observe(0, [2], 1)              # e2 (freq 1) is not more frequent than e0 (1): stays out
    assert _slots(c, 6) == [0, 1, -1, -1, -1, -1]
    c.observe(0, [2], 1)              # e2 (2) > e0 (1, the lower of the two least frequent)
    assert _slots(c, 6) == [-1, 1, 0, -1, -1, -1]
    c.observe(0, [1, 3], 2)           # e1 hits; e3 (1) does not beat e2 (2)
    assert _slots(c, 6) == [-1, 1, 0, -1, -1, -1]
    # staging before use (max_admit = -1): every selected miss gets a slot,
    # evicting the cached experts not selected now (least frequent, lower id first)
    c.observe(0, [4, 5], -1)
    assert _slots(c, 6) == [-1, -1, -1, -1, 1, 0]      # e4 into e1's slot, then e5 into e2's
    st = c.stats()
    # hits: e1 once; misses: e0 e1 e2 e2 e3 e4 e5
    assert (st["hits"], st["misses"], st["admitted"], st["evicted"]) == (1, 7, 5, 3)
    c.close()


def test_resident_experts_are_hits_and_never_cached():
    c = _cache(1, 4, 2, [0, 1, 0, 1])
    c.observe(0, [0, 1, 2, 3], 4)
    assert c.slot_of(0, 0) == -1 and c.slot_of(0, 2) == -1
    assert c.slot_of(0, 1) >= 0 and c.slot_of(0, 3) >= 0
    assert c.stats()["hits"] == 2 and c.stats()["misses"] == 2
    c.observe(0, [0, 1, 2, 3], 4)
    assert c.stats()["hits"] == 6
    c.close()


def test_staging_fits_every_selection_of_a_token():
    c = _cache(2, 64, 8, [1] * 128)
    rng = np.random.default_rng(3)
    for _ in range(50):
        for l in range(2):
            ids = rng.choice(64, 8, replace=False)
            c.observe(l, ids, -1)
            assert all(c.slot_of(l, int(e)) >= 0 for e in ids)
    c.close()


def test_skewed_stream_converges_to_the_hot_set():
    """Routing skewed like the verify workload (51 of 512 experts take about
    60 % of top-8 selections): with 51 slots and at most 2 admissions per
    step, the cache ends up holding mostly hot experts and hits well above
    the 10 % a random set would get; slots never hold an expert twice."""
    from synth import workloads as W
    w = W.WORKLOADS[3]
    E, k, slots = w.experts, w.top_k, 51
    c = _cache(1, E, slots, [1] * E)
    logits = W.logits(w, 0, 1000, 1500)
    top = np.argpartition(-logits, k - 1, axis=1)[:, :k]
    for t in range(1000):
        c.observe(0, top[t], 2)
    before = c.stats()
    for t in range(1000, 1500):
        c.observe(0, top[t], 2)
    after = c.stats()
    hit_rate = (after["hits"] - before["hits"]) / (
        after["hits"] - before["hits"] + after["misses"] - before["misses"])
    cached = [e for e in range(E) if c.slot_of(0, e) >= 0]
    slots_used = [c.slot_of(0, e) for e in cached]
    assert len(set(slots_used)) == len(slots_used) == slots
    hot = set(W.hot_set(w, 0).tolist())
    assert len(hot & set(cached)) >= 40
    assert hit_rate > 0.45, hit_rate
    assert after["admitted"] <= 2 * 1500
    c.close()


def test_bad_ids_are_refused():
    c = _cache(1, 8, 2, [1] * 8)
    with pytest.raises(eo.HfqError) as e:
        c.observe(0, [3, 9], 1)
    assert e.value.status == -1
    c.close()


def test_flush_without_device_tables_is_a_no_op():
    c = _cache(1, 4, 2, [1] * 4)
    c.observe(0, [0, 1], 2)
    c.flush()
    assert c.slot_of(0, 0) >= 0 and c.slot_of(0, 1) >= 0
    c.close()
