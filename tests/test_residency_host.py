"""Host logic of the hot-set policy: plan_swaps puts the n_hot most used
entries into the hot slots with disjoint exchanges that keep the table a
permutation, stops once nothing is left to trade, and raises the hit rate
of a drifting routing stream."""
import numpy as np
import pytest

from bit_expert_ffn_router_b200 import residency as R


def _table(rng, n_entries, n_slots):
    return rng.permutation(n_slots)[:n_entries].astype(np.int32)


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_plan_swaps_brings_the_most_used_into_hot_slots(seed):
    rng = np.random.default_rng(seed)
    n, n_hot = 600, 100
    slot_of = _table(rng, n, n)
    counts = rng.zipf(1.3, size=n) % 1000
    counts[rng.choice(n, 40, replace=False)] = 7  # many ties
    a, b = R.plan_swaps(counts, slot_of, n_hot)
    both = np.concatenate([a, b])
    assert np.unique(both).size == both.size  # disjoint exchanges
    after = R.apply_swaps(slot_of, a, b)
    assert sorted(after) == sorted(slot_of)  # still a permutation of the same slots
    hot = after < n_hot
    assert counts[~hot].max() <= counts[hot].min()  # no colder entry is used more than a hot one
    assert (after[a] < n_hot).all() and (after[b] >= n_hot).all()
    assert (counts[a] > counts[b]).all()  # every exchange is a strict gain
    a2, b2 = R.plan_swaps(counts, after, n_hot)
    assert a2.size == 0 and b2.size == 0  # nothing left to trade


def test_plan_swaps_ties_go_to_the_lower_entry_and_max_swaps():
    slot_of = np.arange(8, dtype=np.int32)[::-1].copy()  # entry i in slot 7 - i
    counts = np.array([5, 5, 5, 5, 0, 0, 0, 0])
    a, b = R.plan_swaps(counts, slot_of, 2)
    # wanted: entries 0 and 1 (ties to the lower index); the hot slots 0, 1 hold entries 7, 6
    assert list(a) == [0, 1] and sorted(b) == [6, 7]
    a1, b1 = R.plan_swaps(counts, slot_of, 2, max_swaps=1)
    assert list(a1) == [0] and b1.size == 1


def test_a_seeded_hot_set_stays_until_usage_beats_it():
    slot_of = np.arange(6, dtype=np.int32)
    counts = np.array([0, 0, 3, 0, 0, 0])  # hot slots 0, 1 hold unused entries 0, 1
    a, b = R.plan_swaps(counts, slot_of, 2)
    assert list(a) == [2] and list(b) == [1]  # only the used newcomer comes in (entry 0 wins the tie)
    a, b = R.plan_swaps(np.zeros(6, dtype=np.int64), slot_of, 2)
    assert a.size == 0  # no usage: the seeded set stays


def test_adapting_the_hot_set_raises_the_hit_rate_under_drift():
    rng = np.random.default_rng(5)
    L, E, k, n_hot = 4, 64, 4, 4 * 16
    slot_of = _table(rng, L * E, L * E)
    pop = [rng.permutation(E) for _ in range(L)]  # popularity order per layer, which drifts below
    def draw(step):
        out = []
        for l in range(L):
            shift = step // 20  # the favourites move every 20 steps
            ranks = np.minimum(rng.zipf(1.5, size=k) - 1, E - 1)
            out.append(pop[l][(ranks + shift) % E])
        return out
    static = slot_of.copy()
    adaptive = slot_of.copy()
    counts = np.zeros(L * E, dtype=np.int64)
    hs = ha = 0.0
    for step in range(200):
        ex = draw(step)
        hs += R.hot_hit_rate(ex, static, E, n_hot)
        ha += R.hot_hit_rate(ex, adaptive, E, n_hot)
        counts = counts * 0.9
        for l, e in enumerate(ex):
            np.add.at(counts, l * E + e, 1.0)
        if step % 10 == 9:
            a, b = R.plan_swaps(np.round(counts * 1000).astype(np.int64), adaptive, n_hot)
            adaptive = R.apply_swaps(adaptive, a, b)
    assert ha / 200 > hs / 200 + 0.2
