"""Pins for the oracle's LRU refinement cache (CPU only).

The oracle implements the policy from its definition (victims sorted by
(last_use, unit) each step).  Here an independent brute force keeps an
``OrderedDict`` in recency order instead -- touched units moved to the end in
ascending unit order at the end of each step, victims taken from the front --
and must agree on hits, misses, bypass and slot placement.
"""

from collections import OrderedDict

import numpy as np
import pytest

from oracle.cache import LRUCache, effective_set


class OrderedLRU:
    def __init__(self, capacity):
        self.cap = capacity
        self.od = OrderedDict()       # unit -> slot, least recent first
        self.free = list(range(capacity))

    def step(self, S, budget=None):
        hits = [u for u in S if u in self.od]
        misses = [u for u in S if u not in self.od]
        late = [] if budget is None else misses[budget:]
        misses = misses if budget is None else misses[:budget]
        in_S = set(S)
        victims = [u for u in self.od if u not in in_S]     # recency order
        avail = [(s, None) for s in sorted(self.free)] + [(self.od[v], v) for v in victims]
        placed, bypass = [], []
        for i, u in enumerate(misses):
            if i < len(avail):
                slot, old = avail[i]
                if old is None:
                    self.free.remove(slot)
                else:
                    del self.od[old]
                self.od[u] = slot
                placed.append((u, slot))
            else:
                bypass.append(u)
        for u in sorted(hits + [u for u, _ in placed]):
            self.od.move_to_end(u)
        return hits, misses + late, bypass, placed


def _random_steps(seed, K, C, n_steps, k, hot):
    rng = np.random.default_rng(seed)
    hot_set = rng.choice(K, size=hot, replace=False)
    for _ in range(n_steps):
        rest = rng.choice(K, size=k, replace=False)
        yield sorted(set(hot_set.tolist()) | set(rest[:k - hot].tolist()))


@pytest.mark.parametrize("K,C,k,hot", [(512, 40, 30, 5), (256, 16, 24, 4), (128, 128, 20, 3), (64, 0, 8, 2)])
def test_against_ordered_dict(K, C, k, hot):
    a, b = LRUCache(K, C), OrderedLRU(C)
    for S in _random_steps(K + C, K, C, 60, k, hot):
        r = a.step(S)
        h, m, by, placed = b.step(S)
        assert r["hits"] == h and r["misses"] == m and r["bypass"] == by
        assert r["inserted"] == placed
        assert len(r["hits"]) + len(r["misses"]) == len(S)
        assert set(r["bypass"]) <= set(r["misses"])
        assert a.snapshot() == dict(b.od)
        assert len(a.snapshot()) <= C


def test_preloaded_all_hits():
    K = 512
    c = LRUCache(K, K)
    c.preload(range(K))
    for S in _random_steps(1, K, K, 10, 26, 5):
        r = c.step(S)
        assert r["hits"] == S and r["misses"] == [] and r["bypass"] == []
    assert c.snapshot() == {u: u for u in range(K)}


def test_by_hand():
    c = LRUCache(10, 3)
    r = c.step([1, 4, 7])            # cold: slots 0,1,2 in unit order
    assert r["inserted"] == [(1, 0), (4, 1), (7, 2)] and r["hits"] == []
    r = c.step([4, 8])               # 4 hits; 8 replaces the LRU unit not in S: (last 0, unit 1)
    assert r["hits"] == [4] and r["inserted"] == [(8, 0)]
    r = c.step([2, 3, 9])            # victims by (last_use, unit): 7 (t0), 4 (t1), 8 (t1)
    assert r["inserted"] == [(2, 2), (3, 1), (9, 0)] and r["bypass"] == []
    r = c.step([0, 1, 2, 5])         # capacity 3, |S| = 4: one hit (2), 2 slots for 3 misses
    assert r["hits"] == [2] and r["misses"] == [0, 1, 5]
    assert r["inserted"] == [(0, 1), (1, 0)] and r["bypass"] == [5]
    assert c.snapshot() == {0: 1, 1: 0, 2: 2}


def test_rejects_unsorted():
    c = LRUCache(10, 3)
    with pytest.raises(ValueError):
        c.step([3, 1])


@pytest.mark.parametrize("K,C,k,hot,budget", [(512, 40, 30, 5, 7), (256, 100, 24, 4, 0), (128, 16, 20, 3, 3),
                                              (300, 60, 25, 10, 1000)])
def test_fetch_budget_against_ordered_dict(K, C, k, hot, budget):
    """C7: with a per-step fetch budget only the first F misses (ascending)
    are fetched; the late ones are neither cached nor touched."""
    a, b = LRUCache(K, C), OrderedLRU(C)
    late_total = 0
    for S in _random_steps(K + C + 1, K, C, 60, k, hot):
        r = a.step(S, budget=budget)
        h, m, by, placed = b.step(S, budget=budget)
        assert r["hits"] == h and r["misses"] == m and r["bypass"] == by and r["inserted"] == placed
        assert r["late"] == r["misses"][min(len(r["misses"]), budget):]
        assert not set(r["late"]) & set(a.snapshot())
        late_total += len(r["late"])
        assert a.snapshot() == dict(b.od)
    assert a.late == late_total


def test_fetch_budget_by_hand():
    c = LRUCache(10, 3)
    r = c.step([1, 4, 7], budget=2)   # two fetched, 7 is late
    assert r["inserted"] == [(1, 0), (4, 1)] and r["late"] == [7]
    r = c.step([4, 7, 8], budget=1)   # 4 hits; 7 fetched into the free slot; 8 late
    assert r["hits"] == [4] and r["inserted"] == [(7, 2)] and r["late"] == [8]
    r = c.step([2, 3], budget=0)      # nothing fetched, nothing evicted
    assert r["inserted"] == [] and r["late"] == [2, 3]
    assert c.snapshot() == {1: 0, 4: 1, 7: 2}
    r = c.step([2, 3])                # no budget: C1-C5 (victims by (last use, unit): 1, then 4)
    assert r["inserted"] == [(2, 0), (3, 1)] and r["late"] == []


def test_effective_set_of_the_deadline_reading():
    """C8: the GEMV refines the selected units cached when the step starts;
    the step itself then runs on the whole selection."""
    c = LRUCache(20, 4)
    c.step([1, 2, 3])
    cached = c.snapshot()
    assert effective_set([2, 3, 5, 9], cached) == [2, 3]
    assert effective_set([], cached) == [] and effective_set([7], {}) == []
    r = c.step([2, 3, 5, 9])
    assert r["hits"] == [2, 3] and r["misses"] == [5, 9]
