"""LRU refinement cache (oracle; test infrastructure).

StrataFlux caches fetched precision on the GPU and reuses it across decode
steps (arXiv 2611.08363 abstract; rag-lover.com explainer, TL;DR and 解説
sections).  The pages give no policy, so this module takes an LRU reading.
One cache per weight matrix holds up to C units (a unit is one input
column's refinement bits).  At step t, given the ascending selected set S:

C1  hits H = S ∩ cached; misses M = S \\ H.
C2  every hit gets last_use = t.
C3  slots for misses come first from free slots, lowest slot index first,
    then from victims: cached units not in S, ordered by (last_use
    ascending, unit ascending).
C4  misses take those slots in ascending unit order until none are left; the
    misses left over form the bypass set: fetched for this step only, never
    cached.
C5  every inserted unit gets last_use = t; then t advances by one.
C6  for weights the correction always uses all of S (every fetch completes
    before use), so the GEMV result does not depend on cache state; what is
    compared is the hit / miss / bypass sets and the slot each unit lands in.
C7  a fetch budget F (the deadline reading, for caches whose consumer does
    not wait for the fetch): only the first F misses in ascending unit order
    are fetched and go through C4; the misses after them are *late* --
    neither fetched nor cached nor touched, so their precision stays the
    resident one (a miss keeps resident precision: rag-lover.com explainer,
    限界と未検証の範囲).  No budget (F = None) is C1-C5 unchanged.
C8  the deadline reading of a weight matrix's cache (its GEMV does not wait
    for the fetch of its own selection): the GEMV refines E = S ∩ (units
    cached when the step starts), :func:`effective_set`; then the step runs
    as above on S, so the misses are fetched for later steps.  C6 then holds
    with E in place of S.

``preload`` fills an empty cache with the given units in slots 0, 1, ...
with last_use = -1 (older than any step), and counts nothing.
"""

from __future__ import annotations


class LRUCache:
    def __init__(self, num_units: int, capacity: int):
        if capacity < 0 or num_units < 0:
            raise ValueError("negative size")
        self.num_units = num_units
        self.capacity = capacity
        self.slot_of: dict[int, int] = {}
        self.last_use: dict[int, int] = {}
        self.free: list[int] = list(range(capacity))
        self.t = 0
        self.hits = self.misses = self.bypass = self.late = 0

    def preload(self, units) -> None:
        units = list(units)
        if self.slot_of or len(units) > self.capacity or len(set(units)) != len(units):
            raise ValueError("preload needs an empty cache and at most C distinct units")
        for u in units:
            if not 0 <= u < self.num_units:
                raise ValueError("unit out of range")
            slot = self.free.pop(0)
            self.slot_of[u] = slot
            self.last_use[u] = -1

    def step(self, S, budget: int | None = None) -> dict:
        S = [int(u) for u in S]
        if S != sorted(set(S)):
            raise ValueError("S must be strictly ascending")
        t = self.t
        in_S = set(S)
        H = [u for u in S if u in self.slot_of]                       # C1
        M = [u for u in S if u not in self.slot_of]
        if budget is not None and budget < 0:
            raise ValueError("negative budget")
        nf = len(M) if budget is None else min(len(M), budget)        # C7
        fetched, late = M[:nf], M[nf:]
        for u in H:                                                    # C2
            self.last_use[u] = t
        victims = sorted((u for u in self.slot_of if u not in in_S),  # C3
                         key=lambda u: (self.last_use[u], u))
        free_sorted = sorted(self.free)
        avail = [("free", s, None) for s in free_sorted] + [("victim", self.slot_of[v], v) for v in victims]
        inserted, bypass = [], []
        for i, u in enumerate(fetched):                                # C4
            if i >= len(avail):
                bypass.append(u)
                continue
            kind, slot, old = avail[i]
            if kind == "victim":
                del self.slot_of[old]
                del self.last_use[old]
            else:
                self.free.remove(slot)
            self.slot_of[u] = slot
            self.last_use[u] = t                                       # C5
            inserted.append((u, slot))
        self.t = t + 1
        self.hits += len(H)
        self.misses += len(M)
        self.bypass += len(bypass)
        self.late += len(late)
        return dict(hits=H, misses=M, bypass=bypass, late=late, inserted=inserted)

    def snapshot(self) -> dict[int, int]:
        """unit -> slot for every cached unit."""
        return dict(self.slot_of)


def effective_set(S, cached) -> list[int]:
    """C8: the selected units that were cached when the step started
    (``cached``: a set or dict of units), ascending."""
    return [int(u) for u in S if int(u) in cached]
