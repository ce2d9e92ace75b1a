"""Pins of the oracle's hot-pool residency (CPU only).

The pages say only that predicted blocks are kept in GPU memory and fetched from the CPU
cold pool; the policy (keep resident rows, evict the least recently needed) is this
build's reading.  The oracle is pinned by a hand trace, by reduction to a textbook LRU
cache when every trigger wants a single entry, and by invariants on random traces."""
import collections
import json
import os

import numpy as np
import pytest

from oracle import lsa_oracle as O

HERE = os.path.dirname(os.path.abspath(__file__))


def test_hand_trace():
    d = json.load(open(os.path.join(HERE, "golden", "hot_pool_trace.json")))
    hp = O.HotPool(d["N"], d["slots"])
    for tr in d["triggers"]:
        moves = hp.update(tr["U"], tr["t"])
        exp = None if tr["moves"] is None else [tuple(m) for m in tr["moves"]]
        assert moves == exp, tr["t"]
    resident = {e: s for e, s in enumerate(hp.slot_of) if s >= 0}
    assert resident == {int(k): v for k, v in d["final_slot_of"].items()}


@pytest.mark.parametrize("slots", [1, 3, 8])
def test_single_entry_triggers_are_a_textbook_lru_cache(slots):
    """With one entry per trigger the pool is an LRU cache of `slots` lines: the
    resident set and the misses must match collections.OrderedDict's LRU."""
    g = np.random.default_rng(slots)
    N = 20
    hp = O.HotPool(N, slots)
    lru = collections.OrderedDict()
    for t, e in enumerate(g.integers(0, N, size=400), start=1):
        e = int(e)
        moves = hp.update([e], t)
        if e in lru:
            lru.move_to_end(e)
            assert moves == []
        else:
            if len(lru) == slots:
                lru.popitem(last=False)
            lru[e] = True
            assert [m[0] for m in moves] == [e]
        assert {x for x in range(N) if hp.slot_of[x] >= 0} == set(lru)


def test_invariants_on_random_traces():
    g = np.random.default_rng(5)
    N, slots, R = 200, 60, 4
    cold = g.integers(0, 256, size=(N, R))
    hot = np.zeros((slots, R), dtype=cold.dtype)
    hp = O.HotPool(N, slots)
    prev = set()
    for t in range(1, 80):
        U = set(int(x) for x in g.choice(N, size=int(g.integers(0, 70)), replace=False))
        resident_before = {e for e in range(N) if hp.slot_of[e] >= 0}
        moves = hp.update(U, t, cold, hot)
        if len(U) > slots:
            assert moves is None
            continue
        assert sorted(m[0] for m in moves) == sorted(U - resident_before)     # only missing rows move
        for e in U:
            assert hp.slot_of[e] >= 0                                          # the fetch set is resident
        for s in range(slots):
            e = hp.entry_of[s]
            if e >= 0:
                assert hp.slot_of[e] == s and np.array_equal(hot[s], cold[e])  # maps are inverse, rows intact
        assert sum(1 for e in range(N) if hp.slot_of[e] >= 0) == sum(1 for s in range(slots) if hp.entry_of[s] >= 0)
        prev = U
    assert prev is not None
