"""Pins of oracle/cache.py: q* against the pages' profiles and its closed
form, the LRU against a textbook move-to-front list, Belady's bound, a
hand-worked sequence and the capacity special cases."""
from collections import OrderedDict
from fractions import Fraction

import numpy as np
import pytest

from oracle import cache
from oracle.cache import DECODE, HIT, PREFILL, STAGED, STREAMED
from conftest import read_golden


def test_qstar_table_from_page_profiles():
    rows = [tuple(int(v) for v in r.split()) for r in read_golden("qstar_profiles.txt")]
    assert len(rows) == 18
    for bp, bh, m, q in rows:
        assert cache.qstar(m, bp, bh) == q, (bp, bh, m)


def test_qstar_within_half_of_ratio_and_monotone():
    rng = np.random.default_rng(0)
    for _ in range(3000):
        bh = int(rng.integers(1, 200000))
        bp = int(rng.integers(0, bh + 1))
        m = int(rng.integers(0, 300))
        q = cache.qstar(m, bp, bh)
        exact = Fraction(m * bp, bh)
        assert abs(Fraction(q) - exact) <= Fraction(1, 2)
        if abs(Fraction(q) - exact) == Fraction(1, 2):
            assert Fraction(q) > exact  # halves round up
        assert cache.qstar(m + 1, bp, bh) >= q
    for m in range(0, 50):
        assert cache.qstar(m, 0, 77300) == 0
        assert cache.qstar(m, 77300, 77300) == m
        assert cache.qstar(m, 90000, 77300) == m


def _single_access_trace(n, keys, rng, skew=1.2):
    w = np.arange(1, keys + 1, dtype=float) ** -skew
    return rng.choice(keys, size=n, p=w / w.sum())


def _run_ours(trace, L, E, C):
    c = cache.ExpertCache(L, E, C, 1, 1)
    out = []
    for key in trace:
        layer, e = divmod(int(key), E)
        counts = np.zeros(E, int); counts[e] = 1
        rec = c.forward(layer, DECODE, counts)
        out.append(rec["kinds"][e])
    return out, c


@pytest.mark.parametrize("C", [1, 3, 7, 20])
def test_single_access_equals_textbook_lru(C):
    L, E = 3, 8
    rng = np.random.default_rng(C)
    trace = _single_access_trace(2000, L * E, rng)
    ours, _ = _run_ours(trace, L, E, C)
    lru = OrderedDict()
    ref = []
    for key in trace:
        key = int(key)
        if key in lru:
            lru.move_to_end(key)
            ref.append(HIT)
        else:
            if len(lru) >= C:
                lru.popitem(last=False)
            lru[key] = True
            ref.append(STAGED)
    assert ours == ref


def _belady_misses(trace, C):
    cached = set()
    misses = 0
    for i, key in enumerate(trace):
        if key in cached:
            continue
        misses += 1
        if len(cached) >= C:
            def next_use(k):
                for j in range(i + 1, len(trace)):
                    if trace[j] == k:
                        return j
                return len(trace) + 1
            cached.remove(max(cached, key=next_use))
        cached.add(key)
    return misses


@pytest.mark.parametrize("C", [2, 5, 9])
def test_misses_not_below_belady_optimum(C):
    L, E = 2, 8
    trace = [int(k) for k in _single_access_trace(600, L * E, np.random.default_rng(10 + C))]
    ours, _ = _run_ours(trace, L, E, C)
    assert sum(1 for o in ours if o != HIT) >= _belady_misses(trace, C)


def test_full_capacity_has_only_compulsory_misses():
    L, E, k = 3, 16, 4
    c = cache.ExpertCache(L, E, L * E, 52700, 77300)
    rng = np.random.default_rng(11)
    seen = set()
    staged_total = 0
    for step in range(60):
        for layer in range(L):
            counts = np.zeros(E, int)
            counts[rng.choice(E, k, replace=False)] = 1
            rec = c.forward(layer, DECODE, counts)
            for e, kind in rec["kinds"].items():
                key = layer * E + e
                assert (kind == HIT) == (key in seen)
                seen.add(key) if kind == STAGED else None
            staged_total += rec["qstage"]
    # with q* < m some misses are streamed and seen later again as misses,
    # so count first touches only when everything is staged:
    c2 = cache.ExpertCache(L, E, L * E, 1, 1)
    keys = set()
    rng = np.random.default_rng(12)
    for step in range(60):
        for layer in range(L):
            counts = np.zeros(E, int)
            chosen = rng.choice(E, k, replace=False)
            counts[chosen] = 1
            c2.forward(layer, DECODE, counts)
            keys.update(layer * E + int(e) for e in chosen)
    assert c2.n["misses"] == len(keys)


def test_zero_capacity_streams_everything():
    c = cache.ExpertCache(2, 8, 0, 52700, 77300)
    for step in range(10):
        counts = np.zeros(8, int); counts[[1, 3, 6]] = 2
        rec = c.forward(step % 2, DECODE, counts)
        assert all(k == STREAMED for k in rec["kinds"].values())
        assert rec["qstage"] == 0 and rec["m"] == 3
    assert c.n["hits"] == 0 and c.n["staged"] == 0 and c.n["streamed"] == 30


def test_hand_worked_sequence():
    c = cache.ExpertCache(2, 4, 3)
    code = {"H": HIT, "S": STAGED, "R": STREAMED}
    for row in read_golden("lru_worked_example.txt"):
        head, bw, kinds, keys = (p.strip() for p in row.split("|"))
        layer, experts = head.split()
        experts = [int(e) for e in experts.split(",")]
        c.bp, c.bh = (int(v) for v in bw.split())
        counts = np.zeros(4, int); counts[experts] = 1
        rec = c.forward(int(layer), DECODE, counts)
        assert [rec["kinds"][e] for e in experts] == [code[k] for k in kinds.split(",")], row
        assert c.key_of == [int(v) for v in keys.split(",")], row


def test_prefill_double_buffer_loads_next_layer():
    L, E = 4, 8
    c = cache.ExpertCache(L, E, 2 * E)
    full = np.ones(E, int)
    rec = c.forward(0, PREFILL, full)
    assert len(rec["lookups"]) == 2 * E and rec["n_cur"] == E
    assert all(c.slot_of.get(k) is not None for k in range(0, 2 * E))
    for layer in range(1, L):
        rec = c.forward(layer, PREFILL, full)
        assert rec["n_cur"] == 0  # already prefetched by the previous call
        nxt = layer + 1
        if nxt < L:
            assert [lk[0] for lk in rec["lookups"]] == [nxt] * E
            assert all(k == STAGED for _, _, k in rec["lookups"])
            # exactly layers `layer` and `layer+1` are resident with C = 2E
            assert sorted(c.slot_of) == list(range(layer * E, (layer + 2) * E))
        else:
            assert rec["lookups"] == []
    assert c.n["misses"] == L * E and c.n["hits"] == 0


def test_prefill_with_small_cache_follows_decode_rules():
    E = 8
    c = cache.ExpertCache(2, E, E, 1, 2)
    counts = np.zeros(E, int); counts[[0, 2, 4, 6]] = 5
    rec = c.forward(0, PREFILL, counts)
    assert rec["m"] == 4 and rec["qstar"] == 2 and rec["qstage"] == 2
    assert [rec["kinds"][e] for e in (0, 2, 4, 6)] == [STAGED, STAGED, STREAMED, STREAMED]


def test_empty_call_changes_nothing():
    c = cache.ExpertCache(1, 4, 2)
    rec = c.forward(0, DECODE, np.zeros(4, int))
    assert rec["lookups"] == [] and c.n["layer_calls"] == 0 and c.clock == 0


@pytest.mark.parametrize("schedule", [(7, 3, 12, 5), (20, 1, 20), (4, 4, 9, 0, 6)])
def test_resize_equals_truncated_textbook_lru(schedule):
    """Elastic capacity: with one access per step, running segments of a trace
    at capacities C_0, C_1, ... with a resize between them gives the same
    hit/miss sequence as a move-to-front list that, on a shrink, drops its
    least recently used entries down to the new capacity."""
    L, E = 3, 8
    rng = np.random.default_rng(sum(schedule))
    segs = [[int(k) for k in _single_access_trace(300, L * E, rng)] for _ in schedule]
    c = cache.ExpertCache(L, E, schedule[0], 1, 1)
    lru = OrderedDict()
    for i, (C, seg) in enumerate(zip(schedule, segs)):
        if i:
            before = dict(zip(*c.contents()))
            old_slot = {k: s for s, k in enumerate(c.contents()[0]) if k >= 0}
            c.resize(C)
            while len(lru) > C:
                lru.popitem(last=False)
            key_of, stamp = c.contents()
            assert len(key_of) == C
            assert sorted(k for k in key_of if k >= 0) == sorted(lru)
            for s, k in enumerate(key_of):
                if k < 0:
                    assert stamp[s] == 0
                    continue
                assert stamp[s] == before[k]                # stamps survive
                if old_slot[k] < C:
                    assert s == old_slot[k]                 # no needless move
        for key in seg:
            layer, e = divmod(key, E)
            counts = np.zeros(E, int); counts[e] = 1
            kind = c.forward(layer, DECODE, counts)["kinds"][e]
            if key in lru:
                lru.move_to_end(key)
                assert kind == HIT
            else:
                assert kind == (STAGED if C > 0 else STREAMED)
                if C > 0:
                    if len(lru) >= C:
                        lru.popitem(last=False)
                    lru[key] = True


def test_resize_moves_survivors_to_lowest_free_slots():
    """Hand-worked shrink: 6 slots holding keys 10..15 with stamps
    [5, 1, 6, 2, 4, 3] (slot 0..5) shrunk to 3 keeps the three most recent,
    keys 12 (stamp 6, slot 2), 10 (stamp 5, slot 0) and 14 (stamp 4, slot 4);
    12 and 10 stay, 14 moves to the only free slot below 3, slot 1."""
    c = cache.ExpertCache(1, 16, 6)
    c.key_of = [10, 11, 12, 13, 14, 15]
    c.stamp = [5, 1, 6, 2, 4, 3]
    c.slot_of = {k: s for s, k in enumerate(c.key_of)}
    c.clock = 6
    c.resize(3)
    assert c.contents() == ([10, 14, 12], [5, 4, 6])
    assert c.slot_of == {10: 0, 14: 1, 12: 2} and c.clock == 6
    c.resize(5)
    assert c.contents() == ([10, 14, 12, -1, -1], [5, 4, 6, 0, 0])


def test_prefill_after_resize_reloads_its_layer():
    """The layer-ahead state is cleared by a resize: the next prefill call
    looks its own layer up again (hits for what survived)."""
    L, E = 3, 4
    c = cache.ExpertCache(L, E, 2 * E)
    full = np.ones(E, int)
    c.forward(0, PREFILL, full)            # loads 0, prefetches 1
    c.resize(2 * E + 2)
    rec = c.forward(1, PREFILL, full)
    assert [k for (l, _, k) in rec["lookups"] if l == 1] == [HIT] * E
    assert rec["n_cur"] == E


def test_static_hot_placement_is_the_best_static_placement():
    """Brute force over every placement of C slots on small random traces:
    none misses less than the most-looked-up keys."""
    import itertools
    rng = np.random.default_rng(7)
    for _ in range(6):
        keys = 7
        batches = [sorted(set(int(k) for k in rng.choice(keys, size=rng.integers(1, 4),
                                                          p=np.arange(keys, 0, -1) / (keys * (keys + 1) / 2))))
                   for _ in range(30)]
        counts = {}
        for b in batches:
            for k in b:
                counts[k] = counts.get(k, 0) + 1
        for C in range(0, keys + 1):
            hot = cache.static_hot_placement(counts, C)
            assert len(hot) == min(C, len(counts))
            _, m = cache.static_placement_misses(batches, hot)
            best = min(cache.static_placement_misses(batches, set(S))[1]
                       for S in itertools.combinations(range(keys), C))
            assert m == best, (C, m, best)
    # the extremes
    lookups, m = cache.static_placement_misses(batches, set())
    assert m == lookups
    assert cache.static_placement_misses(batches, set(range(keys)))[1] == 0


def test_policy_comparison_runs_on_a_short_trace():
    """The LRU-against-static comparison script on 8 steps of the 43-layer
    trace: rates in [0, 1], hindsight never worse than the profiled placement."""
    from oracle import policy_compare
    rows = policy_compare.run(steps=8, fracs=(0.37,))
    (C, f, lru, lru_half, st_prior, st_best, pf, link_lru, link_pf), = rows
    assert C == int(0.37 * 43 * 256)
    for r in (lru, lru_half, st_prior, st_best):
        assert 0.0 <= r <= 1.0
    assert st_best <= st_prior
    assert 0.0 <= pf <= 1.0 and link_lru > 0 and link_pf > 0


@pytest.mark.parametrize("C", [1, 3, 6])
def test_prefetch_matches_a_textbook_lru_list(C):
    """Accesses mixed with prefetches, one key per call, q* = m: a prefetch
    inserts a non-resident key at the most-recent end (evicting the least
    recent) and leaves a resident key where it is; the hit/miss sequence and
    the contents match a move-to-front list doing the same."""
    L, E = 2, 6
    rng = np.random.default_rng(100 + C)
    c = cache.ExpertCache(L, E, C, 1, 1)
    lru = OrderedDict()
    for _ in range(400):
        key = int(rng.integers(0, L * E))
        layer, e = divmod(key, E)
        if rng.random() < 0.4:
            n = c.prefetch(layer, [e])
            if key in lru:
                assert n == 0
            else:
                assert n == 1
                if len(lru) >= C:
                    lru.popitem(last=False)
                lru[key] = True
            continue
        counts = np.zeros(E, int); counts[e] = 1
        kind = c.forward(layer, DECODE, counts)["kinds"][e]
        if key in lru:
            lru.move_to_end(key)
            assert kind == HIT
        else:
            assert kind == STAGED
            if len(lru) >= C:
                lru.popitem(last=False)
            lru[key] = True
        assert sorted(k for k in c.contents()[0] if k >= 0) == sorted(lru)


def test_prefetch_keeps_pinned_keys():
    c = cache.ExpertCache(2, 4, 3, 1, 1)
    c.forward(0, DECODE, np.array([1, 1, 1, 0]))          # layer 0 experts 0..2 fill the cache
    before = set(k for k in c.contents()[0] if k >= 0)
    assert c.prefetch(1, [0, 1], pinned_keys=[0, 1, 2]) == 0  # everything pinned: nothing moves
    assert set(k for k in c.contents()[0] if k >= 0) == before
    assert c.prefetch(1, [0], pinned_keys=[0, 1]) == 1        # evicts the one unpinned key, 2
    assert set(k for k in c.contents()[0] if k >= 0) == {0, 1, 4}
    assert c.n["prefetched"] == 1 and c.n["misses"] == 3 and c.n["lookups"] == 3


@pytest.mark.parametrize("C,L", [(1, 3), (2, 3), (2, 4), (4, 3), (3, 1)])
def test_prefetch_mode_matches_a_textbook_lru_list(C, L):
    """One key per call, q* = m, prefetch on: after the access of (l, e) the
    key layer (l+1) mod L accessed last is inserted at the most-recent end if
    absent, evicting the least recent key other than the one just accessed
    (nothing if there is none); contents and hit/miss sequence match."""
    E = 4
    rng = np.random.default_rng(300 + 10 * C + L)
    c = cache.ExpertCache(L, E, C, 1, 1)
    c.prefetch_on = True
    lru = OrderedDict()
    last = {}
    for step in range(150):
        for layer in range(L):
            e = int(rng.integers(0, E))
            key = layer * E + e
            counts = np.zeros(E, int); counts[e] = 1
            kind = c.forward(layer, DECODE, counts)["kinds"][e]
            if key in lru:
                lru.move_to_end(key)
                assert kind == HIT
            else:
                assert kind == STAGED
                if len(lru) >= C:
                    lru.popitem(last=False)
                lru[key] = True
            nxt = (layer + 1) % L
            if nxt in last and last[nxt] not in lru:
                if len(lru) < C:
                    lru[last[nxt]] = True
                else:
                    victims = [k for k in lru if k != key]
                    if victims:
                        del lru[victims[0]]
                        lru[last[nxt]] = True
            last[layer] = key
            assert sorted(k for k in c.contents()[0] if k >= 0) == sorted(lru), (step, layer)
    # with one key per call the next layer's last key was used within the last
    # L calls: it can only have been evicted (and need a prefetch) when C < L
    if 1 < C < L:
        assert c.n["prefetched"] > 0
    else:
        assert c.n["prefetched"] == 0
