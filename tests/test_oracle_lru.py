"""Pins for the oracle's shared (layer, expert) LRU slot cache (CPU only).

 - a hand-traced run (golden fixture) covering ties, refusals and resizes;
 - with one expert per call (no ties possible) the hit / miss / evicted-key
   sequence equals a textbook LRU built on collections.OrderedDict;
 - Belady's MIN never misses more than LRU on the same sequence;
 - invariants on random multi-expert, multi-layer runs.
"""
import collections
import os

import numpy as np

GOLD = os.path.join(os.path.dirname(__file__), "golden")
EV = {"HIT": 0, "MISS": 1, "EVICT": 2, "MOVE": 3}


def _parse_golden():
    ops, shape = [], None
    for raw in open(os.path.join(GOLD, "lru_hand_trace.txt")):
        line = raw.split("#")[0].rstrip()
        if not line:
            continue
        tok = line.split()
        if tok[0] == "shape":
            shape = tuple(int(t) for t in tok[1:])
        elif tok[0] in ("call", "resize"):
            ops.append([tok[0], [int(t) for t in tok[1:]], []])
        else:
            ops[-1][2].append(tok)
    return shape, ops


def test_hand_trace(orc):
    (L, E, C), ops = _parse_golden()
    lru = orc.Lru(L, E, C)
    for kind, args, expect in ops:
        if kind == "call":
            rc, recs, _ = lru.call(args[0], args[1:])
        else:
            rc, recs = lru.resize(args[0])
        if expect == [["CAPACITY"]]:
            assert rc == orc.ORC_ERR_CAPACITY
            assert len(recs) == 0
            continue
        assert rc == 0
        got = [[str(r["call"]), [k for k, v in EV.items() if v == r["event"]][0],
                str(r["layer"]), str(r["expert"]), str(r["slot"])] for r in recs]
        assert got == expect, (kind, args)


def test_single_key_calls_equal_textbook_lru(orc):
    rng = np.random.default_rng(7)
    L, E, C = 3, 32, 11
    lru = orc.Lru(L, E, C)
    od = collections.OrderedDict()
    for _ in range(3000):
        l = int(rng.integers(L))
        e = int(min(E - 1, rng.zipf(1.3) - 1))
        rc, recs, slots = lru.call(l, [e])
        assert rc == 0
        key = (l, e)
        if key in od:
            od.move_to_end(key)
            assert [r["event"] for r in recs] == [0]
        else:
            ev = None
            if len(od) == C:
                ev, _ = od.popitem(last=False)
            od[key] = True
            if ev is None:
                assert [r["event"] for r in recs] == [1]
            else:
                assert [r["event"] for r in recs] == [2, 1]
                assert (int(recs[0]["layer"]), int(recs[0]["expert"])) == ev
        assert slots[e] >= 0


def _belady_misses(seq, C):
    cache, misses = set(), 0
    for i, k in enumerate(seq):
        if k in cache:
            continue
        misses += 1
        if len(cache) == C:
            def nxt(c):
                for j in range(i + 1, len(seq)):
                    if seq[j] == c:
                        return j
                return len(seq) + 1
            cache.remove(max(cache, key=nxt))
        cache.add(k)
    return misses


def test_belady_bound(orc):
    rng = np.random.default_rng(11)
    E, C = 40, 8
    seq = [int(min(E - 1, rng.zipf(1.2) - 1)) for _ in range(600)]
    lru = orc.Lru(1, E, C)
    misses = 0
    for e in seq:
        _, recs, _ = lru.call(0, [e])
        misses += sum(r["event"] == 1 for r in recs)
    assert _belady_misses(seq, C) <= misses


def test_invariants_random_runs(orc):
    rng = np.random.default_rng(5)
    L, E, C, k = 4, 48, 20, 3
    lru = orc.Lru(L, E, C)
    last_use = {}
    slot_key = {}
    for step in range(400):
        l = int(rng.integers(L))
        n = int(rng.integers(1, 6))
        idx = np.minimum(E - 1, rng.zipf(1.15, size=(n, k)) - 1)
        R = sorted(set(int(v) for v in idx.reshape(-1)))
        before_clock = lru.clock
        rc, recs, slots = lru.call(l, idx)
        if len(R) > C:
            assert rc == orc.ORC_ERR_CAPACITY and len(recs) == 0 and lru.clock == before_clock
            continue
        assert rc == 0 and lru.clock == before_clock + 1
        T = lru.clock
        hits = [r for r in recs if r["event"] == 0]
        miss = [r for r in recs if r["event"] == 1]
        evic = [r for r in recs if r["event"] == 2]
        assert len(hits) + len(miss) == len(R)
        assert [int(r["expert"]) for r in hits] == sorted(int(r["expert"]) for r in hits)
        assert [int(r["expert"]) for r in miss] == sorted(int(r["expert"]) for r in miss)
        for r in recs:
            key = (int(r["layer"]), int(r["expert"]))
            if r["event"] == 2:
                assert not (key[0] == l and key[1] in R)       # never evict a requested key
                # the victim is the least recently used non-requested key (ties: slot)
                cands = [(last_use[kk], s) for s, kk in slot_key.items()
                         if not (kk[0] == l and kk[1] in R)]
                assert (last_use[key], int(r["slot"])) == min(cands)
                del slot_key[int(r["slot"])]
            else:
                last_use[key] = T
                slot_key[int(r["slot"])] = key
        # resident set is consistent with the state dump
        slot_of, key_of, stamp = lru.state()
        assert sum(key_of >= 0) <= C
        assert {s: (int(kk) // E, int(kk) % E) for s, kk in enumerate(key_of) if kk >= 0} == slot_key
        for e in R:
            assert slots[e] >= 0 and key_of[slots[e]] == l * E + e and stamp[slots[e]] == T
        assert np.all(slots[[e for e in range(E) if e not in R]] == -1)


def test_resize_keeps_most_recent_and_packs(orc):
    rng = np.random.default_rng(2)
    L, E, C = 2, 30, 12
    lru = orc.Lru(L, E, C)
    for _ in range(60):
        lru.call(int(rng.integers(L)), rng.integers(0, E, size=2))
    slot_of, key_of, stamp = lru.state()
    live = [(int(stamp[s]), s, int(key_of[s])) for s in range(C) if key_of[s] >= 0]
    keep = sorted(live)[-5:]
    rc, recs = lru.resize(5)
    assert rc == 0
    slot_of2, key_of2, stamp2 = lru.state()
    assert lru.capacity == 5
    assert sorted(int(k) for k in key_of2) == sorted(k for _, _, k in keep)
    # packed in old-slot order
    assert [int(k) for k in key_of2] == [k for _, _, k in sorted(keep, key=lambda t: t[1])]
    assert sum(r["event"] == 2 for r in recs) == len(live) - 5
    # grow again: new slots free, next miss takes the lowest free slot
    rc, _ = lru.resize(9)
    _, key_of3, _ = lru.state()
    assert list(key_of3[5:]) == [-1] * 4
