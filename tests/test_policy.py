"""Host policy study: the shared-LRU simulator reproduces the oracle LRU
(and so the GPU cache) call by call; the static placements count as defined."""
import numpy as np
import pytest

from expert_cached_sparse_b200 import policy as P

MISS = 1


@pytest.mark.parametrize("layers,experts,capacity,k", [(1, 8, 3, 2), (3, 16, 10, 4), (5, 64, 40, 6)])
def test_shared_lru_matches_oracle(orc, layers, experts, capacity, k):
    rng = np.random.default_rng(capacity)
    sim = P.SharedLru(capacity)
    lru = orc.Lru(layers, experts, capacity)
    p = 1.0 / np.arange(1, experts + 1)
    p /= p.sum()
    for step in range(300):
        layer = int(rng.integers(layers))
        n = int(rng.integers(1, 4))
        idx = np.stack([rng.choice(experts, size=k, replace=False, p=p) for _ in range(n)]).astype(np.int32)
        rc, recs, _ = lru.call(layer, idx)
        if len(np.unique(idx)) > capacity:   # refused by both, nothing changes
            assert rc != 0
            clock = sim.clock
            with pytest.raises(ValueError):
                sim.call(layer, idx)
            assert sim.clock == clock
            continue
        assert rc == 0
        reads, misses = sim.call(layer, idx)
        assert reads == len(np.unique(idx))
        assert misses == int(np.sum(recs["event"] == MISS))
    # same resident keys in the same slots (oracle keys are layer * E + expert)
    _, key_of, _ = lru.state()
    want = {(int(key) // experts, int(key) % experts): s for s, key in enumerate(key_of) if key >= 0}
    assert sim.resident() == want


def test_shared_lru_refuses_oversized_call():
    sim = P.SharedLru(2)
    with pytest.raises(ValueError):
        sim.call(0, [1, 2, 3])
    assert sim.clock == 0


def test_static_placements():
    keys = P.layer_split(layers=3, experts=4, capacity=6)
    assert keys == [(0, 0), (0, 1), (0, 2), (0, 3), (1, 0), (1, 1)]
    st = P.StaticPlacement(keys)
    assert st.call(0, [0, 3, 3]) == (2, 0)
    assert st.call(1, [1, 2]) == (2, 1)
    assert st.call(2, [0]) == (1, 1)
    prefill = [(0, np.array([[1, 2], [1, 3]])), (1, np.array([[2, 0], [2, 1]]))]
    assert P.prefill_hot(prefill, 3) == [(0, 1), (1, 2), (0, 2)]
    r = P.replay(P.StaticPlacement(P.prefill_hot(prefill, 3)), [(0, [1, 3]), (1, [2])])
    assert r == {"reads": 3, "misses": 1, "miss_rate": 1 / 3}


def test_lru_beats_static_split_on_skewed_routing():
    """On Zipf-skewed routing that every layer shares, the shared LRU misses
    less than the routing-unaware layer split at equal capacity."""
    rng = np.random.default_rng(0)
    layers, experts, k, cap = 8, 64, 4, 128
    p = 1.0 / np.arange(1, experts + 1) ** 1.0
    p /= p.sum()
    perms = [rng.permutation(experts) for _ in range(layers)]
    trace = [(l, perms[l][rng.choice(experts, size=k, replace=False, p=p)])
             for _ in range(200) for l in range(layers)]
    lru = P.replay(P.SharedLru(cap), trace)["miss_rate"]
    split = P.replay(P.StaticPlacement(P.layer_split(layers, experts, cap)), trace)["miss_rate"]
    assert lru < split


def test_belady_is_a_lower_bound_and_optimal_on_a_hand_trace():
    # one layer, capacity 2, reads a b c a b: optimal evicts c's slot owner with the farthest next use
    trace = [(0, [0]), (0, [1]), (0, [2]), (0, [0]), (0, [1])]
    # a, b miss; c misses and evicts b (next read at 4) rather than a (3); a hits; b misses
    assert P.belady(trace, 2) == {"reads": 5, "misses": 4, "miss_rate": 0.8}
    rng = np.random.default_rng(3)
    for cap in (4, 9, 20):
        trace = [(int(rng.integers(3)), rng.choice(16, size=3, replace=False)) for _ in range(400)]
        opt = P.belady(trace, cap)["misses"]
        lru = P.replay(P.SharedLru(cap), trace)["misses"]
        hot = P.replay(P.StaticPlacement(P.layer_split(3, 16, cap)), trace)["misses"]
        assert opt <= lru and opt <= hot


def test_balanced_miss_split():
    m, bp, bh = 10.0, 54.0, 18.0
    q = P.balanced_miss_split(m, bp, bh)
    assert q == pytest.approx(7.5)
    assert q / bp == pytest.approx((m - q) / bh)          # both paths take the same time
    assert 0 <= q <= m
    assert P.balanced_miss_split(m, 1e9, 1.0) == pytest.approx(m, rel=1e-6)
    with pytest.raises(ValueError):
        P.balanced_miss_split(m, 0.0, 1.0)
