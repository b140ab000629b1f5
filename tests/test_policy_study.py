"""The placement study reproduced on the CPU: the 40-layer trace workload
routed by the oracle router (64 one-token steps: two drift epochs; a 64-token
prefill for hot placement), replayed through the shared LRU, the layer split,
prefill-hot placement and the offline optimum.  The ordering the pages report
for the shared LRU against a routing-unaware split must hold, and the optimum
must bound the LRU."""
import pytest

from expert_cached_sparse_b200 import policy as P
from expert_cached_sparse_b200 import workloads as W

from helpers import oracle_route_trace

STEPS, PREFILL = 64, 64


@pytest.fixture(scope="module")
def traces(orc):
    return oracle_route_trace(orc, W.TRACE40, STEPS, PREFILL)


@pytest.mark.parametrize("capacity", [512, 1024])
def test_shared_lru_beats_the_layer_split(traces, capacity):
    cfg = W.TRACE40
    decode, prefill = traces
    lru = P.replay(P.SharedLru(capacity), decode)
    split = P.replay(P.StaticPlacement(P.layer_split(cfg.layers, cfg.experts, capacity)), decode)
    hot = P.replay(P.StaticPlacement(P.prefill_hot(prefill, capacity)), decode)
    opt = P.belady(decode, capacity)
    reads = sum(len(set(int(e) for e in ids)) for _, ids in decode)
    for r in (lru, split, hot, opt):
        assert r["reads"] == reads
    # a layer split keeps capacity / E whole layers: every read of the other layers misses
    resident_layers = capacity // cfg.experts
    assert split["miss_rate"] >= 1 - resident_layers / cfg.layers - 1e-9
    # the ordering the pages report: the shared LRU misses far less than the static split
    assert lru["miss_rate"] < 0.6 * split["miss_rate"]
    # the offline optimum bounds every demand-filled cache from the same cold start (the
    # static placements start warm and cache nothing, so it does not bound them)
    assert opt["miss_rate"] <= lru["miss_rate"]
