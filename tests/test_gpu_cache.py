"""GPU expert-slot cache through the C ABI against the oracle LRU.

Bit-exact: every trace record (call, event, key, slot), the slot of every
requested expert, the slot table / keys / stamps after every call, and the
bytes of every resident slot (each must hold its key's packed blob).
Also: a call that asks for more experts than slots fails and changes
nothing; resize (shrink, in place, grow); an injected fill failure on the
host leaves a consistent cache.
"""
import os

import numpy as np
import pytest
import torch

from expert_cached_sparse_b200 import api as A
from expert_cached_sparse_b200 import workloads as W

from helpers import Layer, dev, make_cache, trace_rows

pytestmark = pytest.mark.gpu


def _orc_rows(recs):
    return [(int(r["call"]), int(r["event"]), int(r["layer"]), int(r["expert"]), int(r["slot"])) for r in recs]


def _check_state(cache, lru):
    s_gpu, k_gpu, st_gpu = cache.snapshot()
    s_orc, k_orc, st_orc = lru.state()
    np.testing.assert_array_equal(s_gpu, s_orc)
    np.testing.assert_array_equal(k_gpu, k_orc)
    np.testing.assert_array_equal(st_gpu, st_orc)


def _check_pool(cache, L, cfg):
    _, key_of, _ = cache.snapshot()
    sb = cache.slot_bytes
    for s, key in enumerate(key_of):
        if key < 0:
            continue
        l, e = divmod(int(key), cfg.experts)
        got = cache.pool[s * sb:(s + 1) * sb].cpu()
        assert torch.equal(got, L.blob(l, e)), (s, l, e)


def _requests(rng, cfg, steps):
    for _ in range(steps):
        l = int(rng.integers(cfg.layers))
        n = int(rng.integers(1, 5))
        idx = np.minimum(cfg.experts - 1, rng.zipf(1.2, size=(n, cfg.top_k)) - 1).astype(np.int32)
        yield l, idx


def test_trace_and_state_match_oracle(orc):
    cfg = W.scaled(W.DS_DECODE, layers=3, experts=16, hidden=256, ffn=256, top_k=3, capacity=10)
    L = Layer(cfg, 0)
    cache = make_cache(L)
    lru = orc.Lru(cfg.layers, cfg.experts, cfg.capacity)
    rng = np.random.default_rng(1)
    cs = torch.cuda.Stream()
    slot_out = torch.empty(cfg.experts, dtype=torch.int32, device="cuda")
    for step, (l, idx) in enumerate(_requests(rng, cfg, 150)):
        rc, recs, slots = lru.call(l, idx)
        if rc == orc.ORC_ERR_CAPACITY:
            with pytest.raises(A.MoeError) as e:
                cache.lookup_update(l, dev(idx), slot_out, copy_stream=cs)
            assert e.value.code == -2
            continue
        cache.lookup_update(l, dev(idx), slot_out, copy_stream=cs)
        torch.cuda.synchronize()
        np.testing.assert_array_equal(slot_out.cpu().numpy(), slots)
        assert trace_rows(cache.read_trace()) == _orc_rows(recs), step
        if step % 25 == 0:
            _check_state(cache, lru)
            _check_pool(cache, L, cfg)
    _check_state(cache, lru)
    _check_pool(cache, L, cfg)
    st = cache.stats()
    assert st["misses"] * cache.slot_bytes == st["fill_bytes"]


def test_capacity_error_changes_nothing(orc):
    cfg = W.scaled(W.DS_DECODE, layers=2, experts=16, hidden=256, ffn=256, top_k=2, capacity=4)
    L = Layer(cfg, 0)
    cache = make_cache(L)
    cs = torch.cuda.Stream()
    cache.lookup_update(0, dev(np.array([1, 2, 3], np.int32)), copy_stream=cs)
    cache.read_trace()
    before = cache.snapshot()
    with pytest.raises(A.MoeError) as e:
        cache.lookup_update(1, dev(np.arange(5, dtype=np.int32)), copy_stream=cs)
    assert e.value.code == -2
    after = cache.snapshot()
    for a, b in zip(before, after):
        np.testing.assert_array_equal(a, b)
    assert len(cache.read_trace()) == 0
    # the clock did not advance: the next call is call 2
    cache.lookup_update(1, dev(np.array([0], np.int32)), copy_stream=cs)
    assert trace_rows(cache.read_trace()) == [(2, 1, 1, 0, 3)]


@pytest.mark.parametrize("in_place", [False, True])
def test_resize_matches_oracle(orc, in_place):
    cfg = W.scaled(W.DS_DECODE, layers=2, experts=24, hidden=256, ffn=256, top_k=2, capacity=12)
    L = Layer(cfg, 0)
    cache = make_cache(L)
    lru = orc.Lru(cfg.layers, cfg.experts, cfg.capacity)
    rng = np.random.default_rng(3)
    cs = torch.cuda.Stream()

    def run(steps):
        for l, idx in _requests(rng, cfg, steps):
            rc, recs, _ = lru.call(l, idx)
            if rc:
                continue
            cache.lookup_update(l, dev(idx), copy_stream=cs)
            assert trace_rows(cache.read_trace()) == _orc_rows(recs)

    run(40)
    for newc in (5, 9, 16, 3, 12):
        rc, recs = lru.resize(newc)
        cache.resize(newc, in_place=in_place)
        assert trace_rows(cache.read_trace()) == _orc_rows(recs), newc
        _check_state(cache, lru)
        _check_pool(cache, L, cfg)
        run(25)
        _check_state(cache, lru)
        _check_pool(cache, L, cfg)


def test_trace40_scale_lru(orc):
    """The 40-layer, 1024-slot cache at full size: 256 steps x 40 layers of 6 experts each."""
    cfg = W.scaled(W.TRACE40, hidden=256, ffn=256)   # tiny blobs, full cache geometry
    L = Layer(cfg, 0, distinct=32)
    cache = make_cache(L, trace_capacity=1 << 20)
    lru = orc.Lru(cfg.layers, cfg.experts, cfg.capacity)
    rng = np.random.default_rng(5)
    cs = torch.cuda.Stream()
    p = 1.0 / np.arange(1, cfg.experts + 1) ** 1.0
    p /= p.sum()
    all_gpu, all_orc = [], []
    for step in range(256):
        for l in range(cfg.layers):
            perm = W.zipf_rank_perm(cfg, 0, l, W.drift_epoch(cfg, step))
            idx = perm[rng.choice(cfg.experts, size=cfg.top_k, replace=False, p=p)].astype(np.int32)
            rc, recs, _ = lru.call(l, idx)
            assert rc == 0
            cache.lookup_update(l, dev(idx), copy_stream=cs)
            all_orc += _orc_rows(recs)
        if step % 32 == 31:
            all_gpu += trace_rows(cache.read_trace())
    all_gpu += trace_rows(cache.read_trace())
    assert all_gpu == all_orc
    _check_state(cache, lru)
    st = cache.stats()
    assert st["lookups"] == 256 * 40 and st["hits"] + st["misses"] == 256 * 40 * 6


def test_injected_fill_failure_is_rolled_back(orc, monkeypatch):
    cfg = W.scaled(W.DS_DECODE, layers=1, experts=8, hidden=256, ffn=256, top_k=2, capacity=4)
    L = Layer(cfg, 0)
    monkeypatch.setenv("MOE_FAULT_INJECT", "fill_fail:3")
    cache = make_cache(L)
    monkeypatch.delenv("MOE_FAULT_INJECT")
    cs = torch.cuda.Stream()
    cache.lookup_update(0, dev(np.array([0, 1], np.int32)), copy_stream=cs)      # fills 1, 2
    with pytest.raises(A.MoeError) as e:
        cache.lookup_update(0, dev(np.array([2, 3], np.int32)), copy_stream=cs)  # fill 3 fails
    assert e.value.code == -4
    slot_of, key_of, _ = cache.snapshot()
    assert slot_of[2] == -1 and slot_of[3] == -1       # not resident after the failure
    assert slot_of[0] >= 0 and slot_of[1] >= 0
    assert sorted(int(k) for k in key_of if k >= 0) == [0, 1]
    cache.read_trace()
    cache.lookup_update(0, dev(np.array([2, 3], np.int32)), copy_stream=cs)      # injection is one-shot
    ev = [r[1] for r in trace_rows(cache.read_trace())]
    assert ev == [1, 1]
    _check_pool(cache, L, cfg)
