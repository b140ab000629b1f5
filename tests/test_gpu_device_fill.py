"""Device-initiated miss fills (moe_cache_set_fill_mode(MOE_FILL_DEVICE)).

A copy kernel takes the miss list from the lookup on the device and loads
the blobs from mapped pinned host memory, so no call reads anything back and
a decode step with misses can be captured in a CUDA graph.  Misses run in
miss groups, each FFN pass after its own fills.  Checked against
the oracle: routing and the cache trace bit-exact on every call, outputs
within the layer tolerance, slot contents equal to the blobs; and against
host fills: the same bits.
"""
import numpy as np
import pytest
import torch

from expert_cached_sparse_b200 import _lib as L
from expert_cached_sparse_b200 import api as A
from expert_cached_sparse_b200 import workloads as W

from helpers import ALARM_REL_L2, TOL_REL_L2, Layer, dev, host, make_cache, rel_l2, trace_rows

pytestmark = pytest.mark.gpu

# 48 experts, 16 slots, k = 4: a call of <= 4 tokens asks for <= 16 distinct
# experts; flat routing (Zipf 0.3) keeps the stream missing and evicting
SMALL = W.scaled(W.DS_DECODE, experts=48, hidden=256, ffn=256, top_k=4, capacity=16, zipf_s=0.3)


def _rows(recs):
    return [(int(r["call"]), int(r["event"]), int(r["layer"]), int(r["expert"]), int(r["slot"])) for r in recs]


class Step:
    """One layer's fixed-size step buffers (reused, so a graph can capture them)."""

    def __init__(self, cache, cfg, shape, n, seed=0, layer=0):
        self.cache, self.cfg, self.n, self.layer = cache, cfg, n, layer
        self.wg_np = W.gen_wg(cfg, seed, layer)
        self.bias_np = W.gen_bias(cfg, seed, layer, 0)
        self.wg, self.bias = dev(self.wg_np), dev(self.bias_np)
        self.x = torch.empty(n, cfg.hidden, dtype=torch.bfloat16, device="cuda")
        self.out = torch.empty_like(self.x)
        self.idx = torch.empty(n, cfg.top_k, dtype=torch.int32, device="cuda")
        self.ws = torch.empty(A.moe_layer_workspace_bytes(shape, n), dtype=torch.uint8, device="cuda")
        self.stream = torch.cuda.Stream()
        self.copy = torch.cuda.Stream()

    def enqueue(self):
        A.moe_layer_forward(self.cache, self.layer, self.x, self.wg, self.bias, self.out, self.ws,
                            stream=self.stream, copy_stream=self.copy, topk_idx_out=self.idx)

    def run(self, x_np):
        self.x.copy_(dev(x_np))
        torch.cuda.synchronize()
        with torch.cuda.stream(self.stream):
            self.enqueue()
        self.stream.synchronize()
        return host(self.out), host(self.idx)


def _oracle_out(orc, Ly, cfg, step, x, tokens=None):
    fn = lambda e: Ly.expert(step.layer, e)
    return orc.moe_layer(x, step.wg_np, step.bias_np, cfg.top_k, cfg.wfmt, cfg.hidden, cfg.ffn, fn, tokens=tokens)


def _check_slots(cache, Ly, cfg):
    """Every resident slot holds the bytes of its key's blob."""
    _, key_of, _ = cache.snapshot()
    sb = cache.slot_bytes
    for s, key in enumerate(key_of):
        if key < 0:
            continue
        blob = Ly.blob(int(key) // cfg.experts, int(key) % cfg.experts).to("cuda")
        assert torch.equal(cache.pool[s * sb:(s + 1) * sb], blob), (s, key)


@pytest.mark.parametrize("n", [1, 16])
def test_device_fill_cold_decode_stream(orc, n):
    """DeepSeek-V4-Flash-shaped MXFP4 decode, 64 slots, cold start, device fills."""
    cfg = W.DS_DECODE
    Ly = Layer(cfg, 0)
    cache = make_cache(Ly, trace_capacity=1 << 20)
    cache.set_fill_mode(L.FILL_DEVICE)
    assert cache.fill_mode == L.FILL_DEVICE
    st = Step(cache, cfg, Ly.shape, n)
    lru = orc.Lru(1, cfg.experts, cfg.capacity)
    steps = 12
    for s in range(steps):
        x = W.gen_x(cfg, 0, n, "decode", s)
        out, idx = st.run(x)
        toks = None if (n == 1 or s % 4 == 0) else [0, n // 2, n - 1]
        ref, i_ref, _, _ = _oracle_out(orc, Ly, cfg, st, x, tokens=toks)
        if toks is None:
            np.testing.assert_array_equal(idx, i_ref)
            err = rel_l2(out, ref)
        else:
            np.testing.assert_array_equal(idx[toks], i_ref)
            err = rel_l2(out[toks], ref)
        assert err < TOL_REL_L2 and err < ALARM_REL_L2, (n, s, err)
        rc, recs, _ = lru.call(0, idx)
        assert rc == 0
        assert trace_rows(cache.read_trace()) == _rows(recs), s
    stats = cache.stats()
    assert stats["host_syncs"] == 0
    assert stats["misses"] > 0
    assert stats["fill_bytes"] == stats["misses"] * cache.slot_bytes
    assert cache.device_status() == 0
    _check_slots(cache, Ly, cfg)


def test_device_fill_matches_host_fill_bits(orc):
    """The same stream through host fills and device fills: identical outputs, traces and state."""
    cfg = SMALL
    Ly = Layer(cfg, 3)
    c_host = make_cache(Ly)
    c_dev = make_cache(Ly)
    c_dev.set_fill_mode(L.FILL_DEVICE)
    n = 4
    s_host, s_dev = Step(c_host, cfg, Ly.shape, n, 3), Step(c_dev, cfg, Ly.shape, n, 3)
    for s in range(10):
        x = W.gen_x(cfg, 3, n, "decode", s)
        o1, i1 = s_host.run(x)
        o2, i2 = s_dev.run(x)
        np.testing.assert_array_equal(i1, i2)
        np.testing.assert_array_equal(o1, o2)
        assert trace_rows(c_host.read_trace()) == trace_rows(c_dev.read_trace())
    for a, b in zip(c_host.snapshot(), c_dev.snapshot()):
        np.testing.assert_array_equal(a, b)
    assert c_dev.stats()["host_syncs"] == 0 and c_host.stats()["host_syncs"] == 10
    assert c_dev.stats()["fill_bytes"] == c_host.stats()["fill_bytes"]


def test_device_fill_step_with_misses_replays_from_a_cuda_graph(orc):
    """A whole layer step, misses included, captured once and replayed on
    fresh inputs: routing, trace and outputs as eager host-fill calls give."""
    cfg = W.scaled(SMALL, capacity=8)   # 2 tokens x top-4 <= 8 distinct experts
    Ly = Layer(cfg, 5)
    c_ref = make_cache(Ly)
    c_dev = make_cache(Ly)
    c_dev.set_fill_mode(L.FILL_DEVICE)
    n = 2
    s_ref, s_dev = Step(c_ref, cfg, Ly.shape, n, 5), Step(c_dev, cfg, Ly.shape, n, 5)
    lru = orc.Lru(1, cfg.experts, cfg.capacity)
    xs = [W.gen_x(cfg, 5, n, "graph", i) for i in range(16)]
    # capture on the first input (the capture itself runs nothing)
    s_dev.x.copy_(dev(xs[0]))
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s_dev.stream):
        s_dev.enqueue()
    misses = evictions = 0
    for i, x in enumerate(xs):
        o_ref, i_ref = s_ref.run(x)
        s_dev.x.copy_(dev(x))
        torch.cuda.synchronize()
        g.replay()
        torch.cuda.synchronize()
        np.testing.assert_array_equal(host(s_dev.idx), i_ref)
        np.testing.assert_array_equal(host(s_dev.out), o_ref)
        rc, recs, _ = lru.call(0, i_ref)
        assert rc == 0
        rows = trace_rows(c_dev.read_trace())
        assert rows == _rows(recs), i
        assert rows == trace_rows(c_ref.read_trace())
        misses += sum(1 for r in rows if r[1] == 1)
        evictions += sum(1 for r in rows if r[1] == 2)
        if i in (0, 7):
            ref, _, _, _ = _oracle_out(orc, Ly, cfg, s_ref, x)
            assert rel_l2(o_ref, ref) < ALARM_REL_L2
    del g
    assert misses > cfg.capacity and evictions > 0   # the stream kept evicting and refilling
    assert c_dev.stats()["host_syncs"] == 0
    _check_slots(c_dev, Ly, cfg)


def test_device_fill_capacity_error_is_reported_on_the_device(orc):
    cfg = SMALL
    Ly = Layer(cfg, 7)
    cache = make_cache(Ly)
    cache.set_fill_mode(L.FILL_DEVICE)
    st = Step(cache, cfg, Ly.shape, 2, 7)
    st.run(W.gen_x(cfg, 7, 2, "decode", 0))
    cache.read_trace()
    before = cache.snapshot()
    too_many = torch.arange(cfg.capacity + 1, dtype=torch.int32, device="cuda")
    slot_of = torch.zeros(cfg.experts, dtype=torch.int32, device="cuda")
    cache.lookup_update(0, too_many, slot_of=slot_of, stream=st.stream, copy_stream=st.copy)
    torch.cuda.synchronize()
    assert cache.device_status() == L.MOE_ERR_CAPACITY
    assert cache.device_status(clear=True) == L.MOE_ERR_CAPACITY
    assert cache.device_status() == 0
    assert (host(slot_of) == -1).all()
    for a, b in zip(before, cache.snapshot()):
        np.testing.assert_array_equal(a, b)
    assert len(cache.read_trace()) == 0


def test_fill_mode_switch_back_to_host(orc):
    """Device fills, then host fills on the same cache: the host mirror of the
    resident keys is rebuilt, so the trace and residency stay right."""
    cfg = SMALL
    Ly = Layer(cfg, 9)
    cache = make_cache(Ly)
    lru = orc.Lru(1, cfg.experts, cfg.capacity)
    st = Step(cache, cfg, Ly.shape, 4, 9)
    cache.set_fill_mode(L.FILL_DEVICE)
    for s in range(12):
        if s == 6:
            cache.set_fill_mode(L.FILL_HOST)
        x = W.gen_x(cfg, 9, 4, "decode", s)
        _, idx = st.run(x)
        rc, recs, _ = lru.call(0, idx)
        assert trace_rows(cache.read_trace()) == _rows(recs), s
    assert cache.stats()["host_syncs"] == 6
    _check_slots(cache, Ly, cfg)


def test_device_fill_rejects_pageable_blobs():
    cfg = SMALL
    shape = A.shape_of(cfg)
    sb = A.moe_slot_bytes(shape)
    pageable = [np.zeros(sb, np.uint8) for _ in range(cfg.layers * cfg.experts)]
    cache = A.MoeCache(shape, cfg.capacity, pageable)
    with pytest.raises(A.MoeError) as ei:
        cache.set_fill_mode(L.FILL_DEVICE)
    assert ei.value.code == L.MOE_ERR_INVALID_ARG
    assert cache.fill_mode == L.FILL_HOST
    cache.close()


@pytest.fixture
def profiling():
    A.moe_profile_enable(True)
    A.moe_profile_read(reset=True)
    yield
    A.moe_profile_enable(False)
    A.moe_profile_read(reset=True)


@pytest.mark.parametrize("fill", [L.FILL_HOST, L.FILL_DEVICE], ids=["host", "device"])
def test_misses_run_in_miss_groups(orc, profiling, fill):
    """With nm misses a call runs its hit pass, then one FFN pass per miss group:
    min(nm, 4) with host fills (the host knows nm), always 4 with device fills
    (the empty ones compute nothing).  Seed 12's stream has calls with 0, 1, 2,
    3, 4, 5 and 8 misses (oracle router and LRU), so every grouping occurs;
    outputs and the trace as the oracle gives them."""
    cfg = SMALL
    Ly = Layer(cfg, 12)
    cache = make_cache(Ly)
    if fill == L.FILL_DEVICE:
        cache.set_fill_mode(fill)
    st = Step(cache, cfg, Ly.shape, 4, 12)
    lru = orc.Lru(1, cfg.experts, cfg.capacity)
    seen = set()
    for s in range(12):
        x = W.gen_x(cfg, 12, 4, "decode", s)
        out, idx = st.run(x)
        passes = A.moe_profile_read(reset=True)["ffn"]["timed"]
        rc, recs, _ = lru.call(0, idx)
        assert rc == 0
        assert trace_rows(cache.read_trace()) == _rows(recs), s
        nm = sum(1 for r in recs if int(r["event"]) == 1)
        seen.add(nm)
        assert passes == 1 + (4 if fill == L.FILL_DEVICE else min(nm, 4)), (s, nm, passes)
        ref, i_ref, _, _ = _oracle_out(orc, Ly, cfg, st, x)
        np.testing.assert_array_equal(idx, i_ref)
        err = rel_l2(out, ref)
        assert err < TOL_REL_L2 and err < ALARM_REL_L2, (s, nm, err)
    assert {0, 1, 2, 3, 4, 5, 8} <= seen
    _check_slots(cache, Ly, cfg)
