"""The whole layer (moe_layer_forward through the C ABI) against the oracle,
on the five workloads at their full sizes.

Every call: routing indices bit-exact and the cache trace bit-exact against
the oracle LRU fed the oracle's own routing.  Outputs: all tokens where the
oracle is fast enough (tiny layer, decode batches), seeded token samples for
the prefills and chosen (step, layer) calls of the 40-layer trace; relative
L2 against the fp64 oracle within 2e-2.
"""
import numpy as np
import pytest
import torch

from expert_cached_sparse_b200 import api as A
from expert_cached_sparse_b200 import workloads as W

from helpers import ALARM_REL_L2, TOL_REL_L2, Layer, dev, host, make_cache, preload, rel_l2, trace_rows

pytestmark = pytest.mark.gpu


class Runner:
    def __init__(self, cfg, capacity=None, distinct=None, seed=0):
        self.cfg, self.seed = cfg, seed
        self.L = Layer(cfg, seed, distinct)
        self.cache = make_cache(self.L, capacity=capacity, trace_capacity=1 << 20)
        self.stream = torch.cuda.Stream()
        self.copy = torch.cuda.Stream()
        self.wg = {}
        self.bias = {}

    def router(self, layer, epoch=0):
        if layer not in self.wg:
            self.wg[layer] = W.gen_wg(self.cfg, self.seed, layer)
        key = (layer, epoch)
        if key not in self.bias:
            self.bias[key] = W.gen_bias(self.cfg, self.seed, layer, epoch)
        return self.wg[layer], self.bias[key]

    def forward(self, layer, x, epoch=0):
        cfg = self.cfg
        wg, bias = self.router(layer, epoch)
        n = x.shape[0]
        xd = dev(x) if cfg.x_dtype == "bf16" else dev(x.astype(np.float32))
        out = torch.empty_like(xd)
        ws = torch.empty(A.moe_layer_workspace_bytes(self.L.shape, n), dtype=torch.uint8, device="cuda")
        idx = torch.empty(n, cfg.top_k, dtype=torch.int32, device="cuda")
        w = torch.empty(n, cfg.top_k, dtype=torch.float32, device="cuda")
        wgd, bd = dev(wg), None if bias is None else dev(bias)
        torch.cuda.synchronize()   # inputs copied on the default stream are complete
        with torch.cuda.stream(self.stream):
            A.moe_layer_forward(self.cache, layer, xd, wgd, bd, out, ws,
                                stream=self.stream, copy_stream=self.copy, topk_idx_out=idx, topk_w_out=w)
        self.stream.synchronize()
        return host(out), host(idx), host(w)

    def oracle_out(self, orc, layer, x, tokens=None, epoch=0):
        cfg = self.cfg
        wg, bias = self.router(layer, epoch)
        fn = lambda e: self.L.expert(layer, e)
        return orc.moe_layer(x, wg, bias, cfg.top_k, cfg.wfmt, cfg.hidden, cfg.ffn, fn, tokens=tokens)


def _check_out(got, ref, what):
    err = rel_l2(got, ref)
    assert err < TOL_REL_L2, (what, err)
    assert err < ALARM_REL_L2, (what, err)
    return err


def test_tiny_layer(orc):
    cfg = W.TINY
    R = Runner(cfg)
    preload(R.cache, cfg)
    R.cache.read_trace()
    x = W.gen_x(cfg, 0, 64, "layer")
    out, idx, w = R.forward(0, x)
    ref, i_ref, w_ref, _ = R.oracle_out(orc, 0, x)
    np.testing.assert_array_equal(idx, i_ref)
    _check_out(out, ref, "tiny")
    assert rel_l2(w, w_ref) < 1e-5
    # fully resident: every record is a hit
    assert all(r[1] == 0 for r in trace_rows(R.cache.read_trace()))


@pytest.mark.parametrize("n", [1, 4, 16])
def test_ds_decode_cold_cache(orc, n):
    """DeepSeek-V4-Flash-shaped MXFP4 decode, 64 slots, cold start, misses filled on the copy stream."""
    cfg = W.DS_DECODE
    R = Runner(cfg)
    lru = orc.Lru(1, cfg.experts, cfg.capacity)
    steps = 10 if n < 16 else 6
    for s in range(steps):
        x = W.gen_x(cfg, 0, n, "decode", s)
        out, idx, w = R.forward(0, x)
        full = s < 3 or n == 1
        toks = None if full else [0, n // 2, n - 1]
        ref, i_ref, w_ref, _ = R.oracle_out(orc, 0, x, tokens=None if full else toks)
        if full:
            np.testing.assert_array_equal(idx, i_ref)
            _check_out(out, ref, ("decode", n, s))
        else:
            np.testing.assert_array_equal(idx[toks], i_ref)
            _check_out(out[toks], ref, ("decode", n, s))
        # trace: the oracle LRU fed the GPU's routing (equal to the oracle's, checked above)
        rc, recs, _ = lru.call(0, idx)
        assert rc == 0
        assert trace_rows(R.cache.read_trace()) == _rows(recs)
    st = R.cache.stats()
    assert st["misses"] > 0 and st["host_syncs"] == steps


def test_ds_prefill_sampled(orc):
    """4096-token MXFP4 prefill, all experts resident, 24 sampled tokens against the oracle."""
    cfg = W.DS_PREFILL
    R = Runner(cfg)
    preload(R.cache, cfg)
    R.cache.read_trace()
    n = 4096
    x = W.gen_x(cfg, 0, n, "prefill")
    out, idx, w = R.forward(0, x)
    toks = sorted(np.random.default_rng(0).choice(n, 24, replace=False).tolist()) + [n - 1]
    # full-size routing is cheap for the oracle's router alone: check every token
    _, i_all, _ = orc.router(x, *R.router(0), cfg.top_k)
    np.testing.assert_array_equal(idx, i_all)
    ref, _, _, _ = R.oracle_out(orc, 0, x, tokens=toks)
    _check_out(out[toks], ref, "ds-prefill")
    assert R.cache.stats()["host_syncs"] == 1   # only the preload lookup read anything back


def test_qwen_bf16_prefill_and_decode(orc):
    cfg = W.QWEN_BF16
    R = Runner(cfg)
    preload(R.cache, cfg)
    x = W.gen_x(cfg, 0, 512, "prefill")
    out, idx, _ = R.forward(0, x)
    toks = sorted(np.random.default_rng(1).choice(512, 48, replace=False).tolist())
    ref, i_ref, _, _ = R.oracle_out(orc, 0, x, tokens=toks)
    np.testing.assert_array_equal(idx[toks], i_ref)
    _check_out(out[toks], ref, "qwen-prefill")
    for s in range(4):
        x = W.gen_x(cfg, 0, 8, "decode", s)
        out, idx, _ = R.forward(0, x)
        ref, i_ref, _, _ = R.oracle_out(orc, 0, x)
        np.testing.assert_array_equal(idx, i_ref)
        _check_out(out, ref, ("qwen-decode", s))


def _rows(recs):
    return [(int(r["call"]), int(r["event"]), int(r["layer"]), int(r["expert"]), int(r["slot"])) for r in recs]


def test_trace40_nvfp4(orc):
    """40 layers x 1024 shared slots, NVFP4, Zipf(1.0) routing with drift every 32 steps.

    48 steps (drift epochs 0 and 1) x 40 layers; blobs aliased to 48 distinct
    expert weight sets (the cache does not depend on blob contents).
    """
    cfg = W.TRACE40
    R = Runner(cfg, distinct=48)
    lru = orc.Lru(cfg.layers, cfg.experts, cfg.capacity)
    checks = {(0, 0), (0, 39), (31, 7), (32, 20), (47, 39)}
    for s in range(48):
        ep = W.drift_epoch(cfg, s)
        expect = []
        for l in range(cfg.layers):
            x = W.gen_x(cfg, 0, 1, "trace", s, l)
            out, idx, _ = R.forward(l, x, epoch=ep)
            _, i_ref, _ = orc.router(x, *R.router(l, ep), cfg.top_k)
            np.testing.assert_array_equal(idx, i_ref)
            rc, recs, _ = lru.call(l, idx)
            assert rc == 0
            expect += _rows(recs)
            if (s, l) in checks:
                ref, _, _, _ = R.oracle_out(orc, l, x, epoch=ep)
                _check_out(out, ref, ("trace", s, l))
        assert trace_rows(R.cache.read_trace()) == expect, s
    st = R.cache.stats()
    assert st["lookups"] == 48 * 40


def test_resident_layer_replays_from_a_cuda_graph(orc):
    """With every expert of the layer resident, moe_layer_forward reads
    nothing back to the host, so a whole layer step can be captured in a CUDA
    graph and replayed; replays with fresh inputs match eager calls exactly."""
    cfg = W.scaled(W.DS_DECODE, experts=16, hidden=256, ffn=256, top_k=4, capacity=16)
    R = Runner(cfg)
    preload(R.cache, cfg)
    wg, bias = R.router(0)
    wgd, bd = dev(wg), dev(bias)
    n = 8
    xs = [W.gen_x(cfg, 0, n, "graph", i) for i in range(3)]
    eager = []
    for x in xs:
        out, idx, _ = R.forward(0, x)
        eager.append((out, idx))
    xin = dev(xs[0]).clone()
    out = torch.empty_like(xin)
    idx = torch.empty(n, cfg.top_k, dtype=torch.int32, device="cuda")
    ws = torch.empty(A.moe_layer_workspace_bytes(R.L.shape, n), dtype=torch.uint8, device="cuda")
    s = torch.cuda.Stream()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        A.moe_layer_forward(R.cache, 0, xin, wgd, bd, out, ws, stream=s, copy_stream=R.copy, topk_idx_out=idx)
    for x, (o_ref, i_ref) in zip(xs, eager):
        xin.copy_(dev(x))
        g.replay()
        torch.cuda.synchronize()
        np.testing.assert_array_equal(host(idx), i_ref)
        np.testing.assert_array_equal(host(out), o_ref)
    del g
