"""The whole layer (moe_layer_forward through the C ABI) against the oracle,
on the five workloads at their full sizes.

Every call: routing indices bit-exact and the cache trace bit-exact against
the oracle LRU fed the GPU's routing.  Outputs (relative L2 against the fp64
oracle within 2e-2): every token of the tiny layer, of the BF16 decode
batches and of 512-token prefill batches (seeded from the 4096-token MXFP4
prefill; the whole BF16 prefill); every token of a seeded subset of the 256
steps of the MXFP4 decode stream at 1, 4 and 16 tokens; and every layer of
steps 0, 31, 32, 63, 64 and 255 of the 40-layer trace.  The full-size oracle
runs on a pool of host processes (``oracle_pool``).
"""
import numpy as np
import pytest
import torch

from expert_cached_sparse_b200 import api as A
from expert_cached_sparse_b200 import workloads as W

from helpers import ALARM_REL_L2, TOL_REL_L2, Layer, dev, host, make_cache, preload, rel_l2, trace_rows
from oracle_pool import layer_outputs

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

    def pooled(self, orc, calls):
        """calls: [(layer, x, epoch, tokens)] -> oracle (out, idx, w) per call, on the pool."""
        return layer_outputs(orc, self.cfg, self.seed, self.L.distinct,
                             [(l, x, *self.router(l, ep), toks) for l, x, ep, toks in calls])

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
    """DeepSeek-V4-Flash-shaped MXFP4 decode, 64 slots, cold start, 256 steps:
    routing and trace bit-exact on every step, every token's output on 12
    seeded steps (the first three and the last among them)."""
    cfg = W.DS_DECODE
    R = Runner(cfg)
    lru = orc.Lru(1, cfg.experts, cfg.capacity)
    steps = 256
    rng = np.random.default_rng(100 + n)
    check = sorted({0, 1, 2, steps - 1} | set(rng.choice(np.arange(3, steps - 1), 8, replace=False).tolist()))
    got = {}
    for s in range(steps):
        x = W.gen_x(cfg, 0, n, "decode", s)
        out, idx, w = R.forward(0, x)
        _, i_ref, _ = orc.router(x, *R.router(0), cfg.top_k)
        np.testing.assert_array_equal(idx, i_ref)
        # trace: the oracle LRU fed the routing (equal to the oracle's, checked above)
        rc, recs, _ = lru.call(0, idx)
        assert rc == 0
        assert trace_rows(R.cache.read_trace()) == _rows(recs), s
        if s in check:
            got[s] = (x, out, w)
    refs = R.pooled(orc, [(0, got[s][0], 0, None) for s in check])
    for s, (ref, i_ref, w_ref) in zip(check, refs):
        _check_out(got[s][1], ref, ("decode", n, s))
        assert rel_l2(got[s][2], w_ref) < 1e-5
    st = R.cache.stats()
    assert st["misses"] > 0 and st["host_syncs"] == steps and st["lookups"] == steps


def test_ds_prefill_sampled(orc):
    """4096-token MXFP4 prefill, all experts resident: routing of every token,
    outputs of 512 seeded tokens (the last one among them)."""
    cfg = W.DS_PREFILL
    R = Runner(cfg)
    preload(R.cache, cfg)
    R.cache.read_trace()
    n = 4096
    x = W.gen_x(cfg, 0, n, "prefill")
    out, idx, w = R.forward(0, x)
    toks = sorted(np.random.default_rng(0).choice(n - 1, 511, replace=False).tolist()) + [n - 1]
    # full-size routing is cheap for the oracle's router alone: check every token
    _, i_all, _ = orc.router(x, *R.router(0), cfg.top_k)
    np.testing.assert_array_equal(idx, i_all)
    (ref, _, _), = R.pooled(orc, [(0, x, 0, toks)])
    _check_out(out[toks], ref, "ds-prefill")
    assert R.cache.stats()["host_syncs"] == 1   # only the preload lookup read anything back


def test_qwen_bf16_prefill_and_decode(orc):
    cfg = W.QWEN_BF16
    R = Runner(cfg)
    preload(R.cache, cfg)
    x = W.gen_x(cfg, 0, 512, "prefill")
    out, idx, _ = R.forward(0, x)
    dec = [W.gen_x(cfg, 0, 8, "decode", s) for s in range(16)]
    got = [R.forward(0, xd) for xd in dec]
    refs = R.pooled(orc, [(0, x, 0, None)] + [(0, xd, 0, None) for xd in dec])
    ref, i_ref, _ = refs[0]
    np.testing.assert_array_equal(idx, i_ref)
    _check_out(out, ref, "qwen-prefill")
    for s, ((o, i, _), (ref, i_ref, _)) in enumerate(zip(got, refs[1:])):
        np.testing.assert_array_equal(i, i_ref)
        _check_out(o, ref, ("qwen-decode", s))


def _rows(recs):
    return [(int(r["call"]), int(r["event"]), int(r["layer"]), int(r["expert"]), int(r["slot"])) for r in recs]


def test_trace40_nvfp4(orc):
    """40 layers x 1024 shared slots, NVFP4, Zipf(1.0) routing with drift every
    32 steps, 256 steps from a cold cache: routing and trace bit-exact on every
    one of the 10,240 layer calls; every layer's output at steps 0, 31, 32, 63,
    64 and 255 (drift-epoch edges and the last step).  Blobs aliased to 64
    distinct expert weight sets (the cache does not depend on blob contents).
    """
    cfg = W.TRACE40
    R = Runner(cfg, distinct=64)
    lru = orc.Lru(cfg.layers, cfg.experts, cfg.capacity)
    out_steps = {0, 31, 32, 63, 64, 255}
    steps = 256
    got, calls = [], []
    for s in range(steps):
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
            if s in out_steps:
                got.append(((s, l), out))
                calls.append((l, x, ep, None))
        assert trace_rows(R.cache.read_trace()) == expect, s
    for ((s, l), out), (ref, _, _) in zip(got, R.pooled(orc, calls)):
        _check_out(out, ref, ("trace", s, l))
    st = R.cache.stats()
    assert st["lookups"] == steps * cfg.layers and st["evictions"] > 0


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
