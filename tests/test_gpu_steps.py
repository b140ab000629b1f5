"""GPU parity of the individual steps, called through the C ABI, against the
CPU oracle on the same seeded inputs.

Router: logits and top-k indices bit-exact, weights within tolerance.
Permute: offsets / row_of / assign_of bit-exact, x_perm bit-exact.
Grouped FFN: per-expert relative L2 against the fp64 oracle, all formats,
ragged groups (0, 1, 7, 8, 9, 33, 70 rows), permuted slots, two passes.
Combine: against the oracle combine of the same bf16 rows.
"""
import numpy as np
import pytest
import torch

from expert_cached_sparse_b200 import api as A
from expert_cached_sparse_b200 import workloads as W

from helpers import ALARM_REL_L2, TOL_REL_L2, Layer, bf16_bits, dev, host, make_cache, rel_l2

pytestmark = pytest.mark.gpu


def _x_dev(cfg, x):
    return dev(x) if cfg.x_dtype == "bf16" else dev(x.astype(np.float32))


# ------------------------------------------------------------------ router
ROUTER_CASES = [(W.TINY, 64), (W.TINY, 1), (W.DS_DECODE, 1), (W.DS_DECODE, 4), (W.DS_DECODE, 16),
                (W.DS_DECODE, 37), (W.DS_PREFILL, 300), (W.QWEN_BF16, 512), (W.QWEN_BF16, 8),
                (W.TRACE40, 1),
                # expert counts of the other top-k kernels (more than 256, more than 1024) and k = E
                (W.scaled(W.DS_DECODE, hidden=256, experts=600, top_k=8), 5),
                (W.scaled(W.DS_DECODE, hidden=256, experts=2048, top_k=32), 3),
                (W.scaled(W.DS_DECODE, hidden=256, experts=32, top_k=32), 7)]


@pytest.mark.parametrize("cfg,n", ROUTER_CASES, ids=lambda v: getattr(v, "name", str(v)))
def test_router_parity(orc, cfg, n):
    x = W.gen_x(cfg, 0, n, "router")
    wg = W.gen_wg(cfg, 0, 0)
    bias = W.gen_bias(cfg, 0, 0)
    l_ref, i_ref, w_ref = orc.router(x, wg, bias, cfg.top_k)
    E, k = cfg.experts, cfg.top_k
    logits = torch.empty(n, E, dtype=torch.float32, device="cuda")
    idx = torch.empty(n, k, dtype=torch.int32, device="cuda")
    w = torch.empty(n, k, dtype=torch.float32, device="cuda")
    A.moe_router_topk(_x_dev(cfg, x), dev(wg), None if bias is None else dev(bias), n, cfg.hidden, E, k,
                      logits, idx, w)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(host(logits).view(np.uint32), l_ref.view(np.uint32))
    np.testing.assert_array_equal(host(idx), i_ref)
    assert rel_l2(host(w), w_ref) < 1e-5


def test_router_ties_nan_and_empty(orc):
    cfg = W.scaled(W.TINY, hidden=64, experts=8, top_k=3)
    rng = np.random.default_rng(0)
    x = rng.standard_normal((6, 64)).astype(np.float32)
    x[2, 5] = np.nan
    wg = W.gen_wg(cfg, 0, 0)
    wg[3] = wg[6]
    wg[1] = wg[4]
    l_ref, i_ref, w_ref = orc.router(x, wg, None, 3)
    logits = torch.empty(6, 8, device="cuda")
    idx = torch.empty(6, 3, dtype=torch.int32, device="cuda")
    w = torch.empty(6, 3, device="cuda")
    A.moe_router_topk(dev(x), dev(wg), None, 6, 64, 8, 3, logits, idx, w)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(host(idx), i_ref)
    assert list(host(idx)[2]) == [0, 1, 2]
    ok = ~np.isnan(w_ref)
    np.testing.assert_allclose(host(w)[ok], w_ref[ok], rtol=1e-5)
    A.moe_router_topk(dev(x), dev(wg), None, 0, 64, 8, 3, logits, idx, w)   # n = 0: no work


# ------------------------------------------------------------------ permute
PERM_CASES = [(1, 8, 2, "f32"), (64, 8, 2, "f32"), (5, 256, 6, "bf16"), (16, 256, 6, "bf16"),
              (333, 128, 8, "bf16"), (4096, 256, 6, "bf16")]


@pytest.mark.parametrize("n,E,k,xd", PERM_CASES)
def test_permute_parity(orc, n, E, k, xd):
    rng = np.random.default_rng(n * E)
    H = 256
    if n > 100:
        # Zipf-like skew: a few experts take most rows
        idx = np.minimum(E - 1, rng.zipf(1.3, size=(n, k)) - 1).astype(np.int32)
    else:
        idx = rng.integers(0, E, size=(n, k)).astype(np.int32)
    xf = rng.standard_normal((n, H)).astype(np.float32)
    x = xf if xd == "f32" else W.f32_to_bf16_bits(xf)
    off_ref, row_ref, asg_ref = orc.permute(idx, E)
    offs = torch.empty(E + 1, dtype=torch.int32, device="cuda")
    row_of = torch.empty(n * k, dtype=torch.int32, device="cuda")
    asg = torch.empty(n * k, dtype=torch.int32, device="cuda")
    xp = torch.empty(n * k, H, dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(A.moe_permute_workspace_bytes(n, E, k), dtype=torch.uint8, device="cuda")
    A.moe_permute(dev(idx), n, E, k, dev(x), H, offs, row_of, asg, xp, ws)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(host(offs), off_ref)
    np.testing.assert_array_equal(host(row_of), row_ref)
    np.testing.assert_array_equal(host(asg), asg_ref)
    xb = W.f32_to_bf16_bits(xf) if xd == "f32" else x
    np.testing.assert_array_equal(bf16_bits(xp), xb[asg_ref // k])


# ------------------------------------------------------------------ grouped FFN
def _ffn_case(orc, cfg, counts, slots, pool_slots, seed=0, passes=1):
    E = cfg.experts
    L = Layer(cfg, seed)
    shape = A.shape_of(cfg)
    sb = A.moe_slot_bytes(shape)
    pool = torch.zeros(pool_slots * sb, dtype=torch.uint8, device="cuda")
    for e in range(E):
        if 0 <= slots[e] < pool_slots:
            pool[slots[e] * sb:(slots[e] + 1) * sb].copy_(L.blob(0, e), non_blocking=False)
    rows = int(sum(counts))
    offsets = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    rng = np.random.default_rng(seed + 7)
    xb = W.f32_to_bf16_bits(rng.standard_normal((rows, cfg.hidden)).astype(np.float32))
    y = torch.full((rows, cfg.hidden), float("nan"), dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(A.moe_ffn_workspace_bytes(shape, rows), dtype=torch.uint8, device="cuda")
    sl = np.asarray(slots, np.int32)
    if passes == 1:
        A.moe_grouped_ffn(shape, pool, pool_slots, dev(sl), dev(offsets), dev(xb), rows, y, ws)
    else:
        half = np.where(np.arange(E) % 2 == 0, sl, -1).astype(np.int32)
        other = np.where(np.arange(E) % 2 == 1, sl, -1).astype(np.int32)
        A.moe_grouped_ffn(shape, pool, pool_slots, dev(half), dev(offsets), dev(xb), rows, y, ws)
        A.moe_grouped_ffn(shape, pool, pool_slots, dev(other), dev(offsets), dev(xb), rows, y, ws)
    torch.cuda.synchronize()
    yg = host(y)
    xf = W.bf16_bits_to_f32(xb).astype(np.float64)
    worst = 0.0
    for e in range(E):
        r0, r1 = offsets[e], offsets[e + 1]
        if r0 == r1:
            continue
        if not 0 <= slots[e] < pool_slots:
            assert np.all(np.isnan(yg[r0:r1])), "rows of a skipped expert were written"
            continue
        w13, w2 = orc.dequant_expert(cfg.wfmt, L.expert(0, e), cfg.hidden, cfg.ffn)
        ref = np.stack([orc.expert_ffn(w13, w2, xf[r]) for r in range(r0, r1)])
        err = rel_l2(yg[r0:r1], ref)
        worst = max(worst, err)
        assert err < TOL_REL_L2, (e, err)
    return worst


SMALL = dict(hidden=256, ffn=256, experts=8, top_k=2, layers=1)


@pytest.mark.parametrize("base", [W.TINY, W.DS_DECODE, W.TRACE40], ids=["bf16", "mxfp4", "nvfp4"])
@pytest.mark.parametrize("passes", [1, 2])
def test_grouped_ffn_ragged(orc, base, passes):
    cfg = W.scaled(base, **SMALL)
    counts = [0, 1, 7, 8, 9, 33, 70, 3]
    slots = [3, 9, 0, -1, 5, 2, 7, 1]        # permuted, one expert not resident
    worst = _ffn_case(orc, cfg, counts, slots, pool_slots=10, passes=passes)
    assert worst < ALARM_REL_L2, worst


@pytest.mark.parametrize("base", [W.DS_DECODE, W.TRACE40, W.QWEN_BF16], ids=["mxfp4", "nvfp4", "bf16"])
def test_grouped_ffn_full_size(orc, base):
    """Full expert shapes (H, F of the workload), decode-like group sizes."""
    cfg = W.scaled(base, experts=6, top_k=2, layers=1)
    counts = [1, 0, 2, 16, 5, 1]
    slots = [4, 1, 0, 2, 5, 3]
    worst = _ffn_case(orc, cfg, counts, slots, pool_slots=6, seed=3)
    assert worst < ALARM_REL_L2, worst


@pytest.mark.parametrize("base", [W.DS_DECODE, W.TRACE40, W.QWEN_BF16], ids=["mxfp4", "nvfp4", "bf16"])
@pytest.mark.parametrize("passes", [1, 2])
def test_grouped_ffn_split_k(orc, base, passes, monkeypatch):
    """Full expert shapes with decode tiles: the units' K chunks are cut into
    equal ranges over the CTAs and the pieces added up; rows of a skipped
    expert stay untouched, and a second pass over the other experts keeps the
    first's."""
    monkeypatch.setenv("MOE_FFN_TILE", "decode")
    cfg = W.scaled(base, experts=6, top_k=2, layers=1)
    counts = [1, 3, 2, 9, 0, 1]
    slots = [4, -1, 0, 2, 5, 3]
    worst = _ffn_case(orc, cfg, counts, slots, pool_slots=6, seed=5, passes=passes)
    assert worst < ALARM_REL_L2, worst
    assert A.L.lib.moe_get_device_error(1) == 0


def test_grouped_ffn_slot_out_of_range_is_skipped(orc):
    cfg = W.scaled(W.DS_DECODE, **SMALL)
    counts = [2, 2, 0, 0, 0, 0, 0, 1]
    slots = [0, 50, -1, -1, -1, -1, -1, 1]   # 50 >= pool_slots: skipped, not read
    _ffn_case(orc, cfg, counts, slots, pool_slots=2)


# ------------------------------------------------------------------ activation terms
@pytest.mark.parametrize("xd", ["bf16", "f32"])
@pytest.mark.parametrize("terms", [3, 4])
@pytest.mark.parametrize("wfmt", [W.W_MXFP4, W.W_NVFP4], ids=["mxfp4", "nvfp4"])
def test_act_terms_bit_exact(orc, wfmt, terms, xd):
    """The FP4 path's activation encoding (codes, block scales, row exponent)
    is bit-exact with the oracle's: both take every rounding decision in fp32."""
    rng = np.random.default_rng(10 * wfmt + terms)
    n, K = 12, 1024
    x = rng.standard_normal((n, K)).astype(np.float32)
    x[1] *= np.float32(1e-6)
    x[2] *= np.float32(1e5)
    x[3, ::3] = 0.0
    x[4] = np.round(x[4] * 4) / 4                     # exact ties on the grids
    x[5] = 0.0
    x[6] = (rng.standard_normal(K) * 3).astype(np.float32) ** 3   # heavy tails, like h
    x[7, :512] *= np.float32(1e-4)                    # blocks far below the row maximum
    xo = W.f32_to_bf16_bits(x) if xd == "bf16" else x
    vs = 32 if wfmt == W.W_MXFP4 else 16
    codes = torch.empty(n, terms, K, dtype=torch.uint8, device="cuda")
    scales = torch.empty(n, terms, K // vs, dtype=torch.uint8, device="cuda")
    rex = torch.empty(n, dtype=torch.int32, device="cuda")
    A.moe_act_terms(dev(xo), n, K, wfmt, terms, codes, scales, rex)
    torch.cuda.synchronize()
    c_ref, s_ref, p_ref = orc.act_terms(xo, wfmt, terms)
    np.testing.assert_array_equal(host(rex), p_ref)
    np.testing.assert_array_equal(host(scales), s_ref)
    np.testing.assert_array_equal(host(codes), c_ref)


# ------------------------------------------------------------------ combine
@pytest.mark.parametrize("n,k,H,out", [(64, 2, 256, "f32"), (16, 6, 4096, "bf16"), (37, 8, 2048, "bf16")])
def test_combine_parity(orc, n, k, H, out):
    rng = np.random.default_rng(n)
    yb = W.f32_to_bf16_bits(rng.standard_normal((n * k, H)).astype(np.float32) * 100)
    perm = rng.permutation(n * k).astype(np.int32)       # row_of
    w = rng.random((n, k)).astype(np.float32)
    w /= w.sum(1, keepdims=True)
    ref_rows = W.bf16_bits_to_f32(yb).astype(np.float64)[perm]   # assignment order
    ref = orc.combine(ref_rows, w.astype(np.float64))
    o = torch.empty(n, H, dtype=torch.float32 if out == "f32" else torch.bfloat16, device="cuda")
    A.moe_combine(dev(yb), dev(perm), dev(w), n, k, H, o)
    torch.cuda.synchronize()
    err = rel_l2(host(o), ref)
    assert err < (1e-6 if out == "f32" else 4e-3), err
    # deterministic: a second run is bitwise identical
    o2 = torch.empty_like(o)
    A.moe_combine(dev(yb), dev(perm), dev(w), n, k, H, o2)
    torch.cuda.synchronize()
    assert torch.equal(o.view(torch.int16) if o.dtype == torch.bfloat16 else o,
                       o2.view(torch.int16) if o2.dtype == torch.bfloat16 else o2)


TC_CASES = {
    # ragged groups, an expert of 300 rows (five token groups) and one of 256
    "ragged": ([0, 1, 17, 300, 33, 70, 3, 256], [3, 9, 0, 4, 5, 2, 7, 1]),
    # token-group boundaries: one full group, one row over, two full groups, one over
    "block_edges": ([64, 65, 128, 129, 16, 15, 1, 0], [1, 0, 3, 2, 5, 4, 7, 6]),
}


@pytest.mark.parametrize("case", sorted(TC_CASES))
@pytest.mark.parametrize("base", [W.DS_DECODE, W.TRACE40], ids=["mxfp4", "nvfp4"])
def test_grouped_ffn_prefill_tiles(orc, base, case, monkeypatch):
    """The block-scaled grouped GEMM with prefill tiles (64 tokens x 3 terms per
    tile, whole units), forced on small shapes: ragged groups, several token
    groups per expert, and group sizes on and around the tile edge."""
    monkeypatch.setenv("MOE_FFN_TILE", "prefill")
    cfg = W.scaled(base, hidden=256, ffn=256, experts=8, top_k=2, layers=1)
    counts, slots = TC_CASES[case]
    worst = _ffn_case(orc, cfg, counts, slots, pool_slots=10, seed=11)
    assert worst < ALARM_REL_L2, worst
    assert A.L.lib.moe_get_device_error(1) == 0


# ------------------------------------------------------------------ self-consistency
def _ffn_run(cfg, blobs, counts, xb, path, monkeypatch):
    """y of one moe_grouped_ffn call with expert e in slot e (blobs: host uint8 arrays)."""
    monkeypatch.setenv("MOE_FFN_TILE", path)
    shape = A.shape_of(cfg)
    sb = A.moe_slot_bytes(shape)
    pool = torch.from_numpy(np.concatenate(blobs)).to("cuda")
    rows = int(sum(counts))
    offsets = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    slots = np.arange(cfg.experts, dtype=np.int32)
    y = torch.empty(rows, cfg.hidden, dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(A.moe_ffn_workspace_bytes(shape, rows), dtype=torch.uint8, device="cuda")
    torch.cuda.synchronize()
    A.moe_grouped_ffn(shape, pool, cfg.experts, dev(slots), dev(offsets), dev(xb), rows, y, ws)
    torch.cuda.synchronize()
    assert pool.numel() == cfg.experts * sb
    return y.view(torch.int16).cpu().numpy()


@pytest.mark.parametrize("path,counts", [("decode", [1, 3, 2, 9, 0, 1]), ("prefill", [40, 3, 200, 9, 0, 70])],
                         ids=["decode_tiles", "prefill_tiles"])
def test_ffn_is_deterministic_and_scale_exact(path, counts, monkeypatch):
    """Two calls on the same inputs give the same bits (no atomics in any sum),
    and raising every W2 block-scale code by one doubles y exactly (power-of-two
    scaling commutes with every rounding step)."""
    cfg = W.scaled(W.DS_DECODE, experts=6, top_k=2, layers=1)
    shape = A.shape_of(cfg)
    experts = [W.gen_expert(cfg, 4, 0, e) for e in range(cfg.experts)]
    blobs = [A.moe_pack_expert(shape, ew) for ew in experts]
    rng = np.random.default_rng(9)
    xb = W.f32_to_bf16_bits(rng.standard_normal((int(sum(counts)), cfg.hidden)).astype(np.float32))
    y1 = _ffn_run(cfg, blobs, counts, xb, path, monkeypatch)
    y2 = _ffn_run(cfg, blobs, counts, xb, path, monkeypatch)
    np.testing.assert_array_equal(y1, y2)
    for ew in experts:
        ew.w2_scales = (ew.w2_scales + 1).astype(np.uint8)
    blobs2 = [A.moe_pack_expert(shape, ew) for ew in experts]
    y3 = _ffn_run(cfg, blobs2, counts, xb, path, monkeypatch)
    f1 = W.bf16_bits_to_f32(y1.view(np.uint16))
    f3 = W.bf16_bits_to_f32(y3.view(np.uint16))
    np.testing.assert_array_equal(f3, 2 * f1)


@pytest.mark.parametrize("base", [W.DS_DECODE, W.TRACE40], ids=["mxfp4", "nvfp4"])
def test_fused_decode_ffn_matches_the_separate_kernels_bitwise(base, monkeypatch):
    """The fused decode kernel encodes x and h itself (two items per warp,
    interleaved; NVFP4 row exponents once per row a warp meets); the separate
    decode-tile kernels take both encodings from fp4_terms_kernel, whose codes
    are bit-exact with the oracle (test_act_terms_bit_exact).  With the same
    stream-K split the two paths must give the same bits, at full expert size,
    for ragged groups, single rows, and rows of every expert."""
    monkeypatch.setenv("MOE_FFN_TILE", "decode")
    cfg = W.scaled(base, experts=6, top_k=2, layers=1)
    shape = A.shape_of(cfg)
    blobs = [A.moe_pack_expert(shape, W.gen_expert(cfg, 11, 0, e)) for e in range(cfg.experts)]
    rng = np.random.default_rng(21)
    for counts in ([1, 3, 2, 9, 0, 1], [16, 0, 1, 5, 12, 2], [1, 0, 0, 0, 0, 0], [4, 4, 4, 4, 4, 4]):
        x = rng.standard_normal((int(sum(counts)), cfg.hidden)).astype(np.float32)
        x[0] *= 1e-3                                  # a row far below the others (NVFP4 row exponent)
        xb = W.f32_to_bf16_bits(x)
        monkeypatch.delenv("MOE_FFN_UNFUSED", raising=False)
        y_fused = _ffn_run(cfg, blobs, counts, xb, "decode", monkeypatch)
        monkeypatch.setenv("MOE_FFN_UNFUSED", "1")
        y_sep = _ffn_run(cfg, blobs, counts, xb, "decode", monkeypatch)
        np.testing.assert_array_equal(y_fused, y_sep)
        assert A.L.lib.moe_get_device_error(1) == 0


def test_fused_decode_layer_matches_the_separate_kernels_bitwise(monkeypatch):
    """The same through moe_layer_forward, where the fused kernel gathers x rows
    from the tokens (a token routed to k experts is one source row of k items)."""
    cfg = W.scaled(W.TRACE40, experts=32, top_k=4, layers=1, capacity=32)
    Ly = Layer(cfg, 13)
    wg, bias = dev(W.gen_wg(cfg, 13, 0)), dev(W.gen_bias(cfg, 13, 0, 0))
    outs = []
    for unfused in (False, True):
        if unfused:
            monkeypatch.setenv("MOE_FFN_UNFUSED", "1")
        else:
            monkeypatch.delenv("MOE_FFN_UNFUSED", raising=False)
        cache = make_cache(Ly)
        res = []
        for s in range(3):
            x = dev(W.gen_x(cfg, 13, 16, "decode", s))
            out = torch.empty(16, cfg.hidden, dtype=torch.bfloat16, device="cuda")
            ws = torch.empty(A.moe_layer_workspace_bytes(Ly.shape, 16), dtype=torch.uint8, device="cuda")
            A.moe_layer_forward(cache, 0, x, wg, bias, out, ws)
            torch.cuda.synchronize()
            res.append(host(out))
        outs.append(res)
        cache.close()
    for a, b in zip(*outs):
        np.testing.assert_array_equal(a, b)
