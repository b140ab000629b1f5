"""The pooled oracle layer equals the oracle's own layer, bit for bit."""
import numpy as np

from expert_cached_sparse_b200 import workloads as W

from oracle_pool import layer_outputs


def test_pooled_layer_equals_moe_layer(orc):
    cfg = W.scaled(W.TRACE40, layers=3, experts=16, hidden=256, ffn=128, top_k=4)
    distinct = 5
    calls, refs = [], []
    for layer in range(3):
        x = W.gen_x(cfg, 1, 9, "pool", layer)
        wg, bias = W.gen_wg(cfg, 1, layer), W.gen_bias(cfg, 1, layer, 0)
        toks = None if layer != 1 else [0, 3, 8]
        calls.append((layer, x, wg, bias, toks))
        fn = lambda e, layer=layer: W.gen_expert(cfg, 1, *W.blob_alias(cfg, layer, e, distinct))
        refs.append(orc.moe_layer(x, wg, bias, cfg.top_k, cfg.wfmt, cfg.hidden, cfg.ffn, fn, tokens=toks))
    for (out, idx, w), (r_out, r_idx, r_w, _) in zip(layer_outputs(orc, cfg, 1, distinct, calls), refs):
        np.testing.assert_array_equal(idx, r_idx)
        np.testing.assert_array_equal(w, r_w)
        np.testing.assert_array_equal(out, r_out)
