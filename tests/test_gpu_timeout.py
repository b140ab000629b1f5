"""Bounded device waits that run out, on every grouped-FFN kernel.

moe_test_set_wait shortens the wait limit and makes the first CTA's copy
issuer leave its first ring stage unfilled.  The consumer's wait for that
stage runs out: the kernel must record MOE_ERR_TIMEOUT, let its own copies
and MMAs finish, and return (no fault, no hang, the context stays usable).
A normal call afterwards must give the same bits as one made before.
Nothing here faults the GPU: the withheld stage is simply never filled.
"""
import time

import numpy as np
import pytest
import torch

from expert_cached_sparse_b200 import _lib as L
from expert_cached_sparse_b200 import api as A
from expert_cached_sparse_b200 import workloads as W

from helpers import dev

pytestmark = pytest.mark.gpu

SHORT = 2_000_000   # SM cycles, about 1 ms: far above any wait of these small calls

# (id, base workload, environment) -> kernel
PATHS = [
    ("bf16", W.TINY, {}),                                                             # ffn_kernel
    ("mxfp4_fused", W.DS_DECODE, {}),                                                 # ffn_fp4_fused_kernel
    ("nvfp4_fused", W.TRACE40, {}),                                                   # ffn_fp4_fused_kernel
    ("nvfp4_split", W.TRACE40, {"MOE_FFN_TILE": "decode", "MOE_FFN_UNFUSED": "1"}),   # ffn_fp4_kernel, decode tiles
    ("mxfp4_prefill", W.DS_DECODE, {"MOE_FFN_TILE": "prefill"}),                      # ffn_fp4_kernel, prefill tiles
]


@pytest.fixture
def hook():
    A.moe_test_set_wait(0, False)
    A.moe_get_device_error(clear=True)
    yield
    A.moe_test_set_wait(0, False)
    A.moe_get_device_error(clear=True)


class Call:
    def __init__(self, base):
        self.cfg = cfg = W.scaled(base, hidden=256, ffn=256, experts=8, top_k=2, layers=1)
        self.shape = A.shape_of(cfg)
        blobs = [A.moe_pack_expert(self.shape, W.gen_expert(cfg, 6, 0, e)) for e in range(cfg.experts)]
        self.pool = torch.from_numpy(np.concatenate(blobs)).to("cuda")
        counts = [1, 3, 2, 9, 0, 1, 5, 4]
        self.rows = int(sum(counts))
        self.offsets = dev(np.concatenate([[0], np.cumsum(counts)]).astype(np.int32))
        self.slots = dev(np.arange(cfg.experts, dtype=np.int32))
        rng = np.random.default_rng(13)
        self.x = dev(W.f32_to_bf16_bits(rng.standard_normal((self.rows, cfg.hidden)).astype(np.float32)))
        self.y = torch.empty(self.rows, cfg.hidden, dtype=torch.bfloat16, device="cuda")
        self.ws = torch.empty(A.moe_ffn_workspace_bytes(self.shape, self.rows), dtype=torch.uint8, device="cuda")
        torch.cuda.synchronize()

    def run(self):
        self.y.fill_(0)
        A.moe_grouped_ffn(self.shape, self.pool, self.cfg.experts, self.slots, self.offsets, self.x, self.rows,
                          self.y, self.ws)
        torch.cuda.synchronize()
        return self.y.view(torch.int16).cpu().numpy().copy()


@pytest.mark.parametrize("pid,base,env", PATHS, ids=[p[0] for p in PATHS])
def test_withheld_stage_times_out_and_the_next_call_is_exact(hook, monkeypatch, pid, base, env):
    for k, v in env.items():
        monkeypatch.setenv(k, v)
    c = Call(base)
    y_ref = c.run()
    assert A.moe_get_device_error() == 0
    # a short limit alone changes nothing
    A.moe_test_set_wait(SHORT, False)
    np.testing.assert_array_equal(c.run(), y_ref)
    assert A.moe_get_device_error() == 0
    # a withheld stage: the wait runs out, the kernel drains and returns
    A.moe_test_set_wait(SHORT, True)
    t0 = time.perf_counter()
    c.run()
    dt = time.perf_counter() - t0
    assert A.moe_get_device_error(clear=True) == L.MOE_ERR_TIMEOUT
    assert A.moe_get_device_error() == 0
    assert dt < 1.0, dt   # gave up after the short limit, not the default one
    # back to normal: the same bits as before
    A.moe_test_set_wait(0, False)
    np.testing.assert_array_equal(c.run(), y_ref)
    assert A.moe_get_device_error() == 0


def test_wait_hook_rejects_negative_limits(hook):
    with pytest.raises(A.MoeError) as ei:
        A.moe_test_set_wait(-1, False)
    assert ei.value.code == L.MOE_ERR_INVALID_ARG
