"""The placement study's GPU routing (policy_study.route_trace, through
moe_router_topk) equals the oracle router's routing of the same inputs."""
import numpy as np
import pytest
import torch

from expert_cached_sparse_b200 import policy_study as PS
from expert_cached_sparse_b200 import workloads as W

from helpers import oracle_route_trace

pytestmark = pytest.mark.gpu


def test_route_trace_equals_the_oracle_router(orc):
    cfg = W.TRACE40
    steps, prefill = 40, 16   # two drift epochs (the second one partial)
    d_gpu, p_gpu = PS.route_trace(cfg, steps, prefill, torch.device("cuda", 0))
    d_orc, p_orc = oracle_route_trace(orc, cfg, steps, prefill)
    assert len(d_gpu) == len(d_orc) == steps * cfg.layers
    for (lg, ig), (lo, io) in zip(d_gpu, d_orc):
        assert lg == lo
        np.testing.assert_array_equal(ig, io)
    assert len(p_gpu) == len(p_orc) == cfg.layers
    for (lg, ig), (lo, io) in zip(p_gpu, p_orc):
        assert lg == lo
        np.testing.assert_array_equal(ig, io)
