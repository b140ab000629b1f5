"""moe_permute_noalloc -- the variant of moe_permute that allocates nothing --
against moe_permute itself, through the C ABI, on two calls in a row.

The variant exists for callers that cannot allocate device memory of their
own (a host framework that owns every byte of GPU memory, or a serving loop
that must never enter the CUDA allocator).  Its scratch is one static array
inside the library that every call shares, so the two calls below use
different sizes and inputs: anything left over from the first call that the
second one wrongly relied on would show up as a mismatch.  Both calls take the
multi-kernel path (more than 1024 assignments), the one that uses scratch.
Outputs are integers and copied bf16 rows, compared bit for bit.
"""
import numpy as np
import pytest
import torch

from expert_cached_sparse_b200 import api as A
from expert_cached_sparse_b200 import workloads as W

pytestmark = pytest.mark.gpu

CASES = [(4096, 256, 6, 256, 21), (1500, 128, 8, 512, 22)]   # n, experts, k, hidden, seed


def _inputs(n, E, k, H, seed):
    rng = np.random.default_rng(seed)
    idx = np.minimum(E - 1, rng.zipf(1.2, size=(n, k)) - 1).astype(np.int32)
    x = W.f32_to_bf16_bits(rng.standard_normal((n, H)).astype(np.float32))
    return (torch.from_numpy(idx).cuda(), torch.from_numpy(x.view(np.int16)).cuda().view(torch.bfloat16))


def _outputs(n, E, k, H):
    return (torch.full((E + 1,), -7, dtype=torch.int32, device="cuda"),
            torch.full((n * k,), -7, dtype=torch.int32, device="cuda"),
            torch.full((n * k,), -7, dtype=torch.int32, device="cuda"),
            torch.zeros(n * k, H, dtype=torch.bfloat16, device="cuda"))


def test_noalloc_permute_matches_workspace_permute_on_two_calls():
    for n, E, k, H, seed in CASES:
        idx, x = _inputs(n, E, k, H, seed)
        ref = _outputs(n, E, k, H)
        ws = torch.empty(A.moe_permute_workspace_bytes(n, E, k), dtype=torch.uint8, device="cuda")
        A.moe_permute(idx, n, E, k, x, H, *ref, ws)
        got = _outputs(n, E, k, H)
        A.moe_permute_noalloc(idx, n, E, k, x, H, *got)
        torch.cuda.synchronize()
        for r, g in zip(ref[:3], got[:3]):
            assert torch.equal(r, g)
        assert torch.equal(ref[3].view(torch.int16), got[3].view(torch.int16))


def test_noalloc_permute_rejects_sizes_beyond_its_scratch():
    n, E, k, H = 200_000, 256, 6, 64          # the rank array alone exceeds the static scratch
    assert A.moe_permute_workspace_bytes(n, E, k) > (1 << 20)
    # placeholders: the size check refuses the call before any buffer is touched
    i32 = torch.zeros(16, dtype=torch.int32, device="cuda")
    b16 = torch.zeros(16, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(A.MoeError) as e:
        A.moe_permute_noalloc(i32, n, E, k, b16, H, i32, i32, i32, b16)
    assert e.value.code == A.L.MOE_ERR_UNSUPPORTED
