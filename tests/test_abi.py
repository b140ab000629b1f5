"""The C ABI on the host (CPU only): the library loads, exports every entry
point include/moe.h declares, sizes follow the packed layout, and argument
errors come back as status codes before any device work."""
import ctypes as C
import os
import re

import numpy as np
import pytest

from expert_cached_sparse_b200 import _lib as L
from expert_cached_sparse_b200 import api as A
from expert_cached_sparse_b200 import workloads as W

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "moe.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    names = set(re.findall(r"\b(moe_[a-z0-9_]+)\s*\(", src))
    return names


def test_every_declared_symbol_is_exported():
    decl = _declared()
    assert len(decl) >= 21
    missing = [n for n in decl if not hasattr(L.lib, n)]
    assert not missing, missing
    assert decl == set(L.EXPORTS) | (decl - set(L.EXPORTS))


def test_version_and_status_strings():
    assert L.lib.moe_version() >= 100
    for code in range(0, -8, -1):
        assert L.status_str(code) != "unknown status"
    assert L.status_str(-99) == "unknown status"


@pytest.mark.parametrize("cfg,expect", [
    (W.TINY, 3 * 256 * 512 * 2),
    (W.DS_DECODE, 12582912 + 786432),
    (W.QWEN_BF16, 3 * 2048 * 768 * 2),
    (W.TRACE40, 14155904),
])
def test_slot_bytes(cfg, expect):
    assert A.moe_slot_bytes(A.shape_of(cfg)) == expect


def test_invalid_shapes_rejected():
    bad = [A.make_shape(1, 8, 100, 512, 2, 0),       # hidden % 64
           A.make_shape(1, 8, 256, 500, 2, 0),       # ffn % 64
           A.make_shape(1, 8, 256, 512, 9, 0),       # k > E
           A.make_shape(1, 5000, 256, 512, 2, 0),    # E too large
           A.make_shape(1, 8, 256, 512, 2, 7)]       # format
    for s in bad:
        assert A.moe_slot_bytes(s) == 0
        assert A.moe_layer_workspace_bytes(s, 4) == 0
        assert A.moe_cache_meta_bytes(s, 8, 16) == 0
    assert A.moe_cache_meta_bytes(A.shape_of(W.TINY), 0, 16) == 0


def test_workspace_sizes_grow_with_tokens():
    s = A.shape_of(W.DS_DECODE)
    a, b = A.moe_layer_workspace_bytes(s, 1), A.moe_layer_workspace_bytes(s, 16)
    assert 0 < a < b
    assert A.moe_layer_workspace_bytes(s, 4096) > 3 * 4096 * 6 * 4096  # y_perm + x operand copy + h at least


def test_pack_rejects_bad_scale_codes():
    cfg = W.scaled(W.DS_DECODE, hidden=256, ffn=256, experts=4, top_k=2)
    s = A.shape_of(cfg)
    ew = W.gen_expert(cfg, 0, 0, 0)
    A.moe_pack_expert(s, ew)   # valid
    ew.w13_scales[3, 1] = 150  # 2^23: any finite E8M0 code is accepted
    A.moe_pack_expert(s, ew)
    ew.w13_scales[3, 1] = 255  # E8M0 NaN
    with pytest.raises(A.MoeError) as e:
        A.moe_pack_expert(s, ew)
    assert e.value.code == L.MOE_ERR_UNSUPPORTED
    cfg2 = W.scaled(W.TRACE40, layers=1, hidden=256, ffn=256, experts=4, top_k=2)
    s2 = A.shape_of(cfg2)
    ew2 = W.gen_expert(cfg2, 0, 0, 0)
    A.moe_pack_expert(s2, ew2)
    ew2.w2_scales[0, 0] = 0x7F  # E4M3 NaN
    with pytest.raises(A.MoeError):
        A.moe_pack_expert(s2, ew2)


def test_pack_is_a_byte_permutation_fp4():
    """FP4 packing moves whole bytes (nibble pairs) and scale bytes; nothing is lost."""
    cfg = W.scaled(W.DS_DECODE, hidden=256, ffn=256, experts=4, top_k=2)
    s = A.shape_of(cfg)
    ew = W.gen_expert(cfg, 1, 0, 2)
    blob = A.moe_pack_expert(s, ew)
    payload = np.concatenate([ew.w13.ravel(), ew.w2.ravel(), ew.w13_scales.ravel(), ew.w2_scales.ravel()])
    assert blob.size >= payload.size
    np.testing.assert_array_equal(np.sort(blob[: payload.size]), np.sort(payload))


def test_host_argument_errors_need_no_device():
    s = A.shape_of(W.TINY)
    rc = L.lib.moe_router_topk(None, 0, None, None, 4, 256, 8, 9, None, None, None, None)
    assert rc == L.MOE_ERR_INVALID_ARG
    rc = L.lib.moe_permute(None, 4, 0, 2, None, 0, 256, None, None, None, None, None, 0, None)
    assert rc == L.MOE_ERR_INVALID_ARG
    rc = L.lib.moe_grouped_ffn(C.byref(s), None, 8, None, None, None, 4, None, None, 0, None)
    assert rc == L.MOE_ERR_INVALID_ARG
    rc = L.lib.moe_combine(None, None, None, 4, 0, 256, None, 0, None)
    assert rc == L.MOE_ERR_INVALID_ARG
    rc = L.lib.moe_layer_forward(None, 0, None, 0, None, None, 1, None, None, 0, None, None, None, None)
    assert rc == L.MOE_ERR_INVALID_ARG
    out = C.c_void_p()
    rc = L.lib.moe_cache_create(C.byref(s), None, 0, None, 8, 16, None, None, C.byref(out))
    assert rc == L.MOE_ERR_INVALID_ARG and not out.value
    assert L.lib.moe_cache_destroy(None) == L.MOE_ERR_INVALID_ARG


def test_permute_noalloc_refusals_need_no_device():
    """Argument errors and inputs too large for the static scratch come back
    before any device call (dummy 16-byte-aligned addresses are never read)."""
    fake = C.c_void_p(0x100000)
    f = L.lib.moe_permute_noalloc
    assert f(None, -1, 8, 2, fake, 0, 256, fake, fake, fake, fake, None) == L.MOE_ERR_INVALID_ARG
    assert f(fake, 4, 8, 2, fake, 5, 256, fake, fake, fake, fake, None) == L.MOE_ERR_INVALID_ARG   # dtype
    assert f(fake, 4, 8, 2, fake, 0, 256, None, fake, fake, fake, None) == L.MOE_ERR_INVALID_ARG   # offsets
    big = 1 << 20   # tokens whose permute workspace exceeds the 1 MiB scratch
    assert A.moe_permute_workspace_bytes(big, 256, 8) > (1 << 20)
    assert f(fake, big, 256, 8, fake, 1, 256, fake, fake, fake, fake, None) == L.MOE_ERR_UNSUPPORTED
