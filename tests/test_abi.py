"""The C-ABI library builds, loads without a GPU, exports every symbol include/osp.h declares,
and rejects bad arguments on the host before touching the device."""

import ctypes
import os
import re

import pytest

from spacetime_attention_b200 import build as B
from spacetime_attention_b200 import ops

HEADER = os.path.join(B.INCLUDE, "osp.h")


@pytest.fixture(scope="module")
def lib():
    B.build()
    return ops.library()


def declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^\s*(?:int|const char\*)\s+(osp_\w+)\s*\(", text, re.M)))


def test_header_declares_the_boundary():
    names = declared_symbols()
    for n in ("osp_rope3d", "osp_attn_full", "osp_skiparse_gather", "osp_skiparse_scatter", "osp_skiparse_attn",
              "osp_skiparse_index_map", "osp_check_status", "osp_get_last_error"):
        assert n in names
    assert set(names) == set(ops.EXPORTED)


def test_library_exports_every_declared_symbol(lib):
    for n in declared_symbols():
        assert hasattr(lib, n), n
    assert lib.osp_version() >= 100


def shp(B=1, L=0, T=4, H=8, W=8, heads=2, d=64):
    return ctypes.byref(ops.OspShape(B, L, T, H, W, heads, d))


def rc_msg(lib, rc):
    return rc, lib.osp_get_last_error().decode()


@pytest.mark.parametrize("args,code", [
    (dict(B=0), 1), (dict(T=0), 1), (dict(heads=0), 1), (dict(L=-1), 1), (dict(d=80), 2), (dict(d=60), 2)])
def test_attention_rejects_bad_shapes(lib, args, code):
    p = ctypes.c_void_p(256)
    rc, msg = rc_msg(lib, lib.osp_attn_full(p, p, p, p, shp(**args), 0.0, None))
    assert rc == code and msg


def test_rejects_null_and_misaligned(lib):
    p, bad = ctypes.c_void_p(256), ctypes.c_void_p(258)
    assert lib.osp_attn_full(None, p, p, p, shp(), 0.0, None) == 1
    assert lib.osp_attn_full(p, p, bad, p, shp(), 0.0, None) == 1
    assert "aligned" in lib.osp_get_last_error().decode()


def test_rope_split_validation(lib):
    p = ctypes.c_void_p(256)
    for split, code in [((16, 24, 16), 1), ((15, 25, 24), 1), ((-2, 34, 32), 1)]:
        r = ops.make_rope(split)
        assert lib.osp_rope3d(p, p, p, p, shp(), ctypes.byref(r), None) == code
    r = ops.make_rope((16, 24, 24), theta=0.0)
    assert lib.osp_rope3d(p, p, p, p, shp(), ctypes.byref(r), None) == 1
    assert lib.osp_rope3d(p, p, p, p, shp(), None, None) == 1


def test_skiparse_validation(lib):
    p = ctypes.c_void_p(256)
    # text tokens: gather / scatter take video tokens only; Skiparse attention still checks k
    assert lib.osp_skiparse_gather(p, p, p, p, p, p, shp(L=3), 2, 0, None, None) == 2
    assert lib.osp_skiparse_attn(p, p, p, p, shp(L=3), 3, 0, 0.0, None) == 3
    # 4*8*8 = 256 not divisible by 3 / by 9
    assert lib.osp_skiparse_attn(p, p, p, p, shp(), 3, 0, 0.0, None) == 3
    assert lib.osp_skiparse_gather(p, p, p, p, p, p, shp(T=3, H=3, W=3), 2, 1, None, None) == 3
    # group needs k | 128 in the fused kernel
    assert lib.osp_skiparse_attn(p, p, p, p, shp(T=9, H=6, W=6), 3, 1, 0.0, None) == 2
    assert lib.osp_skiparse_attn(p, p, p, p, shp(), 0, 0, 0.0, None) == 1
    assert lib.osp_skiparse_attn(p, p, p, p, shp(), 2, 7, 0.0, None) == 1
    assert lib.osp_skiparse_index_map(10, 4, 0, p, None) == 3
    assert lib.osp_skiparse_index_map(16, 2, 1, None, None) == 1
    assert lib.osp_skiparse_gather(p, p, None, p, None, None, shp(), 2, 0, None, None) == 1  # k w/o k_out
    assert lib.osp_skiparse_scatter(None, p, shp(), 2, 0, None) == 1


def test_binding_refuses_non_cuda_tensors():
    import torch
    x = torch.zeros(1, 256, 2, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        ops.attn_full(x, x, x, (4, 8, 8), 0)


def _i32(vals):
    return (ctypes.c_int32 * len(vals))(*vals)


def test_packed_attention_validation(lib):
    p = ctypes.c_void_p(256)
    ok = _i32([0, 5, 9])
    call = lambda qb, kb, n, heads=2, d=64: lib.osp_attn_packed(p, p, p, p, qb, kb, n, heads, d, 0.0, None)
    assert call(ok, None, 0) == 1                       # no segments
    assert call(ok, None, 257) == 2                     # more than OSP_MAX_SEGMENTS
    assert call(None, None, 2) == 1                     # no bounds
    assert call(_i32([1, 5, 9]), None, 2) == 1          # must start at 0
    assert call(_i32([0, 5, 4]), None, 2) == 1          # decreasing
    assert "decreases" in lib.osp_get_last_error().decode()
    assert call(ok, _i32([0, 3, 3]), 2) == 1            # sample 1: 4 queries, no keys
    assert "no key rows" in lib.osp_get_last_error().decode()
    assert call(ok, None, 2, d=80) == 2
    assert call(ok, None, 2, heads=0) == 1
    assert lib.osp_attn_packed(None, p, p, p, ok, None, 2, 2, 64, 0.0, None) == 1
    assert lib.osp_attn_packed(p, p, p, ctypes.c_void_p(260), ok, None, 2, 2, 64, 0.0, None) == 1


def test_packed_rope_validation(lib):
    p = ctypes.c_void_p(256)
    r = ops.make_rope((16, 24, 24))
    grids = (ops.OspSampleGrid * 2)(ops.OspSampleGrid(3, 2, 4, 4), ops.OspSampleGrid(0, 1, 0, 5))
    assert lib.osp_rope3d_packed(p, p, p, p, grids, 2, 2, 64, ctypes.byref(r), None) == 1   # H = 0
    assert "sample 1" in lib.osp_get_last_error().decode()
    assert lib.osp_rope3d_packed(p, p, p, p, grids, 0, 2, 64, ctypes.byref(r), None) == 1
    assert lib.osp_rope3d_packed(p, p, p, p, None, 1, 2, 64, ctypes.byref(r), None) == 1
    bad = ops.make_rope((16, 24, 16))
    assert lib.osp_rope3d_packed(p, p, p, p, grids, 1, 2, 64, ctypes.byref(bad), None) == 1


def test_factorized_validation(lib):
    p = ctypes.c_void_p(256)
    assert lib.osp_attn_spatial(p, p, p, p, shp(L=4), 0.0, None) == 2          # text not allowed
    assert lib.osp_attn_temporal(p, p, p, p, shp(L=4), 0, 0.0, None) == 2
    assert lib.osp_attn_temporal(p, p, p, p, shp(), 2, 0.0, None) == 1          # causal must be 0/1
    assert lib.osp_attn_temporal(p, p, p, p, shp(d=80), 0, 0.0, None) == 2
    assert lib.osp_attn_frame_causal(None, p, p, p, shp(), 0.0, None) == 1
    assert lib.osp_attn_frame_causal(p, p, p, p, shp(d=60), 0.0, None) == 2


def test_training_validation(lib):
    p, bad = ctypes.c_void_p(256), ctypes.c_void_p(264)
    assert lib.osp_attn_forward_train(p, p, p, p, None, shp(), 1, 0, 0.0, None) == 1          # no lse
    assert lib.osp_attn_forward_train(p, p, p, p, bad, shp(), 1, 0, 0.0, None) == 1           # misaligned lse
    assert lib.osp_attn_forward_train(p, p, p, p, p, shp(L=3), 3, 0, 0.0, None) == 3          # Skiparse + text, 256 % 3
    assert lib.osp_attn_forward_train(p, p, p, p, p, shp(), 3, 0, 0.0, None) == 3             # 256 % 3
    assert lib.osp_attn_backward(p, p, p, p, p, p, p, p, None, shp(), 1, 0, 0.0, None) == 1   # no dv
    assert lib.osp_attn_backward(p, p, p, p, p, p, p, p, p, shp(d=80), 1, 0, 0.0, None) == 2


def test_frame_causal_training_validation(lib):
    p = ctypes.c_void_p(256)
    assert lib.osp_attn_frame_causal_train(p, p, p, p, None, shp(), 0.0, None) == 1
    assert lib.osp_attn_frame_causal_backward(p, p, p, p, p, p, p, p, None, shp(), 0.0, None) == 1
    assert lib.osp_attn_frame_causal_backward(p, p, p, p, p, p, p, p, p, shp(d=80), 0.0, None) == 2


def test_factorized_training_validation(lib):
    p, bad = ctypes.c_void_p(256), ctypes.c_void_p(264)
    assert lib.osp_attn_spatial_train(p, p, p, p, None, shp(), 0.0, None) == 1               # no lse
    assert lib.osp_attn_spatial_train(p, p, p, p, bad, shp(), 0.0, None) == 1                # misaligned lse
    assert lib.osp_attn_spatial_train(p, p, p, p, p, shp(L=2), 0.0, None) == 2               # text not allowed
    assert lib.osp_attn_spatial_backward(p, p, p, p, p, p, p, None, p, shp(), 0.0, None) == 1
    assert lib.osp_attn_spatial_backward(p, p, p, p, p, p, p, p, p, shp(d=80), 0.0, None) == 2
    assert lib.osp_attn_temporal_train(p, p, p, p, p, shp(), 2, 0.0, None) == 1             # causal must be 0/1
    assert lib.osp_attn_temporal_train(p, p, p, p, p, shp(L=1), 0, 0.0, None) == 2
    assert lib.osp_attn_temporal_backward(p, p, p, p, p, p, p, p, p, shp(), -1, 0.0, None) == 1
    assert lib.osp_attn_temporal_backward(p, p, p, p, p, p, p, p, bad, shp(), 1, 0.0, None) == 1
    assert lib.osp_attn_temporal_backward(p, p, p, p, p, p, p, p, p, shp(d=60), 0, 0.0, None) == 2


def test_binding_checks_the_lse_buffer():
    import torch
    q = torch.zeros((1, 32, 2, 64), dtype=torch.bfloat16)
    assert ops.factorized_lse_shape(q, (4, 2, 4), temporal=False) == (4, 2, 128)
    assert ops.factorized_lse_shape(q, (4, 2, 4), temporal=True) == (8, 2, 128)
    with pytest.raises(ValueError):
        ops._lse_buffer(torch.zeros(10), (4, 2, 128), q)                  # too small
    with pytest.raises(ValueError):
        ops._lse_buffer(torch.zeros((4, 2, 128), dtype=torch.float64), (4, 2, 128), q)
    buf = torch.zeros((4, 2, 128))
    assert ops._lse_buffer(buf, (4, 2, 128), q) is buf


def test_binding_shape_checks():
    # the library sizes every access from the shape struct alone, so the bindings compare the
    # tensors with it before any call
    import torch
    bf = torch.bfloat16
    q = torch.zeros((2, 3 + 4 * 2 * 2, 2, 64), dtype=bf)
    assert ops._shape_of(q, (4, 2, 2), 3).T == 4
    with pytest.raises(ValueError, match="text_len"):
        ops._shape_of(q, (4, 2, 2), 0)                 # 16 video tokens + 0 != 19
    with pytest.raises(ValueError, match="text_len"):
        ops._shape_of(q, (5, 2, 2), 3)
    with pytest.raises(ValueError, match="shape"):
        ops._same(torch.zeros((2, 18, 2, 64), dtype=bf), q, "k")     # one token short
    with pytest.raises(ValueError, match="shape"):
        ops._same(torch.zeros((2, 19, 1, 64), dtype=bf), q, "v")     # other head count
    with pytest.raises(ValueError, match="shape"):
        ops._out(torch.zeros((1, 19, 2, 64), dtype=bf), q, "o")
    with pytest.raises(ValueError, match="CUDA"):
        ops._same(torch.zeros_like(q), q, "k")        # right shape, but on the host
    with pytest.raises(ValueError):
        ops._heads_match(torch.zeros((2, 7, 2, 32), dtype=bf), q, "k")
    with pytest.raises(ValueError, match="CUDA"):
        ops._heads_match(torch.zeros((2, 7, 2, 64), dtype=bf), q, "k")   # any token count
    assert ops._packed_rows([(13, 2, 5, 7), (0, 3, 8, 8), (77, 1, 4, 4)]) == 83 + 192 + 93
