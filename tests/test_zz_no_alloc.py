"""osp_attn_full_noalloc: the attention entry point for callers that cannot allocate device
memory (their memory belongs to another allocator's pool, or cudaMalloc's device-wide
synchronisation is not acceptable on their path).  Its scratch is a static device array, so it
must give the same output as osp_attn_full, call after call, with no allocation of its own.

This file is named to be collected last: if it fails, a run that stops at the first failure has
already run every other test.  It passes on its own in a fresh process and after the others."""

import ctypes

import pytest
import torch

from spacetime_attention_b200 import ops, synthetic as syn
from tests.gpu_common import gpu  # noqa: F401
from tests.helpers import ATTN_MAX_ABS, ATTN_REL_L2, attn_errors, to_f64

pytestmark = pytest.mark.gpu


def _call(lib, fn, q, k, v, o, shape, stream):
    rc = getattr(lib, fn)(ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(k.data_ptr()),
                          ctypes.c_void_p(v.data_ptr()), ctypes.c_void_p(o.data_ptr()), ctypes.byref(shape),
                          ctypes.c_float(0.0), ctypes.c_void_p(stream))
    assert rc == 0, f"{fn}: {lib.osp_get_last_error().decode()}"


@pytest.mark.parametrize("B,heads,d,grid,L", [(1, 3, 64, (4, 8, 8), 44), (2, 2, 128, (2, 9, 19), 0),
                                              (1, 2, 96, (3, 7, 13), 5)])
def test_noalloc_matches_osp_attn_full_twice(gpu, B, heads, d, grid, L):
    lib = ops.library()
    w = syn.custom("na", B, heads, d, grid, L, (d // 4, d // 4 + d // 8, d - d // 2 - d // 8))
    q, k, v = (t.to(gpu) for t in syn.make_qkv(w, 21))
    shape = ops.make_shape(B, L, grid, heads, d)
    stream = torch.cuda.current_stream(gpu).cuda_stream
    ref = torch.empty_like(q)
    _call(lib, "osp_attn_full", q, k, v, ref, shape, stream)
    outs = []
    for _ in range(2):   # two calls in a row share the static scratch
        o = torch.full_like(q, float("nan"))
        _call(lib, "osp_attn_full_noalloc", q, k, v, o, shape, stream)
        outs.append(o)
    torch.cuda.synchronize()
    for o in outs:
        mx, rl = attn_errors(o, to_f64(ref))
        assert mx <= ATTN_MAX_ABS and rl <= ATTN_REL_L2, (mx, rl)
        assert torch.equal(o, ref)   # same kernel, same inputs: bit-identical


def test_noalloc_allocates_no_torch_memory_and_rejects_bad_args(gpu):
    lib = ops.library()
    w = syn.custom("na", 1, 2, 64, (2, 8, 8), 0, (16, 24, 24))
    q, k, v = (t.to(gpu) for t in syn.make_qkv(w, 22))
    o = torch.empty_like(q)
    shape = ops.make_shape(1, 0, (2, 8, 8), 2, 64)
    stream = torch.cuda.current_stream(gpu).cuda_stream
    _call(lib, "osp_attn_full_noalloc", q, k, v, o, shape, stream)
    torch.cuda.synchronize()
    before = torch.cuda.memory_allocated(gpu)
    _call(lib, "osp_attn_full_noalloc", q, k, v, o, shape, stream)
    torch.cuda.synchronize()
    assert torch.cuda.memory_allocated(gpu) == before
    bad = ops.make_shape(1, 0, (2, 8, 8), 2, 80)
    p = ctypes.c_void_p(q.data_ptr())
    assert lib.osp_attn_full_noalloc(p, p, p, p, ctypes.byref(bad), ctypes.c_float(0.0), None) == 2
    assert lib.osp_attn_full_noalloc(None, p, p, p, ctypes.byref(shape), ctypes.c_float(0.0), None) == 1
