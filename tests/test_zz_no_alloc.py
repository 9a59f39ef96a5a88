"""osp_attn_full_noalloc: the attention entry point for callers that cannot allocate device
memory (their memory belongs to another allocator's pool, or cudaMalloc's device-wide
synchronisation is not acceptable on their path).  Its scratch is a static device array, so it
must give the same output as osp_attn_full, call after call, with no allocation of its own, and
a timeout recorded in that array must reach the caller through osp_check_status, which must not
allocate either.

This file is named to be collected last: if it fails, a run that stops at the first failure has
already run every other test.  It passes on its own in a fresh process and after the others."""

import ctypes

import numpy as np
import pytest
import torch

import oracle as O
from spacetime_attention_b200 import ops, synthetic as syn
from tests.gpu_common import gpu  # noqa: F401
from tests.helpers import ATTN_MAX_ABS, ATTN_REL_L2, assert_attn_close, attn_errors, to_f64

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


def test_noalloc_against_the_oracle_where_osp_attn_full_splits(gpu):
    # 20 heads x 16 query blocks = 320 units on 148 SMs: osp_attn_full splits the last 24 units
    # over KV ranges (workspace + combine kernel); the allocation-free call cannot, and runs its
    # 320 items in turn on one CTA per SM instead.  Both are compared with the fp64 oracle.
    grid, heads = (4, 32, 32), 20
    w = syn.custom("na", 1, heads, 64, grid, 0, (16, 24, 24))
    q, k, v = syn.make_qkv(w, 23)
    qg, kg, vg = (t.to(gpu) for t in (q, k, v))
    lib = ops.library()
    shape = ops.make_shape(1, 0, grid, heads, 64)
    stream = torch.cuda.current_stream(gpu).cuda_stream
    full = torch.empty_like(qg)
    _call(lib, "osp_attn_full", qg, kg, vg, full, shape, stream)
    outs = []
    for _ in range(2):
        o = torch.full_like(qg, float("nan"))
        _call(lib, "osp_attn_full_noalloc", qg, kg, vg, o, shape, stream)
        outs.append(o)
    assert lib.osp_check_status(ctypes.c_void_p(stream)) == 0
    rows = np.arange(0, w.seq_len, 7)
    ref = O.attn_ref(to_f64(q), to_f64(k), to_f64(v), rows=rows)
    for o in (full, *outs):
        assert_attn_close(o[:, rows], ref, "sampled rows")
    assert torch.equal(outs[0], outs[1])


def test_noalloc_timeout_reaches_osp_check_status(gpu, monkeypatch):
    # the kernel's bounded waits run out (Q is never loaded); the static word records it,
    # osp_check_status reports it once and clears it, and the next call is correct
    lib = ops.library()
    grid = (4, 8, 8)
    w = syn.custom("na", 1, 2, 64, grid, 0, (16, 24, 24))
    q, k, v = syn.make_qkv(w, 24)
    qg, kg, vg = (t.to(gpu) for t in (q, k, v))
    shape = ops.make_shape(1, 0, grid, 2, 64)
    stream = torch.cuda.current_stream(gpu).cuda_stream
    st = ctypes.c_void_p(stream)
    o = torch.empty_like(qg)
    _call(lib, "osp_attn_full_noalloc", qg, kg, vg, o, shape, stream)   # looks up the array first
    assert lib.osp_check_status(st) == 0
    # osp_check_status allocates nothing: the device's free memory is unchanged across it
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info(gpu)[0]
    assert lib.osp_check_status(st) == 0
    assert torch.cuda.mem_get_info(gpu)[0] == free0
    monkeypatch.setenv("OSP_WAIT_TIMEOUT_MS", "100")
    monkeypatch.setenv("OSP_DEBUG_WITHHOLD_Q", "1")
    _call(lib, "osp_attn_full_noalloc", qg, kg, vg, o, shape, stream)
    assert lib.osp_check_status(st) == 5                  # OSP_ERR_TIMEOUT
    assert lib.osp_check_status(st) == 0                  # cleared by the read
    monkeypatch.delenv("OSP_DEBUG_WITHHOLD_Q")
    _call(lib, "osp_attn_full_noalloc", qg, kg, vg, o, shape, stream)
    assert lib.osp_check_status(st) == 0
    assert_attn_close(o, O.attn_ref(to_f64(q), to_f64(k), to_f64(v)), "after the timeout")
