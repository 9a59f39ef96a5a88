"""Failure detection on the GPU without faulting it: every mbarrier wait in the attention kernel
is bounded.  With OSP_DEBUG_WITHHOLD_Q=1 the producer never loads Q, so the MMA and softmax warps
wait for a barrier that nothing completes; after OSP_WAIT_TIMEOUT_MS they give up, record the
timeout in the device status word, drain what they issued, free tensor memory and exit.  The
host sees OSP_ERR_TIMEOUT from osp_check_status and the context stays usable."""

import numpy as np
import pytest
import torch

import oracle as O
from spacetime_attention_b200 import ops, synthetic as syn
from tests.gpu_common import gpu  # noqa: F401
from tests.helpers import assert_attn_close, to_f64

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("heads,grid", [(2, (4, 8, 8)), (16, (4, 8, 16))])
def test_withheld_load_times_out_and_context_recovers(gpu, monkeypatch, heads, grid):
    w = syn.custom("f", 1, heads, 64, grid, 0, (16, 24, 24))
    q, k, v = syn.make_qkv(w, 31)
    qg, kg, vg = q.to(gpu), k.to(gpu), v.to(gpu)
    ops.check_status()                                   # start from a clean status word
    monkeypatch.setenv("OSP_WAIT_TIMEOUT_MS", "100")
    monkeypatch.setenv("OSP_DEBUG_WITHHOLD_Q", "1")
    ops.attn_full(qg, kg, vg, grid, 0)
    with pytest.raises(ops.OspError) as err:
        ops.check_status()
    assert err.value.code == 5                           # OSP_ERR_TIMEOUT
    monkeypatch.delenv("OSP_DEBUG_WITHHOLD_Q")
    ops.check_status()                                   # the word was cleared by the read
    o = ops.attn_full(qg, kg, vg, grid, 0)
    ops.check_status()
    assert_attn_close(o, O.attn_ref(to_f64(q), to_f64(k), to_f64(v)), "after recovery")
    torch.cuda.synchronize()


def test_timeout_with_skiparse_layout(gpu, monkeypatch):
    w = syn.custom("f", 1, 2, 128, (2, 8, 16), 0, (32, 48, 48))
    q, k, v = (t.to(gpu) for t in syn.make_qkv(w, 32))
    monkeypatch.setenv("OSP_WAIT_TIMEOUT_MS", "100")
    monkeypatch.setenv("OSP_DEBUG_WITHHOLD_Q", "1")
    ops.skiparse_attn(q, k, v, (2, 8, 16), 4, ops.OSP_SKIP_GROUP)
    with pytest.raises(ops.OspError) as err:
        ops.check_status()
    assert err.value.code == 5
    monkeypatch.delenv("OSP_DEBUG_WITHHOLD_Q")
    o = ops.skiparse_attn(q, k, v, (2, 8, 16), 4, ops.OSP_SKIP_GROUP)
    ops.check_status()
    assert np.isfinite(to_f64(o)).all()
