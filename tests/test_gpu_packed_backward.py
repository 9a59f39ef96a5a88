"""Training on packed batches (CogVideoX section 3.1, Multi-Resolution Frame Pack): the packed
self-attention forward with its saved log-sum-exp and the backward pass, against the fp64 oracle
(packed_backward_ref, pinned by finite differences), and against the one-sample training calls
on each sample alone."""

import math

import numpy as np
import pytest
import torch

import oracle as O
from spacetime_attention_b200 import ops, synthetic as syn
from tests.gpu_common import gpu  # noqa: F401
from tests.test_gpu_backward import assert_grad_close

pytestmark = pytest.mark.gpu


def _bounds(lengths):
    return O.segment_bounds(lengths).tolist()


def _lse_rows(lengths):
    # sample i's lse rows start at the start of its 256-row blocks
    off, out = 0, []
    for n in lengths:
        out.append(off)
        off += -(-n // 256) * 256
    return out, off


CASES = [
    (64, [300, 45, 1, 513, 128]),     # ragged tails, a one-token sample, exact tiles
    (96, [256, 257, 0, 255]),         # starts off the tile grid, an empty sample
    (128, [200, 60, 131]),
    (64, [1000, 7]),                  # several key tiles per sample: the fused dQ reduce over tiles
]


@pytest.mark.parametrize("d,lengths", CASES, ids=[f"d{c[0]}_{len(c[1])}" for c in CASES])
def test_packed_training_matches_oracle(gpu, d, lengths):
    b = _bounds(lengths)
    heads = 2
    q, k, v = syn.make_packed_qkv(heads, d, b[-1], seed=61)
    do = syn.randn_bf16(tuple(q.shape), 64)
    qg, kg, vg, dog = (t.to(gpu) for t in (q, k, v, do))
    o, lse = ops.attn_packed_train(qg, kg, vg, b)
    dq, dk, dv = ops.attn_packed_backward(qg, kg, vg, o, dog, lse, b)
    ops.check_status()
    # the training forward is the inference call, bit for bit
    assert torch.equal(o, ops.attn_packed(qg, kg, vg, b))
    qd, kd, vd = (t.detach().double().numpy() for t in (q.float(), k.float(), v.float()))
    rq, rk, rv = O.packed_backward_ref(qd, kd, vd, do.float().double().numpy(), b)
    assert_grad_close(dq, rq, "dq")
    assert_grad_close(dk, rk, "dk")
    assert_grad_close(dv, rv, "dv")
    # lse (log2 domain) of every sample and head at its block offset
    starts, total = _lse_rows(lengths)
    assert lse.shape == (heads, total)
    scale = 1 / math.sqrt(d)
    for i, n in enumerate(lengths):
        if n == 0:
            continue
        for h in range(heads):
            ref = O.attention_head_lse_ref(qd[0, b[i]:b[i + 1], h], kd[0, b[i]:b[i + 1], h], scale)
            got = lse[h, starts[i]:starts[i] + n].double().cpu().numpy()
            np.testing.assert_allclose(got, ref / math.log(2.0), rtol=0, atol=2e-3)


@pytest.mark.parametrize("d", [64, 128])
def test_packed_training_equals_each_sample_alone(gpu, monkeypatch, d):
    # every sample's dK and dV (and dQ at d = 128, where no reduction order is involved) are the
    # one-sample training call's bits; at d = 64, dQ sums the key tiles' contributions in an
    # order set by the CTAs' timing, so it is compared within the tolerance
    monkeypatch.setenv("OSP_SPLIT_KV", "0")
    lengths = [300, 130, 513]
    b = _bounds(lengths)
    q, k, v = syn.make_packed_qkv(2, d, b[-1], seed=71)
    do = syn.randn_bf16(tuple(q.shape), 74)
    qg, kg, vg, dog = (t.to(gpu) for t in (q, k, v, do))
    o, lse = ops.attn_packed_train(qg, kg, vg, b)
    grads = ops.attn_packed_backward(qg, kg, vg, o, dog, lse, b)
    for i, n in enumerate(lengths):
        r = slice(b[i], b[i + 1])
        one = [t[:, r].contiguous() for t in (qg, kg, vg, dog)]
        o1, lse1 = ops.attn_forward_train(one[0], one[1], one[2], (1, 1, n), 0)
        g1 = ops.attn_backward(one[0], one[1], one[2], o1, one[3], lse1, (1, 1, n), 0)
        ops.check_status()
        assert torch.equal(o[:, r], o1)
        assert torch.equal(grads[1][:, r], g1[1]) and torch.equal(grads[2][:, r], g1[2])
        if d > 64:
            assert torch.equal(grads[0][:, r], g1[0])
        else:
            err = (grads[0][:, r].float() - g1[0].float()).abs().max().item()
            assert err <= 1e-2 * g1[0].float().abs().max().item()


def test_packed_training_rejects_bad_lse(gpu):
    q, k, v = (t.to(gpu) for t in syn.make_packed_qkv(2, 64, 300, seed=80))
    with pytest.raises(ValueError):
        ops.attn_packed_train(q, k, v, [0, 300], lse=torch.empty((2, 100), device=gpu))
    assert ops.packed_lse_rows([0, 300, 301]) == 512 + 256


def test_packed_training_full_size_sampled(gpu):
    """The frame-pack workload at full size (five samples of 1,576 to 17,776 tokens, 47,360 rows,
    30 heads, d = 64): packed training forward and backward, then per sample sampled dQ rows and
    dK / dV rows of one head against the oracle's row form on that sample alone."""
    w = syn.PACKED_WORKLOADS["frame_pack_cog2b"]
    b = w.bounds
    q, k, v = syn.make_packed_qkv(w.heads, w.head_dim, w.total, w.seed + 3)
    do = syn.randn_bf16(tuple(q.shape), w.seed + 4)
    qg, kg, vg, dog = (t.to(gpu) for t in (q, k, v, do))
    o, lse = ops.attn_packed_train(qg, kg, vg, b)
    dq, dk, dv = ops.attn_packed_backward(qg, kg, vg, o, dog, lse, b)
    ops.check_status()
    h = 11
    scale = 1 / math.sqrt(w.head_dim)
    rng = np.random.default_rng(5)
    for i, n in enumerate(w.lengths):
        r = slice(b[i], b[i + 1])
        rows = sorted({0, n - 1, *rng.integers(0, n, size=4).tolist()})
        qh, kh, vh, dh = (t[0, r, h].double().numpy() for t in (q, k, v, do))
        rq, rk, rv = O.attention_head_backward_rows_ref(qh, kh, vh, dh, scale, rows, rows)
        sel = [b[i] + x for x in rows]
        assert_grad_close(dq[0, sel, h], rq, f"dq sample {i}")
        assert_grad_close(dk[0, sel, h], rk, f"dk sample {i}")
        assert_grad_close(dv[0, sel, h], rv, f"dv sample {i}")
