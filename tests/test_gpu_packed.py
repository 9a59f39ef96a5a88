"""GPU parity of packed batches (videos of different shapes in one batch: per-sample 3D RoPE
grids and block-diagonal attention, "CogVideoX" section 3.1 Multi-Resolution Frame Pack)
against the fp64 oracle, and bit-exact agreement with the one-sample entry points."""

import numpy as np
import pytest
import torch

import oracle as O
from spacetime_attention_b200 import ops, synthetic as syn
from tests.gpu_common import gpu  # noqa: F401
from tests.helpers import assert_attn_close, assert_bf16_close, bf16_round, to_f64

pytestmark = pytest.mark.gpu


def _bounds(lengths):
    return O.segment_bounds(lengths).tolist()


@pytest.mark.parametrize("d,lengths", [
    (64, [300, 45, 1, 513, 128]),          # ragged tails, a one-token sample, exact tiles
    (96, [256, 257, 255]),                 # block boundaries: sample starts off the tile grid
    (128, [700, 60]),
    (64, [5, 0, 77, 0, 130]),              # samples without rows are skipped
])
def test_packed_attention_matches_oracle(gpu, d, lengths):
    b = _bounds(lengths)
    q, k, v = syn.make_packed_qkv(2, d, b[-1], seed=31)
    o = ops.attn_packed(q.to(gpu), k.to(gpu), v.to(gpu), b)
    ops.check_status()
    assert_attn_close(o, O.packed_attn_ref(to_f64(q), to_f64(k), to_f64(v), b), f"d{d} {lengths}")


def test_packed_per_sample_cross_attention(gpu):
    # each video's queries attend to its own prompt: 3 samples with 256 / 45 / 300 video tokens and
    # 77 / 1 / 226 text tokens
    qb, kb = _bounds([256, 45, 300]), _bounds([77, 1, 226])
    q, k, v = syn.make_packed_qkv(3, 96, qb[-1], seed=32, total_kv=kb[-1])
    o = ops.attn_packed(q.to(gpu), k.to(gpu), v.to(gpu), qb, kb)
    ops.check_status()
    assert_attn_close(o, O.packed_attn_ref(to_f64(q), to_f64(k), to_f64(v), qb, kb), "packed cross")


def test_many_small_samples(gpu):
    # the full segment table (256 samples of 1..40 rows): every CTA must find its own sample
    rng = np.random.default_rng(33)
    lengths = rng.integers(1, 41, size=ops.MAX_SEGMENTS).tolist()
    b = _bounds(lengths)
    q, k, v = syn.make_packed_qkv(2, 64, b[-1], seed=34)
    o = ops.attn_packed(q.to(gpu), k.to(gpu), v.to(gpu), b)
    ops.check_status()
    assert_attn_close(o, O.packed_attn_ref(to_f64(q), to_f64(k), to_f64(v), b), "256 samples")


def test_packed_equals_one_sample_calls_bit_for_bit(gpu, monkeypatch):
    # the same tiles per sample as osp_attn_full on that sample alone (no split of the KV range)
    monkeypatch.setenv("OSP_SPLIT_KV", "0")
    samples = [(13, 2, 5, 7), (0, 3, 8, 8), (77, 1, 4, 4)]
    lengths = [L + T * H * W for L, T, H, W in samples]
    b = _bounds(lengths)
    q, k, v = (t.to(gpu) for t in syn.make_packed_qkv(2, 64, b[-1], seed=35))
    o = ops.attn_packed(q, k, v, b)
    for i, (L, T, H, W) in enumerate(samples):
        sl = slice(b[i], b[i + 1])
        one = ops.attn_full(q[:, sl].contiguous(), k[:, sl].contiguous(), v[:, sl].contiguous(), (T, H, W), L)
        assert torch.equal(o[:, sl], one), i


def test_packed_rope_matches_oracle_and_one_sample_calls(gpu):
    samples = [(13, 2, 5, 7), (0, 3, 8, 8), (226, 1, 4, 6), (0, 1, 1, 1)]
    split = (16, 24, 24)
    b = _bounds([L + T * H * W for L, T, H, W in samples])
    q, k, _ = syn.make_packed_qkv(3, 64, b[-1], seed=36)
    qg, kg = q.to(gpu), k.to(gpu)
    qo, ko = ops.rope3d_packed(qg, kg, samples, split)
    assert_bf16_close(qo, bf16_round(O.rope3d_packed_ref(to_f64(q), samples, split)), "q")
    assert_bf16_close(ko, bf16_round(O.rope3d_packed_ref(to_f64(k), samples, split)), "k")
    for i, (L, T, H, W) in enumerate(samples):
        sl = slice(b[i], b[i + 1])
        q1, k1 = ops.rope3d(qg[:, sl].contiguous(), kg[:, sl].contiguous(), (T, H, W), L, split)
        assert torch.equal(qo[:, sl], q1) and torch.equal(ko[:, sl], k1), i
    # in place: same bits, text rows untouched
    qi, ki = qg.clone(), kg.clone()
    ops.rope3d_packed(qi, ki, samples, split, q_out=qi, k_out=ki)
    assert torch.equal(qi, qo) and torch.equal(ki, ko)


def test_full_size_frame_pack_sampled(gpu):
    """The bench's packed batch (five CogVideoX-2B-shaped samples of different durations and
    resolutions, 226 text tokens each): RoPE then block-diagonal attention, sampled rows of every
    head against the oracle."""
    w = syn.PACKED_WORKLOADS["frame_pack_cog2b"]
    q, k, v = syn.make_packed_qkv(w.heads, w.head_dim, w.total, w.seed)
    qr, kr = ops.rope3d_packed(q.to(gpu), k.to(gpu), w.samples, w.split)
    o = ops.attn_packed(qr, kr, v.to(gpu), w.bounds)
    ops.check_status()
    rng = np.random.default_rng(w.seed)
    rows = set()
    for i in range(len(w.samples)):
        a, e = w.bounds[i], w.bounds[i + 1]
        rows |= {a, e - 1, a + 226, *rng.integers(a, e, size=4).tolist()}
    rows = sorted(rows)
    qo = to_f64(bf16_round(O.rope3d_packed_ref(to_f64(q), w.samples, w.split)))
    ko = to_f64(bf16_round(O.rope3d_packed_ref(to_f64(k), w.samples, w.split)))
    ref = O.packed_attn_ref(qo, ko, to_f64(v), w.bounds, rows=rows)
    assert_attn_close(o[:, rows], ref, w.name)
