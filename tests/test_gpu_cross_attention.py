"""GPU parity of video -> text cross-attention (osp_attn_cross) against the fp64 oracle.

Queries are the T*H*W video tokens, keys and values the text tokens ("Open-Sora Plan" section
2.2.1: every block attends from the video to the mT5 text embeddings).  Same tolerance as the
self-attention kernels: max-abs <= 2e-2 and relative-L2 <= 5e-3."""

import numpy as np
import pytest
import torch

import oracle as O
from spacetime_attention_b200 import ops, synthetic as syn
from tests.gpu_common import gpu  # noqa: F401
from tests.helpers import assert_attn_close, to_f64

pytestmark = pytest.mark.gpu

CROSS_CASES = [
    # name, B, heads, d, grid (queries), text_len (keys)
    ("one_key", 2, 3, 64, (4, 8, 8), 1),
    ("ragged_kv_tile", 2, 3, 64, (4, 8, 8), 77),           # 256 queries, one partial KV tile
    ("two_kv_tiles_ragged_q", 1, 2, 96, (3, 7, 13), 226),  # 273 queries: Q tail, KV tail
    ("d128_300", 2, 2, 128, (2, 9, 19), 300),
    ("exact_tiles", 1, 2, 64, (2, 8, 16), 512),           # 256 queries, 4 full KV tiles
    ("few_queries", 1, 4, 96, (1, 5, 9), 130),             # 45 queries, 2 KV tiles (2 keys in the 2nd)
    ("keys_exceed_queries", 1, 2, 64, (1, 3, 5), 1000),    # 15 queries, 8 KV tiles: split-KV eligible
]


def _inputs(B, heads, d, grid, L, seed=21):
    n_v = grid[0] * grid[1] * grid[2]
    q = syn.randn_bf16((B, n_v, heads, d), seed)
    k = syn.randn_bf16((B, L, heads, d), seed + 1)
    v = syn.randn_bf16((B, L, heads, d), seed + 2)
    return q, k, v


@pytest.mark.parametrize("case", CROSS_CASES, ids=[c[0] for c in CROSS_CASES])
def test_cross_attention_matches_oracle(gpu, case):
    name, B, heads, d, grid, L = case
    q, k, v = _inputs(B, heads, d, grid, L)
    o = ops.attn_cross(q.to(gpu), k.to(gpu), v.to(gpu), grid)
    ops.check_status()
    assert o.shape == q.shape
    assert_attn_close(o, O.cross_attn_ref(to_f64(q), to_f64(k), to_f64(v)), name)


def test_one_text_token_returns_its_value(gpu):
    # a single key: softmax weight 1 for every query, so every output row is that key's value
    q, k, v = _inputs(2, 3, 64, (2, 5, 7), 1)
    o = ops.attn_cross(q.to(gpu), k.to(gpu), v.to(gpu), (2, 5, 7))
    assert torch.equal(o.cpu(), v.expand(-1, q.shape[1], -1, -1))


def test_zero_queries_give_mean_of_text_values(gpu):
    q, k, v = _inputs(1, 2, 96, (2, 8, 10), 150)
    o = ops.attn_cross(torch.zeros_like(q).to(gpu), k.to(gpu), v.to(gpu), (2, 8, 10))
    ref = np.broadcast_to(to_f64(v).mean(1, keepdims=True), o.shape)
    assert_attn_close(o, ref, "q=0")


def test_explicit_scale(gpu):
    q, k, v = _inputs(1, 2, 128, (2, 4, 16), 200)
    o = ops.attn_cross(q.to(gpu), k.to(gpu), v.to(gpu), (2, 4, 16), scale=0.03)
    assert_attn_close(o, O.cross_attn_ref(to_f64(q), to_f64(k), to_f64(v), scale=0.03), "scale")


@pytest.mark.parametrize("d", [64, 96, 128])
def test_equal_lengths_match_self_attention_bit_for_bit(gpu, d):
    # with as many text tokens as video tokens the call is dense attention over the video tokens:
    # same tiles, same order, so the same bits as osp_attn_full with no text prefix
    grid = (3, 8, 11)
    q, k, v = _inputs(1, 2, d, grid, 264, seed=40)
    qg, kg, vg = q.to(gpu), k.to(gpu), v.to(gpu)
    cross = ops.attn_cross(qg, kg, vg, grid)
    full = ops.attn_full(qg, kg, vg, grid, 0)
    assert torch.equal(cross, full)


def test_rejects_empty_text(gpu):
    q, k, v = _inputs(1, 2, 64, (1, 4, 4), 1)
    with pytest.raises(ops.OspError) as e:
        ops.attn_cross(q.to(gpu), k[:, :0].to(gpu), v[:, :0].to(gpu), (1, 4, 4))
    assert e.value.code == 1


@pytest.mark.parametrize("name,L", [("open_sora_plan", 226), ("cogvideox_2b", 226), ("long_video", 512)])
def test_full_size_cross_attention_sampled(gpu, name, L):
    """Video tokens of the full-size workloads attending to L text tokens, on sampled query rows
    of every head."""
    w = syn.WORKLOADS[name]
    q, k, v = _inputs(w.B, w.heads, w.head_dim, w.grid, L, seed=w.seed + 7)
    o = ops.attn_cross(q.to(gpu), k.to(gpu), v.to(gpu), w.grid)
    ops.check_status()
    rng = np.random.default_rng(w.seed)
    rows = sorted(set(rng.choice(w.n_video, size=20, replace=False).tolist()) | {0, w.n_video - 1})
    ref = O.cross_attn_ref(to_f64(q), to_f64(k), to_f64(v), rows=rows)
    assert_attn_close(o[:, rows], ref, name)
