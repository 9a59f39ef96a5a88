"""GPU parity of the factorized (2D + 1D) and frame-causal attention variants against the fp64
oracle: per-frame spatial attention, per-position temporal attention (bidirectional and causal
in time) and frame-causal attention with a text block."""

import numpy as np
import pytest
import torch

import oracle as O
from spacetime_attention_b200 import ops, synthetic as syn
from tests.gpu_common import gpu  # noqa: F401
from tests.helpers import assert_attn_close, to_f64

pytestmark = pytest.mark.gpu


def _qkv(B, heads, d, grid, L=0, seed=51):
    N = L + grid[0] * grid[1] * grid[2]
    return tuple(syn.randn_bf16((B, N, heads, d), seed + i) for i in range(3))


@pytest.mark.parametrize("B,heads,d,grid", [(1, 2, 64, (3, 5, 7)), (1, 2, 128, (2, 9, 19)), (2, 3, 96, (4, 8, 16))])
def test_spatial_matches_oracle(gpu, B, heads, d, grid):
    q, k, v = _qkv(B, heads, d, grid)
    o = ops.attn_spatial(q.to(gpu), k.to(gpu), v.to(gpu), grid)
    ops.check_status()
    assert_attn_close(o, O.spatial_attn_ref(to_f64(q), to_f64(k), to_f64(v), grid), f"spatial {grid}")


TEMPORAL = [
    # B, heads, d, grid
    (2, 3, 64, (13, 5, 7)),      # T = 13: one 16-row tile, 3 padded rows
    (1, 2, 96, (16, 4, 5)),      # T = 16 exactly
    (1, 3, 128, (24, 3, 7)),     # two tiles
    (1, 2, 64, (40, 2, 3)),      # three tiles
    (1, 1, 96, (64, 2, 2)),      # four tiles, the limit of the staged kernel
    (1, 2, 64, (1, 4, 6)),       # one frame: every token alone
]


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("case", TEMPORAL, ids=[f"T{c[3][0]}_d{c[2]}" for c in TEMPORAL])
def test_temporal_matches_oracle(gpu, case, causal):
    B, heads, d, grid = case
    q, k, v = _qkv(B, heads, d, grid, seed=52)
    o = ops.attn_temporal(q.to(gpu), k.to(gpu), v.to(gpu), grid, causal=causal)
    ops.check_status()
    assert_attn_close(o, O.temporal_attn_ref(to_f64(q), to_f64(k), to_f64(v), grid, causal=causal),
                      f"temporal {grid} causal={causal}")


def test_temporal_single_frame_returns_v(gpu):
    q, k, v = _qkv(2, 3, 64, (1, 5, 6), seed=53)
    o = ops.attn_temporal(q.to(gpu), k.to(gpu), v.to(gpu), (1, 5, 6))
    assert torch.equal(o.cpu(), v)


def test_causal_temporal_first_frame_returns_v(gpu):
    q, k, v = _qkv(1, 2, 96, (9, 4, 4), seed=54)
    o = ops.attn_temporal(q.to(gpu), k.to(gpu), v.to(gpu), (9, 4, 4), causal=True)
    assert torch.equal(o[:, :16].cpu(), v[:, :16])


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("T,d", [(80, 64), (300, 96), (129, 128)])
def test_long_temporal_uses_single_skip_path(gpu, T, d, causal):
    # T > 64: the position's tokens form Single Skip set pos with k = H*W (causal: the frame-causal
    # mask with one-row blocks); 129 and 300 frames leave ragged query and key tiles
    grid = (T, 2, 3)
    q, k, v = _qkv(1, 2, d, grid, seed=55)
    o = ops.attn_temporal(q.to(gpu), k.to(gpu), v.to(gpu), grid, causal=causal)
    ops.check_status()
    assert_attn_close(o, O.temporal_attn_ref(to_f64(q), to_f64(k), to_f64(v), grid, causal=causal),
                      f"T{T} causal={causal}")


FRAME_CAUSAL = [
    # B, heads, d, grid, text_len
    (1, 2, 64, (4, 6, 8), 0),       # 48-token frames: frame boundaries inside tiles
    (2, 2, 96, (3, 7, 13), 5),      # text block + 91-token frames
    (1, 3, 128, (5, 8, 9), 17),
    (1, 2, 64, (6, 16, 16), 0),     # 256-token frames: boundaries on the query-block grid
    (1, 1, 64, (1, 9, 11), 7),      # one frame: full attention with text attending to text only
]


@pytest.mark.parametrize("case", FRAME_CAUSAL, ids=[f"{c[3]}_L{c[4]}_d{c[2]}" for c in FRAME_CAUSAL])
def test_frame_causal_matches_oracle(gpu, case):
    B, heads, d, grid, L = case
    q, k, v = _qkv(B, heads, d, grid, L, seed=56)
    o = ops.attn_frame_causal(q.to(gpu), k.to(gpu), v.to(gpu), grid, L)
    ops.check_status()
    assert_attn_close(o, O.frame_causal_attn_ref(to_f64(q), to_f64(k), to_f64(v), grid, L), f"frame-causal {grid}")


def test_frame_causal_last_frame_equals_full_attention_bits(gpu, monkeypatch):
    # rows of the last frame see every key: the same per-row computation as osp_attn_full
    monkeypatch.setenv("OSP_SPLIT_KV", "0")
    grid, L = (4, 10, 12), 9
    q, k, v = (t.to(gpu) for t in _qkv(1, 2, 64, grid, L, seed=57))
    fc = ops.attn_frame_causal(q, k, v, grid, L)
    full = ops.attn_full(q, k, v, grid, L)
    last = L + 3 * 120
    assert torch.equal(fc[:, last:], full[:, last:])


def _sample(n, count, seed):
    rng = np.random.default_rng(seed)
    return sorted(set(rng.choice(n, size=count, replace=False).tolist()) | {0, n - 1})


def test_full_size_temporal_and_spatial_sampled(gpu):
    """The CogVideoX-2B grid (13 x 30 x 45, 30 heads, d = 64): temporal attention on sampled
    positions (bidirectional and causal) and spatial attention on sampled frames."""
    w = syn.WORKLOADS["cogvideox_2b"]
    T, H, W = w.grid
    q, k, v = _qkv(1, w.heads, w.head_dim, w.grid, seed=w.seed + 9)
    qg, kg, vg = q.to(gpu), k.to(gpu), v.to(gpu)
    HW = H * W
    pos = _sample(HW, 12, 5)
    idx = (np.arange(T)[:, None] * HW + np.asarray(pos)[None, :]).reshape(-1)   # token t*P + i
    sub = lambda x: to_f64(x[:, idx])
    for causal in (False, True):
        o = ops.attn_temporal(qg, kg, vg, w.grid, causal=causal)
        ops.check_status()
        ref = O.temporal_attn_ref(sub(q), sub(k), sub(v), (T, 1, len(pos)), causal=causal)
        assert_attn_close(o[:, idx], ref, f"temporal causal={causal}")
    o = ops.attn_spatial(qg, kg, vg, w.grid)
    ops.check_status()
    for t in (0, 7, T - 1):
        f = slice(t * HW, (t + 1) * HW)
        ref = O.spatial_attn_ref(to_f64(q[:, f]), to_f64(k[:, f]), to_f64(v[:, f]), (1, H, W))
        assert_attn_close(o[:, f], ref, f"spatial frame {t}")


def test_full_size_frame_causal_sampled(gpu):
    w = syn.WORKLOADS["cogvideox_2b"]
    q, k, v = syn.make_qkv(w)
    o = ops.attn_frame_causal(q.to(gpu), k.to(gpu), v.to(gpu), w.grid, w.text_len)
    ops.check_status()
    rows = _sample(w.seq_len, 20, 6)
    ref = O.frame_causal_attn_ref(to_f64(q), to_f64(k), to_f64(v), w.grid, w.text_len, rows=rows)
    assert_attn_close(o[:, rows], ref, "cog2b frame-causal")
