"""GPU parity of Skiparse attention with a joined text prefix (text tokens as global tokens:
video queries of set g see the text and set g, text queries see everything) against the fp64
oracle."""

import numpy as np
import pytest

import oracle as O
from spacetime_attention_b200 import ops, synthetic as syn
from tests.gpu_common import gpu  # noqa: F401
from tests.helpers import assert_attn_close, to_f64

pytestmark = pytest.mark.gpu

CASES = [
    # B, heads, d, grid, text_len, k
    (1, 2, 64, (4, 8, 8), 13, 2),
    (2, 2, 96, (4, 10, 15), 226, 2),      # two text tiles (ragged), sets of 300
    (1, 2, 128, (4, 16, 18), 77, 4),
    (1, 1, 64, (2, 16, 16), 128, 4),      # text exactly one tile
    (1, 2, 64, (4, 8, 8), 1, 2),          # one text token
]


def _qkv(B, heads, d, grid, L, seed=71):
    N = L + grid[0] * grid[1] * grid[2]
    return tuple(syn.randn_bf16((B, N, heads, d), seed + i) for i in range(3))


@pytest.mark.parametrize("mode", [0, 1])
@pytest.mark.parametrize("case", CASES, ids=[f"{c[3]}_L{c[4]}_k{c[5]}_d{c[2]}" for c in CASES])
def test_skiparse_with_text_matches_oracle(gpu, case, mode):
    B, heads, d, grid, L, k = case
    q, kk, v = _qkv(B, heads, d, grid, L)
    o = ops.skiparse_attn(q.to(gpu), kk.to(gpu), v.to(gpu), grid, k, mode, text_len=L)
    ops.check_status()
    assert_attn_close(o, O.skiparse_text_attn_ref(to_f64(q), to_f64(kk), to_f64(v), L, k, mode),
                      f"{grid} L={L} k={k} mode={mode}")


def test_split_kv_with_text_matches_unsplit(gpu, monkeypatch):
    grid, L, k = (4, 16, 16), 40, 2
    q, kk, v = (t.to(gpu) for t in _qkv(1, 1, 64, grid, L, seed=72))
    split = ops.skiparse_attn(q, kk, v, grid, k, 0, text_len=L)
    monkeypatch.setenv("OSP_SPLIT_KV", "0")
    plain = ops.skiparse_attn(q, kk, v, grid, k, 0, text_len=L)
    ops.check_status()
    ref = O.skiparse_text_attn_ref(to_f64(q.cpu()), to_f64(kk.cpu()), to_f64(v.cpu()), L, k, 0)
    assert_attn_close(split, ref, "split")
    assert_attn_close(plain, ref, "unsplit")


@pytest.mark.parametrize("mode", [0, 1])
def test_full_size_skiparse_with_text_sampled(gpu, mode):
    """The Open-Sora Plan grid (24 x 30 x 40, 24 heads, d = 96, k = 4) with a 226-token text
    prefix, sampled text and video rows of every head."""
    w = syn.WORKLOADS["open_sora_plan"]
    L = 226
    q, kk, v = _qkv(1, w.heads, w.head_dim, w.grid, L, seed=w.seed + 3)
    o = ops.skiparse_attn(q.to(gpu), kk.to(gpu), v.to(gpu), w.grid, 4, mode, text_len=L)
    ops.check_status()
    rng = np.random.default_rng(7 + mode)
    rows = sorted({0, L - 1, L, L + w.n_video - 1, *rng.integers(0, L + w.n_video, size=16).tolist()})
    ref = O.skiparse_text_attn_ref(to_f64(q), to_f64(kk), to_f64(v), L, 4, mode, rows=rows)
    assert_attn_close(o[:, rows], ref, f"osp text mode {mode}")
