"""GPU parity of the attention backward pass (dQ, dK, dV on tcgen05) and of the training
forward's saved log-sum-exp, against the fp64 oracle (chain rule pinned by finite differences).

Tolerance (derived from the arithmetic): P and dS are rounded to bf16 (relative 2^-9) before
the tensor-core products, accumulation is fp32 and the outputs are rounded to bf16 once more;
the expected relative-L2 error is a few 1e-3.  Bound: relative-L2 <= 1e-2 per gradient and
max-abs <= 2e-2 of the gradient's largest magnitude."""

import math

import numpy as np
import pytest
import torch

import oracle as O
from spacetime_attention_b200 import ops, synthetic as syn
from tests.gpu_common import gpu  # noqa: F401
from tests.helpers import assert_attn_close, to_f64

pytestmark = pytest.mark.gpu

GRAD_REL_L2 = 1e-2
GRAD_MAX_REL = 2e-2


def assert_grad_close(got, ref, what):
    g = to_f64(got)
    assert np.isfinite(g).all(), f"{what}: non-finite gradient"
    err = g - ref
    rl = float(np.linalg.norm(err) / max(np.linalg.norm(ref), 1e-30))
    mx = float(np.abs(err).max() / max(np.abs(ref).max(), 1e-30))
    assert rl <= GRAD_REL_L2 and mx <= GRAD_MAX_REL, f"{what}: rel-L2 {rl:.3e}, max-abs/max {mx:.3e}"


def _inputs(B, heads, d, grid, L, seed):
    N = L + grid[0] * grid[1] * grid[2]
    q, k, v, do = (syn.randn_bf16((B, N, heads, d), seed + i) for i in range(4))
    return q, k, v, do


DENSE = [
    # B, heads, d, grid, text_len
    (1, 2, 64, (2, 8, 8), 0),          # 128 tokens: one tile
    (2, 2, 64, (3, 9, 11), 5),         # 302 tokens: ragged query and key tiles
    (1, 3, 96, (3, 7, 13), 17),
    (1, 2, 128, (2, 9, 19), 0),
    (1, 1, 64, (1, 1, 1), 0),          # one token: dQ = dK = 0, dV = dO
]


@pytest.mark.parametrize("case", DENSE, ids=[f"{c[3]}_L{c[4]}_d{c[2]}" for c in DENSE])
def test_dense_backward_matches_oracle(gpu, case):
    B, heads, d, grid, L = case
    q, k, v, do = _inputs(B, heads, d, grid, L, 91)
    qg, kg, vg, dog = (t.to(gpu) for t in (q, k, v, do))
    o, lse = ops.attn_forward_train(qg, kg, vg, grid, L)
    dq, dk, dv = ops.attn_backward(qg, kg, vg, o, dog, lse, grid, L)
    ops.check_status()
    # the training forward is the inference forward, bit for bit
    assert torch.equal(o, ops.attn_full(qg, kg, vg, grid, L))
    rq, rk, rv = O.attn_backward_ref(to_f64(q), to_f64(k), to_f64(v), to_f64(do))
    assert_grad_close(dq, rq, "dq")
    assert_grad_close(dk, rk, "dk")
    assert_grad_close(dv, rv, "dv")
    # saved log-sum-exp (log2 domain) of every row
    N = q.shape[1]
    scale = 1 / math.sqrt(d)
    for b in range(B):
        for h in range(heads):
            ref = O.attention_head_lse_ref(to_f64(q)[b, :, h], to_f64(k)[b, :, h], scale) / math.log(2.0)
            got = lse[b, h, :N].double().cpu().numpy()
            np.testing.assert_allclose(got, ref, rtol=0, atol=2e-3)


SPARSE = [
    # B, heads, d, grid, k
    (1, 2, 64, (4, 8, 8), 2),
    (1, 2, 96, (4, 10, 15), 2),       # sets of 300: ragged tiles
    (1, 1, 128, (4, 16, 18), 4),
    (2, 1, 64, (2, 16, 16), 8),       # B = 2, sets of 64 (one partial tile each)
]


@pytest.mark.parametrize("mode", [0, 1])
@pytest.mark.parametrize("case", SPARSE, ids=[f"{c[3]}_k{c[4]}_d{c[2]}" for c in SPARSE])
def test_skiparse_backward_matches_oracle(gpu, case, mode):
    B, heads, d, grid, kk = case
    q, k, v, do = _inputs(B, heads, d, grid, 0, 92)
    qg, kg, vg, dog = (t.to(gpu) for t in (q, k, v, do))
    o, lse = ops.attn_forward_train(qg, kg, vg, grid, 0, sparse_k=kk, mode=mode)
    dq, dk, dv = ops.attn_backward(qg, kg, vg, o, dog, lse, grid, 0, sparse_k=kk, mode=mode)
    ops.check_status()
    assert torch.equal(o, ops.skiparse_attn(qg, kg, vg, grid, kk, mode))
    rq, rk, rv = O.skiparse_backward_ref(to_f64(q), to_f64(k), to_f64(v), to_f64(do), kk, mode)
    assert_grad_close(dq, rq, f"dq mode {mode}")
    assert_grad_close(dk, rk, f"dk mode {mode}")
    assert_grad_close(dv, rv, f"dv mode {mode}")


def test_split_forward_saves_the_same_lse(gpu, monkeypatch):
    # few work units: the forward splits KV ranges and the combine kernel writes lse
    grid, L = (4, 15, 16), 40
    q, k, v, _ = _inputs(1, 2, 64, grid, L, 93)
    qg, kg, vg = (t.to(gpu) for t in (q, k, v))
    _, lse_split = ops.attn_forward_train(qg, kg, vg, grid, L)
    monkeypatch.setenv("OSP_SPLIT_KV", "0")
    _, lse_plain = ops.attn_forward_train(qg, kg, vg, grid, L)
    N = q.shape[1]
    assert float((lse_split[..., :N] - lse_plain[..., :N]).abs().max()) <= 1e-4


def test_full_size_backward_sampled(gpu):
    """CogVideoX-2B-shaped dense attention (17,776 tokens, 30 heads, d = 64): forward + backward at
    full size; sampled dQ rows and dK / dV rows of two heads against the oracle's row form."""
    w = syn.WORKLOADS["cogvideox_2b"]
    q, k, v, do = _inputs(1, w.heads, w.head_dim, w.grid, w.text_len, w.seed + 5)
    qg, kg, vg, dog = (t.to(gpu) for t in (q, k, v, do))
    o, lse = ops.attn_forward_train(qg, kg, vg, w.grid, w.text_len)
    dq, dk, dv = ops.attn_backward(qg, kg, vg, o, dog, lse, w.grid, w.text_len)
    ops.check_status()
    rng = np.random.default_rng(9)
    rows = sorted({0, w.seq_len - 1, 225, 226, *rng.integers(0, w.seq_len, size=8).tolist()})
    scale = 1 / math.sqrt(w.head_dim)
    for h in (0, 17):
        rq, rk, rv = O.attention_head_backward_rows_ref(to_f64(q)[0, :, h], to_f64(k)[0, :, h], to_f64(v)[0, :, h],
                                                        to_f64(do)[0, :, h], scale, rows, rows)
        assert_grad_close(dq[0, rows, h], rq, f"dq head {h}")
        assert_grad_close(dk[0, rows, h], rk, f"dk head {h}")
        assert_grad_close(dv[0, rows, h], rv, f"dv head {h}")


FRAME_CAUSAL = [
    # B, heads, d, grid, text_len
    (1, 2, 64, (3, 5, 7), 0),          # 35-token frames: block boundaries inside every tile
    (1, 2, 96, (4, 6, 8), 13),
    (2, 1, 128, (3, 9, 15), 5),
    (1, 2, 64, (2, 16, 16), 200),      # text spanning a tile boundary
    (1, 2, 64, (6, 8, 32), 0),         # 256-token frames: later key tiles skip early query tiles
]


@pytest.mark.parametrize("case", FRAME_CAUSAL, ids=[f"{c[3]}_L{c[4]}_d{c[2]}" for c in FRAME_CAUSAL])
def test_frame_causal_backward_matches_oracle(gpu, case):
    B, heads, d, grid, L = case
    q, k, v, do = _inputs(B, heads, d, grid, L, 94)
    qg, kg, vg, dog = (t.to(gpu) for t in (q, k, v, do))
    o, lse = ops.attn_frame_causal_train(qg, kg, vg, grid, L)
    dq, dk, dv = ops.attn_frame_causal_backward(qg, kg, vg, o, dog, lse, grid, L)
    ops.check_status()
    assert torch.equal(o, ops.attn_frame_causal(qg, kg, vg, grid, L))
    rq, rk, rv = O.frame_causal_backward_ref(to_f64(q), to_f64(k), to_f64(v), to_f64(do), grid, L)
    assert_grad_close(dq, rq, "dq")
    assert_grad_close(dk, rk, "dk")
    assert_grad_close(dv, rv, "dv")


SKIP_TEXT = [
    # B, heads, d, grid, k, text_len
    (1, 2, 64, (4, 8, 8), 2, 5),         # sets of 128 plus 5 text rows: the text opens a second key tile
    (2, 1, 64, (2, 16, 16), 4, 140),     # text over a tile boundary; B = 2
    (1, 2, 96, (4, 10, 15), 2, 17),      # sets of 300: ragged tiles
    (1, 1, 128, (4, 16, 18), 4, 33),
    (2, 2, 64, (2, 4, 8), 2, 10),        # sets of 32 rows (one partial tile) and 10 text rows
]


@pytest.mark.parametrize("mode", [0, 1])
@pytest.mark.parametrize("case", SKIP_TEXT, ids=[f"{c[3]}_k{c[4]}_L{c[5]}_d{c[2]}" for c in SKIP_TEXT])
def test_skiparse_text_backward_matches_oracle(gpu, case, mode):
    """Skiparse with a joined text prefix: text queries see every token, a video query of set g
    sees the text and set g.  Training forward = inference forward bit for bit; lse of the video
    rows (set-slot order) and of the text rows against the oracle; gradients against the chain
    rule on the masked score matrix."""
    B, heads, d, grid, kk, L = case
    q, k, v, do = _inputs(B, heads, d, grid, L, 94)
    qg, kg, vg, dog = (t.to(gpu) for t in (q, k, v, do))
    o, lse = ops.attn_forward_train(qg, kg, vg, grid, L, sparse_k=kk, mode=mode)
    dq, dk, dv = ops.attn_backward(qg, kg, vg, o, dog, lse, grid, L, sparse_k=kk, mode=mode)
    ops.check_status()
    assert torch.equal(o, ops.skiparse_attn(qg, kg, vg, grid, kk, mode, text_len=L))
    rq, rk, rv = O.skiparse_text_backward_ref(to_f64(q), to_f64(k), to_f64(v), to_f64(do), L, kk, mode)
    assert_grad_close(dq, rq, f"dq mode {mode}")
    assert_grad_close(dk, rk, f"dk mode {mode}")
    assert_grad_close(dv, rv, f"dv mode {mode}")
    # lse: video rows [B*k][heads][n_pad] in set-slot order, then text rows [B][heads][L_pad]
    nv = grid[0] * grid[1] * grid[2]
    n = nv // kk
    n_pad, l_pad = (n + 127) // 128 * 128, (L + 127) // 128 * 128
    lv = lse[: B * kk * heads * n_pad].view(B * kk, heads, n_pad).double().cpu().numpy()
    lt = lse[B * kk * heads * n_pad:].view(B, heads, l_pad).double().cpu().numpy()
    scale = 1 / math.sqrt(d)
    qd, kd = to_f64(q), to_f64(k)
    sets = O.skiparse_sets(nv, kk, mode)
    for b in range(B):
        for h in range(heads):
            ref = O.attention_head_lse_ref(qd[b, :L, h], kd[b, :, h], scale) / math.log(2.0)
            np.testing.assert_allclose(lt[b, h, :L], ref, rtol=0, atol=2e-3)
            for g, st in enumerate(sets):
                rows = L + np.asarray(st)
                keys = np.concatenate([np.arange(L), rows])
                ref = O.attention_head_lse_ref(qd[b, rows, h], kd[b, keys, h], scale) / math.log(2.0)
                np.testing.assert_allclose(lv[b * kk + g, h, :n], ref, rtol=0, atol=2e-3)


FULL_SKIP = [("open_sora_plan", 0), ("open_sora_plan", 226), ("long_video", 0)]


@pytest.mark.parametrize("wl,L", FULL_SKIP, ids=[f"{w}_L{L}" for w, L in FULL_SKIP])
def test_full_size_skiparse_backward_sampled(gpu, wl, L):
    """Skiparse training at full size (Open-Sora Plan d = 96, 24 heads, 28,800 video tokens, k = 4;
    long video d = 128, 32 heads, 36,864 tokens, k = 4), Single then Group Skip on the same
    buffers, with and without 226 joined text tokens: sampled dQ rows and dK / dV rows of one head
    (video rows from the first and last set, and text rows) against the oracle's row form."""
    w = syn.WORKLOADS[wl]
    kk, nv = w.skiparse_k, w.n_video
    shape = (w.B, L + nv, w.heads, w.head_dim)
    q, k, v, do = (syn.randn_bf16(shape, w.seed + 40 + i) for i in range(4))
    qg, kg, vg, dog = (t.to(gpu) for t in (q, k, v, do))
    h = w.heads - 1
    q1, k1, v1, do1 = (to_f64(t[:, :, h:h + 1]) for t in (q, k, v, do))
    rng = np.random.default_rng(12)
    for mode in (0, 1):
        o, lse = ops.attn_forward_train(qg, kg, vg, w.grid, L, sparse_k=kk, mode=mode)
        dq, dk, dv = ops.attn_backward(qg, kg, vg, o, dog, lse, w.grid, L, sparse_k=kk, mode=mode)
        ops.check_status()
        sets = O.skiparse_sets(nv, kk, mode)
        vid = [sets[0][0], sets[0][-1], sets[-1][0], sets[-1][-1],
               *rng.choice(sets[0], 2).tolist(), *rng.choice(sets[-1], 2).tolist()]
        rows = sorted({L + int(x) for x in vid} | ({0, L - 1} if L else set()))
        rq, rk, rv = O.skiparse_text_backward_rows_ref(q1, k1, v1, do1, L, kk, mode, rows, rows)
        assert_grad_close(dq[0, rows, h], rq[0, :, 0], f"dq mode {mode}")
        assert_grad_close(dk[0, rows, h], rk[0, :, 0], f"dk mode {mode}")
        assert_grad_close(dv[0, rows, h], rv[0, :, 0], f"dv mode {mode}")
