"""GPU parity of the factorized (2D + 1D) training calls: per-frame spatial and per-position
temporal attention, forward with saved log-sum-exp and backward, against the fp64 oracle
(spatial_backward_ref / temporal_backward_ref, pinned by finite differences and by reduction to
the dense, frame-causal and Single Skip backward).  Tolerances as the other backward tests: P and
dS rounded to bf16 before the tensor-core products, fp32 accumulation, bf16 outputs."""

import math

import numpy as np
import pytest
import torch

import oracle as O
from spacetime_attention_b200 import ops, synthetic as syn
from tests.gpu_common import gpu  # noqa: F401
from tests.helpers import assert_attn_close, to_f64
from tests.test_gpu_backward import assert_grad_close

pytestmark = pytest.mark.gpu


def _inputs(B, heads, d, grid, seed):
    N = grid[0] * grid[1] * grid[2]
    return tuple(syn.randn_bf16((B, N, heads, d), seed + i) for i in range(4))


SPATIAL = [
    # B, heads, d, grid
    (1, 2, 64, (3, 8, 16)),       # 128-token frames: one tile each
    (2, 2, 96, (2, 9, 15)),       # 135-token frames: ragged second tile
    (1, 1, 128, (4, 5, 7)),       # 35-token frames
]


@pytest.mark.parametrize("case", SPATIAL, ids=[f"{c[3]}_d{c[2]}_B{c[0]}" for c in SPATIAL])
def test_spatial_backward_matches_oracle(gpu, case):
    B, heads, d, grid = case
    q, k, v, do = _inputs(B, heads, d, grid, 120)
    qg, kg, vg, dog = (t.to(gpu) for t in (q, k, v, do))
    o, lse = ops.attn_spatial_train(qg, kg, vg, grid)
    dq, dk, dv = ops.attn_spatial_backward(qg, kg, vg, o, dog, lse, grid)
    ops.check_status()
    # the training forward is the inference forward, bit for bit
    assert torch.equal(o, ops.attn_spatial(qg, kg, vg, grid))
    rq, rk, rv = O.spatial_backward_ref(to_f64(q), to_f64(k), to_f64(v), to_f64(do), grid)
    assert_grad_close(dq, rq, "dq")
    assert_grad_close(dk, rk, "dk")
    assert_grad_close(dv, rv, "dv")
    # lse of frame t, head h, slot = the token's index within the frame (log2 domain)
    T, H, W = grid
    HW = H * W
    scale = 1 / math.sqrt(d)
    for b, t, h in ((0, 0, 0), (B - 1, T - 1, heads - 1)):
        f = slice(t * HW, (t + 1) * HW)
        ref = O.attention_head_lse_ref(to_f64(q)[b, f, h], to_f64(k)[b, f, h], scale) / math.log(2.0)
        np.testing.assert_allclose(lse[b * T + t, h, :HW].double().cpu().numpy(), ref, rtol=0, atol=2e-3)


TEMPORAL = [
    # B, heads, d, grid
    (1, 2, 64, (13, 3, 4)),       # 13 frames, one partial tile per position
    (1, 2, 96, (33, 2, 5)),       # three 16-row tiles per set (per-set kernel), ragged
    (2, 1, 128, (64, 3, 1)),      # the per-set kernel's largest sets
    (2, 1, 96, (80, 2, 3)),       # longer than the inference kernel's shared-memory limit
    (1, 2, 128, (130, 1, 2)),     # two tiles per position, ragged
    (1, 1, 64, (7, 1, 1)),        # one position: the dense layout
    (1, 1, 64, (13, 16, 20)),     # 320 one-tile work units: the forward runs them in turn
]


@pytest.fixture(params=["per_set", "tiles"])
def temporal_path(request, monkeypatch):
    """T <= 64: the per-set temporal backward kernel, or the Skiparse backward kernels on one
    128-row tile per set (T > 64 always takes the latter)."""
    monkeypatch.setenv("OSP_TEMPORAL_BWD", "1" if request.param == "per_set" else "0")
    return request.param


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("case", TEMPORAL, ids=[f"{c[3]}_d{c[2]}_B{c[0]}" for c in TEMPORAL])
def test_temporal_backward_matches_oracle(gpu, case, causal, temporal_path):
    B, heads, d, grid = case
    q, k, v, do = _inputs(B, heads, d, grid, 130 + causal)
    qg, kg, vg, dog = (t.to(gpu) for t in (q, k, v, do))
    o, lse = ops.attn_temporal_train(qg, kg, vg, grid, causal=causal)
    dq, dk, dv = ops.attn_temporal_backward(qg, kg, vg, o, dog, lse, grid, causal=causal)
    ops.check_status()
    qd, kd, vd = to_f64(q), to_f64(k), to_f64(v)
    assert_attn_close(o, O.temporal_attn_ref(qd, kd, vd, grid, causal=causal), f"temporal train {grid}")
    rq, rk, rv = O.temporal_backward_ref(qd, kd, vd, to_f64(do), grid, causal=causal)
    assert_grad_close(dq, rq, "dq")
    assert_grad_close(dk, rk, "dk")
    assert_grad_close(dv, rv, "dv")
    # lse of position pos, head h, slot t: over keys t' (all, or t' <= t when causal)
    T, H, W = grid
    HW = H * W
    scale = 1 / math.sqrt(d)
    for b, pos, h in ((0, 0, 0), (B - 1, HW - 1, heads - 1)):
        idx = pos + HW * np.arange(T)
        got = lse[b * HW + pos, h, :T].double().cpu().numpy()
        if causal:
            ref = np.array([O.attention_head_lse_ref(qd[b, idx[t:t + 1], h], kd[b, idx[:t + 1], h], scale)[0]
                            for t in range(T)])
        else:
            ref = O.attention_head_lse_ref(qd[b, idx, h], kd[b, idx, h], scale)
        np.testing.assert_allclose(got, ref / math.log(2.0), rtol=0, atol=2e-3)


def test_causal_temporal_first_frame_has_no_query_gradient(gpu, temporal_path):
    # a first-frame query sees only its own key: softmax over one key, so dQ = 0 up to the fp32
    # rounding of dP - rowsum(dO * O) (two sums of the same products in different orders)
    q, k, v, do = _inputs(1, 2, 64, (6, 4, 4), 140)
    qg, kg, vg, dog = (t.to(gpu) for t in (q, k, v, do))
    o, lse = ops.attn_temporal_train(qg, kg, vg, (6, 4, 4), causal=True)
    dq, _, _ = ops.attn_temporal_backward(qg, kg, vg, o, dog, lse, (6, 4, 4), causal=True)
    ops.check_status()
    first, rest = dq[:, :16].float().abs().max().item(), dq[:, 16:].float().abs().max().item()
    assert rest > 0 and first <= 1e-2 * rest


@pytest.mark.parametrize("causal", [False, True])
def test_per_set_temporal_training_forward_equals_inference(gpu, monkeypatch, causal):
    # T <= 64: the training forward runs the inference kernel with its lse output switched on
    monkeypatch.setenv("OSP_TEMPORAL_BWD", "1")
    grid = (13, 6, 10)
    q, k, v, _ = _inputs(2, 3, 64, grid, 150 + causal)
    qg, kg, vg = (t.to(gpu) for t in (q, k, v))
    o_train, _ = ops.attn_temporal_train(qg, kg, vg, grid, causal=causal)
    o_inf = ops.attn_temporal(qg, kg, vg, grid, causal=causal)
    ops.check_status()
    assert torch.equal(o_train, o_inf)


def test_full_size_factorized_and_frame_causal_backward_sampled(gpu):
    """CogVideoX-2B grid at full size (13x30x45, 30 heads, d = 64): spatial, temporal (both in
    time directions) and frame-causal (with the 226 text tokens) training, sampled rows of one
    head against the oracle: spatial on whole frames through the dense row form, temporal on a
    subset of positions through temporal_backward_ref, frame-causal through its row form."""
    w = syn.WORKLOADS["cogvideox_2b"]
    T, H, W = w.grid
    HW, L = H * W, w.text_len
    h = 7
    q, k, v, do = (syn.randn_bf16((1, L + T * HW, w.heads, w.head_dim), w.seed + 60 + i) for i in range(4))
    qg, kg, vg, dog = (t.to(gpu) for t in (q, k, v, do))
    vid = [t[:, L:].contiguous() for t in (qg, kg, vg, dog)]
    qv, kv, vv, dov = (to_f64(t[:, L:, h:h + 1]) for t in (q, k, v, do))
    scale = 1 / math.sqrt(w.head_dim)
    rng = np.random.default_rng(21)
    # spatial: frames 0, 6 and 12, sampled rows of each
    o, lse = ops.attn_spatial_train(*vid[:3], w.grid)
    dq, dk, dv = ops.attn_spatial_backward(vid[0], vid[1], vid[2], o, vid[3], lse, w.grid)
    ops.check_status()
    for t in (0, 6, T - 1):
        f = slice(t * HW, (t + 1) * HW)
        rows = sorted({0, HW - 1, *rng.integers(0, HW, size=4).tolist()})
        rq, rk, rv = O.attention_head_backward_rows_ref(qv[0, f, 0], kv[0, f, 0], vv[0, f, 0], dov[0, f, 0], scale,
                                                        rows, rows)
        sel = [t * HW + r for r in rows]
        assert_grad_close(dq[0, sel, h], rq, f"spatial dq frame {t}")
        assert_grad_close(dk[0, sel, h], rk, f"spatial dk frame {t}")
        assert_grad_close(dv[0, sel, h], rv, f"spatial dv frame {t}")
    # temporal: 64 positions (their T tokens each) against temporal_backward_ref on that subset
    pos = np.sort(rng.choice(HW, size=64, replace=False))
    idx = (pos[None, :] + HW * np.arange(T)[:, None]).reshape(-1)          # frame-major, as a (T, 1, 64) grid
    for causal in (False, True):
        o, lse = ops.attn_temporal_train(*vid[:3], w.grid, causal=causal)
        dq, dk, dv = ops.attn_temporal_backward(vid[0], vid[1], vid[2], o, vid[3], lse, w.grid, causal=causal)
        ops.check_status()
        ref = O.temporal_backward_ref(qv[:, idx], kv[:, idx], vv[:, idx], dov[:, idx], (T, 1, len(pos)), causal=causal)
        for got, r, name in zip((dq, dk, dv), ref, ("dq", "dk", "dv")):
            assert_grad_close(got[0, idx, h], r[0, :, 0], f"temporal {name} causal={causal}")
    # frame-causal over text + video: text rows, rows of the first and last frames
    o, lse = ops.attn_frame_causal_train(qg, kg, vg, w.grid, L)
    dq, dk, dv = ops.attn_frame_causal_backward(qg, kg, vg, o, dog, lse, w.grid, L)
    ops.check_status()
    rows = sorted({0, L - 1, L, L + HW - 1, L + (T - 1) * HW, L + T * HW - 1,
                   *(L + rng.integers(0, T * HW, size=4)).tolist()})
    q1, k1, v1, d1 = (to_f64(t[:, :, h:h + 1]) for t in (q, k, v, do))
    rq, rk, rv = O.frame_causal_backward_rows_ref(q1, k1, v1, d1, w.grid, L, rows, rows)
    assert_grad_close(dq[0, rows, h], rq[0, :, 0], "frame-causal dq")
    assert_grad_close(dk[0, rows, h], rk[0, :, 0], "frame-causal dk")
    assert_grad_close(dv[0, rows, h], rv[0, :, 0], "frame-causal dv")
