"""GPU parity of the tcgen05 attention kernels against the fp64 oracle.

Tolerance: max-abs <= 2e-2 and relative-L2 <= 5e-3 for bf16 inputs.  Small cases
are compared element by element over the whole output; full-size workloads on sampled query
rows (every head) that the oracle computes one by one."""

import numpy as np
import pytest
import torch

import oracle as O
from spacetime_attention_b200 import ops, synthetic as syn
from tests.gpu_common import gpu  # noqa: F401
from tests.helpers import assert_attn_close, bf16_round, to_f64

pytestmark = pytest.mark.gpu

DENSE_CASES = [
    # name, B, heads, d, grid, text_len
    ("tiny", 1, 2, 64, (4, 8, 8), 0),
    ("one_kv_tile_ragged", 1, 2, 64, (1, 5, 9), 0),          # 45 tokens
    ("ragged_text", 2, 3, 64, (4, 8, 8), 44),                # 300 tokens: Q and KV tails
    ("three_q_tiles", 1, 2, 64, (3, 10, 13), 11),            # 401 tokens: 2 CTAs, 2nd half empty
    ("d96", 1, 3, 96, (3, 7, 13), 5),                        # 278 tokens
    ("d128", 2, 2, 128, (2, 9, 19), 0),                      # 342 tokens
    ("single_token", 1, 3, 64, (1, 1, 1), 0),
    ("long_kv", 1, 1, 64, (8, 16, 17), 9),                   # 2185 tokens: many KV tiles
]


def _qkv(dev, B, heads, d, grid, L, seed=3, scale_inputs=1.0):
    w = syn.custom("a", B, heads, d, grid, L, (d // 4, d // 4 + d // 8, d - d // 2 - d // 8))
    q, k, v = syn.make_qkv(w, seed)
    if scale_inputs != 1.0:
        q = (q.float() * scale_inputs).to(torch.bfloat16)
        k = (k.float() * scale_inputs).to(torch.bfloat16)
    return q, k, v, q.to(dev), k.to(dev), v.to(dev)


@pytest.mark.parametrize("case", DENSE_CASES, ids=[c[0] for c in DENSE_CASES])
def test_dense_attention_matches_oracle(gpu, case):
    _, B, heads, d, grid, L = case
    q, k, v, qg, kg, vg = _qkv(gpu, B, heads, d, grid, L)
    o = ops.attn_full(qg, kg, vg, grid, L)
    ops.check_status()
    ref = O.attn_ref(to_f64(q), to_f64(k), to_f64(v))
    assert_attn_close(o, ref, case[0])


def test_single_token_returns_v(gpu):
    q, k, v, qg, kg, vg = _qkv(gpu, 2, 3, 64, (1, 1, 1), 0)
    assert torch.equal(ops.attn_full(qg, kg, vg, (1, 1, 1), 0).cpu(), v)


def test_zero_queries_give_mean_of_v(gpu):
    q, k, v, qg, kg, vg = _qkv(gpu, 1, 2, 128, (2, 8, 10), 3)
    o = ops.attn_full(torch.zeros_like(qg), kg, vg, (2, 8, 10), 3)
    ref = np.broadcast_to(to_f64(v).mean(1, keepdims=True), o.shape)
    assert_attn_close(o, ref, "q=0")


@pytest.mark.parametrize("mag", [3.0, 6.0])
def test_large_scores_exercise_rescaling(gpu, mag):
    # scores with std ~ mag^2: the running max jumps often and the stale-max rescale path runs
    q, k, v, qg, kg, vg = _qkv(gpu, 1, 2, 64, (4, 8, 16), 0, seed=5, scale_inputs=mag)
    o = ops.attn_full(qg, kg, vg, (4, 8, 16), 0)
    assert_attn_close(o, O.attn_ref(to_f64(q), to_f64(k), to_f64(v)), f"mag{mag}")


def test_explicit_softmax_scale(gpu):
    q, k, v, qg, kg, vg = _qkv(gpu, 1, 2, 64, (2, 8, 8), 0)
    o = ops.attn_full(qg, kg, vg, (2, 8, 8), 0, scale=0.05)
    assert_attn_close(o, O.attn_ref(to_f64(q), to_f64(k), to_f64(v), scale=0.05), "scale")


def test_repeat_calls_are_deterministic(gpu):
    q, k, v, qg, kg, vg = _qkv(gpu, 1, 2, 96, (3, 7, 13), 5)
    a = ops.attn_full(qg, kg, vg, (3, 7, 13), 5)
    b = ops.attn_full(qg, kg, vg, (3, 7, 13), 5)
    assert torch.equal(a, b)


SPARSE_CASES = [
    # name, B, heads, d, grid, k
    ("tiny_k2", 1, 2, 64, (4, 8, 8), 2),
    ("ragged_set_k4", 1, 2, 64, (5, 8, 12), 4),       # 480 tokens, sets of 120 (< one tile)
    ("multi_tile_k2", 2, 2, 96, (4, 10, 15), 2),      # 600 tokens, sets of 300: tails
    ("d128_k4", 1, 2, 128, (4, 16, 18), 4),           # 1152 tokens, sets of 288
    ("k8_group", 1, 1, 64, (2, 16, 16), 8),           # 512 tokens, sets of 64
    ("k1", 1, 2, 64, (2, 5, 7), 1),
]


@pytest.mark.parametrize("case", SPARSE_CASES, ids=[c[0] for c in SPARSE_CASES])
@pytest.mark.parametrize("mode", [0, 1])
def test_skiparse_attention_matches_oracle(gpu, case, mode):
    _, B, heads, d, grid, k = case
    q, kk, v, qg, kg, vg = _qkv(gpu, B, heads, d, grid, 0)
    o = ops.skiparse_attn(qg, kg, vg, grid, k, mode)
    ops.check_status()
    ref = O.skiparse_attn_ref(to_f64(q), to_f64(kk), to_f64(v), k, mode)
    assert_attn_close(o, ref, f"{case[0]} mode {mode}")


@pytest.mark.parametrize("mode", [0, 1])
def test_fused_skiparse_equals_gather_dense_scatter(gpu, mode):
    # the fused kernel walks each set's tokens in slot order with the same tiles as dense
    # attention over the gathered k-fold batch: results must be bit-identical
    grid, k = (4, 10, 12), 4
    q, kk, v, qg, kg, vg = _qkv(gpu, 2, 3, 64, grid, 0)
    fused = ops.skiparse_attn(qg, kg, vg, grid, k, mode)
    gq, gk, gv = ops.skiparse_gather(qg, kg, vg, grid, k, mode)
    n_set = grid[0] * grid[1] * grid[2] // k
    dense = ops.attn_full(gq, gk, gv, (1, 1, n_set), 0)
    assert torch.equal(ops.skiparse_scatter(dense, grid, k, mode), fused)


def _sample_rows(n, count, seed):
    rng = np.random.default_rng(seed)
    rows = set(rng.choice(n, size=count - 4, replace=False).tolist())
    rows |= {0, n - 1, n // 2, min(n - 1, 127)}
    return sorted(rows)


@pytest.mark.parametrize("name", ["cogvideox_2b", "open_sora_plan", "cogvideox_5b", "long_video"])
def test_full_size_rope_then_dense_attention_sampled(gpu, name):
    """The bench's step (3D RoPE then dense attention) at full size, on sampled query rows of
    every head and sample.  The oracle rounds RoPE outputs to bf16 like the interface between the
    calls.  CogVideoX-5B (2 samples x 48 heads x 70 query blocks = 6,720 units) leaves 60 units
    for the last wave, which the kernel splits over KV ranges: they are the last 60 query blocks
    of sample 1, head 47, which most of the sampled rows fall in."""
    w = syn.WORKLOADS[name]
    q, k, v = syn.make_qkv(w)
    qr, kr = ops.rope3d(q.to(gpu), k.to(gpu), w.grid, w.text_len, w.split)
    o = ops.attn_full(qr, kr, v.to(gpu), w.grid, w.text_len)
    ops.check_status()
    rows = _sample_rows(w.seq_len, 64, w.seed)
    qo = to_f64(bf16_round(O.rope3d_ref(to_f64(q), w.grid, w.text_len, w.split)))
    ko = to_f64(bf16_round(O.rope3d_ref(to_f64(k), w.grid, w.text_len, w.split)))
    ref = O.attn_ref(qo, ko, to_f64(v), rows=rows)
    assert_attn_close(o[:, rows], ref, name)


@pytest.mark.parametrize("name,mode", [("open_sora_plan", 0), ("open_sora_plan", 1), ("long_video", 0),
                                       ("long_video", 1)])
def test_full_size_skiparse_sampled(gpu, name, mode):
    w = syn.WORKLOADS[name]
    q, k, v = syn.make_qkv(w)
    o = ops.skiparse_attn(q.to(gpu), k.to(gpu), v.to(gpu), w.grid, w.skiparse_k, mode)
    ops.check_status()
    rows = _sample_rows(w.n_video, 24, w.seed + mode)
    ref = O.skiparse_attn_ref(to_f64(q), to_f64(k), to_f64(v), w.skiparse_k, mode, rows=rows)
    assert_attn_close(o[:, rows], ref, f"{name} mode {mode}")


def test_full_size_long_video_skiparse_pair_on_the_bench_buffers(gpu):
    """The long-video bench step: RoPE into qr, kr, then Single Skip and Group Skip attention
    written one after the other into the same output buffer, on sampled rows of every head."""
    w = syn.WORKLOADS["long_video"]
    q, k, v = syn.make_qkv(w)
    qg, kg, vg = q.to(gpu), k.to(gpu), v.to(gpu)
    qr, kr, o = torch.empty_like(qg), torch.empty_like(kg), torch.empty_like(qg)
    ops.rope3d(qg, kg, w.grid, w.text_len, w.split, q_out=qr, k_out=kr)
    ops.skiparse_attn(qr, kr, vg, w.grid, w.skiparse_k, ops.OSP_SKIP_SINGLE, o=o)
    single = o.clone()
    ops.skiparse_attn(qr, kr, vg, w.grid, w.skiparse_k, ops.OSP_SKIP_GROUP, o=o)
    ops.check_status()
    qo = to_f64(bf16_round(O.rope3d_ref(to_f64(q), w.grid, w.text_len, w.split)))
    ko = to_f64(bf16_round(O.rope3d_ref(to_f64(k), w.grid, w.text_len, w.split)))
    rows = _sample_rows(w.n_video, 48, 77)
    for got, mode in ((single, O.SKIP_SINGLE), (o, O.SKIP_GROUP)):
        ref = O.skiparse_attn_ref(qo, ko, to_f64(v), w.skiparse_k, mode, rows=rows)
        assert_attn_close(got[:, rows], ref, f"long video pair, mode {mode}")


@pytest.mark.parametrize("jump", [12.0, 40.0, 200.0])
def test_row_max_jump_in_a_late_kv_tile(gpu, jump):
    """A key in the third KV tile scores far above everything before it (jump in log2 units of
    the scaled score): the running max must be raised and P, O and the row sum rescaled exactly,
    however large the jump."""
    B, heads, d, grid = 1, 2, 64, (2, 16, 16)     # 512 tokens = 4 KV tiles
    q, k, v, _, _, _ = _qkv(gpu, B, heads, d, grid, 0, seed=13)
    q = q.float(); k = k.float()
    q[:, :, :, 0] = 8.0                             # every query has a large first channel
    key = 300                                        # token in KV tile 2
    k[:, key, :, 0] = jump / (8.0 * 1.4426950408889634) * 8.0   # score * scale * log2(e) ~ jump
    q = q.to(torch.bfloat16); k = k.to(torch.bfloat16)
    o = ops.attn_full(q.to(gpu), k.to(gpu), v.to(gpu), grid, 0)
    ops.check_status()
    ref = O.attn_ref(to_f64(q), to_f64(k), to_f64(v))
    assert_attn_close(o, ref, f"jump {jump}")


@pytest.mark.parametrize("d,grid,L,sparse", [(64, (4, 15, 16), 40, None), (96, (4, 15, 16), 40, None),
                                             (128, (4, 15, 16), 40, None), (64, (4, 16, 16), 0, (2, 1)),
                                             (128, (8, 16, 16), 0, (4, 0))])
def test_split_kv_tail_matches_oracle_and_unsplit(gpu, monkeypatch, d, grid, L, sparse):
    """Few work units (fewer than SMs): the kernel splits each unit's KV range into parts whose
    fp32 partials are merged by the combine kernel.  Same result as the unsplit kernel (up to
    summation order) and as the oracle."""
    q, k, v, qg, kg, vg = _qkv(gpu, 1, 2, d, grid, L, seed=17)
    if sparse is None:
        run = lambda: ops.attn_full(qg, kg, vg, grid, L)
        ref = O.attn_ref(to_f64(q), to_f64(k), to_f64(v))
    else:
        kk, mode = sparse
        run = lambda: ops.skiparse_attn(qg, kg, vg, grid, kk, mode)
        ref = O.skiparse_attn_ref(to_f64(q), to_f64(k), to_f64(v), kk, mode)
    split = run()
    ops.check_status()
    monkeypatch.setenv("OSP_SPLIT_KV", "0")
    plain = run()
    ops.check_status()
    assert_attn_close(split, ref, "split")
    assert_attn_close(plain, ref, "unsplit")
    assert float((split.float() - plain.float()).abs().max()) <= 1e-2


def test_maximum_sequence_length_sampled(gpu):
    """A 2^20-token sequence (64 x 128 x 128 grid, one head, d = 64): 4,096 query blocks of 256
    rows and 8,192 KV tiles per block; sampled rows against the oracle."""
    grid = (64, 128, 128)
    N = grid[0] * grid[1] * grid[2]
    q, k, v = (syn.randn_bf16((1, N, 1, 64), 301 + i) for i in range(3))
    o = ops.attn_full(q.to(gpu), k.to(gpu), v.to(gpu), grid, 0)
    ops.check_status()
    rows = _sample_rows(N, 8, 3)
    ref = O.attn_ref(to_f64(q), to_f64(k), to_f64(v), rows=rows)
    assert_attn_close(o[:, rows], ref, "2^20 tokens")


@pytest.mark.parametrize("kind", ["dense", "skiparse", "cross", "frame_causal", "skiparse_text", "spatial"])
def test_items_in_turn_equal_one_item_per_cta(gpu, monkeypatch, kind):
    """CTAs that run several work items in turn (OSP_PERSIST=2, one CTA per SM) compute every item
    exactly as a CTA that runs one (OSP_PERSIST=0): bit-identical outputs, on shapes with more
    items than SMs and several KV tiles per item."""
    grid = (4, 16, 24)                    # 1,536 video tokens; 24 heads x 2 samples: 288+ items
    q, k, v, qg, kg, vg = _qkv(gpu, 2, 24, 64, grid, 40 if kind in ("dense", "frame_causal") else 0, seed=29)
    kt, vt = syn.randn_bf16((2, 300, 24, 64), 31).to(gpu), syn.randn_bf16((2, 300, 24, 64), 32).to(gpu)
    if kind in ("skiparse_text",):
        q, k, v, qg, kg, vg = _qkv(gpu, 2, 24, 64, grid, 77, seed=29)
    calls = {
        "dense": lambda: ops.attn_full(qg, kg, vg, grid, 40),
        "skiparse": lambda: ops.skiparse_attn(qg, kg, vg, grid, 2, 1),
        "cross": lambda: ops.attn_cross(qg, kt, vt, grid),
        "frame_causal": lambda: ops.attn_frame_causal(qg, kg, vg, grid, 40),
        "skiparse_text": lambda: ops.skiparse_attn(qg, kg, vg, grid, 2, 0, text_len=77),
        "spatial": lambda: ops.attn_spatial(qg, kg, vg, grid),
    }
    monkeypatch.setenv("OSP_SPLIT_KV", "0")
    monkeypatch.setenv("OSP_PERSIST", "0")
    one = calls[kind]()
    monkeypatch.setenv("OSP_PERSIST", "2")
    turns = calls[kind]()
    ops.check_status()
    assert torch.equal(one, turns)
