"""Pins of the fp64 oracle against what the pages and the mathematics fix.

Nothing here compares the oracle with itself: every expected value is a hand-written fixture
(tests/golden/, each with its source), a closed form, an invariant, or a brute-force pure-Python
evaluation of the definition on tiny inputs.  Each group is chosen so that a plausible slip in
the oracle (a dropped term, a wrong sign or index, a transposed operand, a wrong frequency or
pairing convention) fails at least one test.
"""

import math
import os

import numpy as np
import pytest

import oracle as O


# ----------------------------------------------------------------------------------------------
# fixtures
# ----------------------------------------------------------------------------------------------

def _read_sets(golden_dir):
    cases = []
    with open(os.path.join(golden_dir, "skiparse_sets.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            head, body = line.split(":")
            mode, n, k = head.split()
            sets = [[int(t) for t in part.split()] for part in body.split("|")]
            cases.append((O.SKIP_SINGLE if mode == "single" else O.SKIP_GROUP, int(n), int(k), sets))
    return cases


def _read_rope(golden_dir):
    rows = []
    with open(os.path.join(golden_dir, "rope_unit_rotations.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            p = line.split()
            rows.append((int(p[0]), int(p[1]), int(p[2]), int(p[3]), int(p[4]), float(p[5]),
                         int(p[6]), float(p[7])))
    return rows


# ----------------------------------------------------------------------------------------------
# index maps
# ----------------------------------------------------------------------------------------------

def test_sets_match_hand_written_golden(golden_dir):
    cases = _read_sets(golden_dir)
    assert len(cases) >= 8
    for mode, n, k, sets in cases:
        assert O.skiparse_sets(n, k, mode) == sets, (mode, n, k)


@pytest.mark.parametrize("mode", [O.SKIP_SINGLE, O.SKIP_GROUP])
def test_sets_are_partitions_exhaustive(mode):
    for k in range(1, 7):
        step = k if mode == O.SKIP_SINGLE else k * k
        for n in range(step, 73, step):
            sets = O.skiparse_sets(n, k, mode)
            assert len(sets) == k
            assert all(len(s) == n // k for s in sets)
            assert sorted(t for s in sets for t in s) == list(range(n))
            assert all(s == sorted(s) for s in sets)
            m = O.skiparse_index_map(n, k, mode)
            assert m.dtype == np.int32 and sorted(m.tolist()) == list(range(n))


def test_single_skip_membership_is_residue_class():
    for k in range(1, 6):
        n = 12 * k
        for g, s in enumerate(O.skiparse_sets(n, k, O.SKIP_SINGLE)):
            assert all(t % k == g for t in s)


def test_group_skip_connects_groups_k_minus_1_apart():
    # tokens i, j in one set: their groups floor(i/k), floor(j/k) differ by a multiple of k,
    # i.e. k-1 groups lie between consecutive groups of a set; and each group is whole.
    for k in range(2, 6):
        n = 3 * k * k
        for s in O.skiparse_sets(n, k, O.SKIP_GROUP):
            groups = sorted({t // k for t in s})
            for a, b in zip(groups, groups[1:]):
                assert b - a == k
            for gr in groups:
                assert all(gr * k + r in s for r in range(k))


def test_k1_is_identity_and_divisibility_errors():
    for mode in (O.SKIP_SINGLE, O.SKIP_GROUP):
        assert O.skiparse_index_map(10, 1, mode).tolist() == list(range(10))
    with pytest.raises(ValueError):
        O.skiparse_sets(10, 4, O.SKIP_SINGLE)
    with pytest.raises(ValueError):
        O.skiparse_sets(8, 4, O.SKIP_GROUP)


def test_config_sizes_divide():
    # 4x8x8 with k=2; 24x30x40 and 16x36x64 with k=4 (single needs k | N, group k^2 | N)
    for n, k in [(256, 2), (28800, 4), (36864, 4)]:
        for mode in (O.SKIP_SINGLE, O.SKIP_GROUP):
            m = O.skiparse_index_map(n, k, mode)
            assert np.array_equal(np.sort(m), np.arange(n))


# ----------------------------------------------------------------------------------------------
# gather / scatter
# ----------------------------------------------------------------------------------------------

def test_gather_layout_and_inverse(golden_dir):
    rng = np.random.default_rng(0)
    x = rng.standard_normal((2, 8, 3, 4))
    y = O.skiparse_gather_ref(x, 2, O.SKIP_GROUP)
    assert y.shape == (4, 4, 3, 4)
    # group, n=8, k=2: set0 = 0 1 4 5, set1 = 2 3 6 7 (golden); batch order b*k + g
    assert np.array_equal(y[0], x[0, [0, 1, 4, 5]])
    assert np.array_equal(y[1], x[0, [2, 3, 6, 7]])
    assert np.array_equal(y[3], x[1, [2, 3, 6, 7]])
    for mode in (O.SKIP_SINGLE, O.SKIP_GROUP):
        assert np.array_equal(O.skiparse_scatter_ref(O.skiparse_gather_ref(x, 2, mode), 2, mode), x)


# ----------------------------------------------------------------------------------------------
# 3D RoPE
# ----------------------------------------------------------------------------------------------

def test_rope_unit_vectors_match_closed_forms(golden_dir):
    rows = _read_rope(golden_dir)
    assert len(rows) >= 6
    for t, h, w, cin, ca, va, cb, vb in rows:
        x = np.zeros((1, 1, 1, 24))
        x[0, 0, 0, cin] = 1.0
        y = O.rope3d_positions_ref(x, [t], [h], [w], (8, 8, 8), 10000.0)[0, 0, 0]
        expect = np.zeros(24)
        expect[ca] = va
        expect[cb] = vb
        np.testing.assert_allclose(y, expect, rtol=0, atol=1e-14)


def test_rope_identity_at_origin_and_on_text_tokens():
    rng = np.random.default_rng(1)
    x = rng.standard_normal((2, 5 + 2 * 3 * 4, 3, 64))
    y = O.rope3d_ref(x, (2, 3, 4), 5, (16, 24, 24))
    assert np.array_equal(y[:, :5], x[:, :5])          # text tokens untouched
    assert np.array_equal(y[:, 5], x[:, 5])            # video token 0 is at (0,0,0)
    assert not np.allclose(y[:, 6], x[:, 6])           # token 1 is at (0,0,1)


def test_rope_token_positions_follow_raster_order():
    # token v of a 2x3x4 grid: t = v // 12, h = (v // 4) % 3, w = v % 4
    t, h, w = O.video_positions(2, 3, 4)
    assert (t[13], h[13], w[13]) == (1, 0, 1)
    assert (t[11], h[11], w[11]) == (0, 2, 3)
    # and rope3d_ref uses them: only the w chunk of token 1 rotates, only h of token 4, t of 12
    x = np.ones((1, 24, 1, 24))
    y = O.rope3d_ref(x, (2, 3, 4), 0, (8, 8, 8))[0, :, 0]
    changed = lambda v: np.nonzero(~np.isclose(y[v], 1.0))[0]
    assert set(changed(1)) <= set(range(16, 24)) and len(changed(1)) > 0
    assert set(changed(4)) <= set(range(8, 16)) and len(changed(4)) > 0
    assert set(changed(12)) <= set(range(0, 8)) and len(changed(12)) > 0


def test_rope_preserves_pair_norms():
    rng = np.random.default_rng(2)
    x = rng.standard_normal((1, 3 * 4 * 5, 2, 96))
    y = O.rope3d_ref(x, (3, 4, 5), 0, (32, 32, 32))
    nx = x[..., 0::2] ** 2 + x[..., 1::2] ** 2
    ny = y[..., 0::2] ** 2 + y[..., 1::2] ** 2
    np.testing.assert_allclose(ny, nx, rtol=1e-13, atol=1e-13)


@pytest.mark.parametrize("split", [(16, 24, 24), (32, 32, 32), (32, 48, 48)])
def test_rope_score_depends_only_on_offset(split):
    d = sum(split)
    rng = np.random.default_rng(3)
    q = rng.standard_normal((1, 6, 1, d))
    k = rng.standard_normal((1, 6, 1, d))
    pt, ph, pw = rng.integers(0, 40, 6), rng.integers(0, 40, 6), rng.integers(0, 40, 6)
    rq = O.rope3d_positions_ref(q, pt, ph, pw, split)[0, :, 0]
    rk = O.rope3d_positions_ref(k, pt, ph, pw, split)[0, :, 0]
    s0 = rq @ rk.T
    for shift in [(1, 0, 0), (0, 5, 0), (0, 0, 7), (3, 11, 29)]:
        sq = O.rope3d_positions_ref(q, pt + shift[0], ph + shift[1], pw + shift[2], split)[0, :, 0]
        sk = O.rope3d_positions_ref(k, pt + shift[0], ph + shift[1], pw + shift[2], split)[0, :, 0]
        np.testing.assert_allclose(sq @ sk.T, s0, rtol=0, atol=1e-11)
    # and it does depend on the offset
    sq = O.rope3d_positions_ref(q, pt + np.arange(6), ph, pw, split)[0, :, 0]
    assert not np.allclose(sq @ rk.T, s0)


def test_rope_one_axis_grid_is_textbook_1d_rope():
    # H = W = 1: the h and w chunks sit at position 0 (identity) and the t chunk is RoFormer's
    # 1D RoPE, written here as complex multiplication z * exp(i * pos * omega).
    T, d_t, d_h, d_w = 9, 16, 8, 8
    rng = np.random.default_rng(4)
    x = rng.standard_normal((1, T, 1, d_t + d_h + d_w))
    y = O.rope3d_ref(x, (T, 1, 1), 0, (d_t, d_h, d_w))
    np.testing.assert_array_equal(y[..., d_t:], x[..., d_t:])
    for pos in range(T):
        for j in range(d_t // 2):
            z = complex(x[0, pos, 0, 2 * j], x[0, pos, 0, 2 * j + 1])
            zr = z * complex(math.cos(pos * 10000.0 ** (-j / 8.0)), math.sin(pos * 10000.0 ** (-j / 8.0)))
            assert abs(y[0, pos, 0, 2 * j] - zr.real) < 1e-12
            assert abs(y[0, pos, 0, 2 * j + 1] - zr.imag) < 1e-12


# ----------------------------------------------------------------------------------------------
# attention
# ----------------------------------------------------------------------------------------------

def _brute_masked_attention(q, k, v, allowed, scale):
    """Pure-Python loops: o_i = sum_j e^{s_ij - m_i} v_j / sum_j e^{s_ij - m_i} over allowed j."""
    n, d = len(q), len(q[0])
    out = []
    for i in range(n):
        js = [j for j in range(len(k)) if allowed(i, j)]
        s = [sum(q[i][c] * k[j][c] for c in range(d)) * scale for j in js]
        m = max(s)
        e = [math.exp(x - m) for x in s]
        z = sum(e)
        out.append([sum(e[t] * v[js[t]][c] for t in range(len(js))) / z for c in range(d)])
    return np.asarray(out)


def test_attention_matches_brute_force():
    rng = np.random.default_rng(5)
    B, N, nh, d = 2, 7, 2, 5
    q, k, v = (rng.standard_normal((B, N, nh, d)) for _ in range(3))
    got = O.attn_ref(q, k, v)
    for b in range(B):
        for h in range(nh):
            ref = _brute_masked_attention(q[b, :, h].tolist(), k[b, :, h].tolist(), v[b, :, h].tolist(),
                                          lambda i, j: True, 1 / math.sqrt(d))
            np.testing.assert_allclose(got[b, :, h], ref, rtol=1e-12, atol=1e-13)


def test_attention_two_key_closed_form():
    # q.k0 - q.k1 = ln 3 (scale 1) -> weights 3/4, 1/4
    q = np.zeros((1, 1, 1, 2)); q[0, 0, 0, 0] = 1.0
    k = np.zeros((1, 2, 1, 2)); k[0, 0, 0, 0] = math.log(3.0)
    v = np.zeros((1, 2, 1, 2)); v[0, 0, 0] = [4.0, 0.0]; v[0, 1, 0] = [0.0, 8.0]
    kk = np.concatenate([k, k], axis=1)[:, :2]
    o = O.attn_ref(np.concatenate([q, q], axis=1), kk, v, scale=1.0)
    np.testing.assert_allclose(o[0, 0, 0], [3.0, 2.0], rtol=1e-14)
    # the softmax scale multiplies the scores: scale 2 -> weights 9/10, 1/10
    o2 = O.attn_ref(np.concatenate([q, q], axis=1), kk, v, scale=2.0)
    np.testing.assert_allclose(o2[0, 0, 0], [3.6, 0.8], rtol=1e-14)


def test_softmax_rows_sum_to_one():
    rng = np.random.default_rng(6)
    s = rng.standard_normal((9, 31)) * 30
    p = O.softmax_rows(s)
    assert (p >= 0).all()
    np.testing.assert_allclose(p.sum(-1), 1.0, rtol=0, atol=1e-14)
    assert np.argmax(p, -1).tolist() == np.argmax(s, -1).tolist()


def test_attention_special_cases():
    rng = np.random.default_rng(7)
    k, v = rng.standard_normal((1, 11, 2, 8)), rng.standard_normal((1, 11, 2, 8))
    o = O.attn_ref(np.zeros((1, 11, 2, 8)), k, v)            # q = 0 -> mean of v
    np.testing.assert_allclose(o, np.broadcast_to(v.mean(1, keepdims=True), o.shape), atol=1e-14)
    q1, k1, v1 = (rng.standard_normal((1, 1, 3, 8)) for _ in range(3))
    np.testing.assert_allclose(O.attn_ref(q1, k1, v1), v1, atol=1e-15)   # one token -> v
    # huge scores do not overflow (max subtraction)
    o = O.attn_ref(q1 * 1e3, k1 * 1e3, v1)
    assert np.isfinite(o).all()


def test_attention_rows_heads_subset():
    rng = np.random.default_rng(8)
    q, k, v = (rng.standard_normal((2, 40, 3, 8)) for _ in range(3))
    full = O.attn_ref(q, k, v)
    rows, heads = [0, 7, 39], [2, 0]
    np.testing.assert_allclose(O.attn_ref(q, k, v, rows=rows, heads=heads),
                               full[:, rows][:, :, heads], rtol=0, atol=1e-14)


@pytest.mark.parametrize("mode,k", [(O.SKIP_SINGLE, 2), (O.SKIP_GROUP, 2), (O.SKIP_SINGLE, 3),
                                    (O.SKIP_GROUP, 3), (O.SKIP_SINGLE, 4)])
def test_skiparse_is_masked_full_attention_brute_force(mode, k):
    # membership written independently of the oracle's set lists:
    # single: same residue mod k; group: same group index mod k.
    N = 36 if k == 3 else 16 if k == 4 else 24
    rng = np.random.default_rng(9 + k)
    q, kk, v = (rng.standard_normal((1, N, 1, 4)) for _ in range(3))
    if mode == O.SKIP_SINGLE:
        allowed = lambda i, j: i % k == j % k
    else:
        allowed = lambda i, j: (i // k) % k == (j // k) % k
    ref = _brute_masked_attention(q[0, :, 0].tolist(), kk[0, :, 0].tolist(), v[0, :, 0].tolist(),
                                  allowed, 0.5)
    got = O.skiparse_attn_ref(q, kk, v, k, mode)[0, :, 0]
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-13)
    # and the sparse result differs from dense attention
    assert not np.allclose(got, O.attn_ref(q, kk, v)[0, :, 0])


def test_skiparse_k1_is_dense_and_rows_subset():
    rng = np.random.default_rng(10)
    q, k, v = (rng.standard_normal((2, 32, 2, 8)) for _ in range(3))
    for mode in (O.SKIP_SINGLE, O.SKIP_GROUP):
        np.testing.assert_allclose(O.skiparse_attn_ref(q, k, v, 1, mode), O.attn_ref(q, k, v),
                                   rtol=0, atol=1e-13)
        full = O.skiparse_attn_ref(q, k, v, 2, mode)
        rows = [1, 5, 30]
        np.testing.assert_allclose(O.skiparse_attn_ref(q, k, v, 2, mode, rows=rows, heads=[1]),
                                   full[:, rows][:, :, [1]], rtol=0, atol=1e-14)


def test_skiparse_equals_gather_dense_scatter():
    # the k-fold batch formulation of the page: gather -> dense attention -> scatter
    rng = np.random.default_rng(11)
    q, k, v = (rng.standard_normal((2, 32, 2, 8)) for _ in range(3))
    for mode in (O.SKIP_SINGLE, O.SKIP_GROUP):
        g = [O.skiparse_gather_ref(t, 2, mode) for t in (q, k, v)]
        o = O.skiparse_scatter_ref(O.attn_ref(*g), 2, mode)
        np.testing.assert_allclose(o, O.skiparse_attn_ref(q, k, v, 2, mode), rtol=0, atol=1e-13)


# ----------------------------------------------------------------------------------------------
# bf16 storage rounding
# ----------------------------------------------------------------------------------------------

def test_round_to_bf16_hand_values():
    # bf16 has 8 significand bits: spacing 2^-7 on [1, 2), 2^-6 on [2, 4)
    cases = [
        (1.0, 1.0),
        (1.0 + 2 ** -8, 1.0),                        # tie -> even (1.0)
        (1.0 + 3 * 2 ** -8, 1.0 + 2 ** -6),          # tie -> even (1 + 2^-6 has even last bit)
        (1.0 + 2 ** -8 + 2 ** -40, 1.0 + 2 ** -7),   # just above the tie: up (needs the sticky bit)
        (1.0 + 2 ** -8 - 2 ** -40, 1.0),             # just below: down
        (-(1.0 + 2 ** -8 + 2 ** -40), -(1.0 + 2 ** -7)),
        (3.0 + 2 ** -7, 3.0),                        # tie on [2,4) -> even
        (0.0, 0.0),
        (2.0 ** -130, 2.0 ** -130),                  # subnormal in fp32, exact in bf16
    ]
    got = O.round_to_bf16(np.array([c[0] for c in cases]))
    np.testing.assert_array_equal(got, [c[1] for c in cases])


def test_round_to_bf16_is_nearest():
    rng = np.random.default_rng(12)
    x = rng.standard_normal(20000) * np.exp(rng.uniform(-20, 20, 20000))
    r = O.round_to_bf16(x)
    # result has at most 8 significant bits and is within half a bf16 spacing of x
    m, e = np.frexp(r)
    assert np.all(m * 2 ** 8 == np.round(m * 2 ** 8))
    spacing = 2.0 ** (np.floor(np.log2(np.abs(x))) - 7)
    assert np.all(np.abs(r - x) <= spacing / 2)


# ----------------------------------------------------------------------------------------------
# cross-attention (video queries, text keys/values)
# ----------------------------------------------------------------------------------------------

def test_cross_attention_brute_force_and_special_cases():
    rng = np.random.default_rng(13)
    q = rng.standard_normal((2, 6, 2, 4))
    k = rng.standard_normal((2, 3, 2, 4))
    v = rng.standard_normal((2, 3, 2, 4))
    got = O.cross_attn_ref(q, k, v)
    for b in range(2):
        for h in range(2):
            ref = _brute_masked_attention(q[b, :, h].tolist(), k[b, :, h].tolist(), v[b, :, h].tolist(),
                                          lambda i, j: True, 0.5)
            np.testing.assert_allclose(got[b, :, h], ref, rtol=1e-12, atol=1e-13)
    # one text token: every video query returns that token's value
    np.testing.assert_allclose(O.cross_attn_ref(q, k[:, :1], v[:, :1]), np.broadcast_to(v[:, :1], q.shape), atol=1e-15)
    # closed form with 3 video queries and 2 text keys: q.k0 - q.k1 = ln 3 -> weights 3/4, 1/4
    q3 = np.zeros((1, 3, 1, 2)); q3[0, :, 0, 0] = 1.0
    k2 = np.zeros((1, 2, 1, 2)); k2[0, 0, 0, 0] = math.log(3.0)
    v2 = np.zeros((1, 2, 1, 2)); v2[0, 0, 0] = [4.0, 0.0]; v2[0, 1, 0] = [0.0, 8.0]
    np.testing.assert_allclose(O.cross_attn_ref(q3, k2, v2, scale=1.0)[0, :, 0], [[3.0, 2.0]] * 3, rtol=1e-14)
    # rows / heads subsets agree with the full result
    np.testing.assert_allclose(O.cross_attn_ref(q, k, v, rows=[5, 0], heads=[1]), got[:, [5, 0]][:, :, [1]],
                               rtol=0, atol=1e-15)


# ----------------------------------------------------------------------------------------------
# packed batches (Multi-Resolution Frame Pack)
# ----------------------------------------------------------------------------------------------

def test_segment_bounds():
    assert O.segment_bounds([3, 1, 4]).tolist() == [0, 3, 4, 8]
    assert O.segment_bounds([]).tolist() == [0]


def test_packed_attention_is_block_diagonal_brute_force():
    rng = np.random.default_rng(21)
    seg = [0, 0, 0, 1, 2, 2, 2, 2]          # sample of each packed token, written out by hand
    q, k, v = (rng.standard_normal((1, 8, 2, 3)) for _ in range(3))
    got = O.packed_attn_ref(q, k, v, [0, 3, 4, 8])
    for h in range(2):
        ref = _brute_masked_attention(q[0, :, h].tolist(), k[0, :, h].tolist(), v[0, :, h].tolist(),
                                      lambda i, j: seg[i] == seg[j], 1 / math.sqrt(3))
        np.testing.assert_allclose(got[0, :, h], ref, rtol=1e-12, atol=1e-13)
    # the one-token sample returns its own value
    np.testing.assert_allclose(got[0, 3], v[0, 3], atol=1e-15)
    # row / head subsets agree with the full result
    np.testing.assert_allclose(O.packed_attn_ref(q, k, v, [0, 3, 4, 8], rows=[7, 3, 0], heads=[1]),
                               got[:, [7, 3, 0]][:, :, [1]], rtol=0, atol=1e-15)


def test_packed_cross_attention_pairs_segments_brute_force():
    rng = np.random.default_rng(22)
    qseg = [0, 0, 1, 1, 1]                   # 2 samples: 2 and 3 queries
    kseg = [0, 0, 0, 1]                      # 3 and 1 keys
    q = rng.standard_normal((1, 5, 1, 4))
    k = rng.standard_normal((1, 4, 1, 4))
    v = rng.standard_normal((1, 4, 1, 4))
    got = O.packed_attn_ref(q, k, v, [0, 2, 5], [0, 3, 4], scale=0.7)
    ref = _brute_masked_attention(q[0, :, 0].tolist(), k[0, :, 0].tolist(), v[0, :, 0].tolist(),
                                  lambda i, j: qseg[i] == kseg[j], 0.7)
    np.testing.assert_allclose(got[0, :, 0], ref, rtol=1e-12, atol=1e-13)
    # sample 1 has one key: its queries all return that value
    np.testing.assert_allclose(got[0, 2:, 0], np.broadcast_to(v[0, 3, 0], (3, 4)), atol=1e-15)


def test_packed_rope_restarts_positions_per_sample():
    # sample 0: 2 text tokens + a 1x2x3 grid; sample 1: no text + a 2x1x2 grid.  Positions written
    # by hand (t, h, w), w fastest, restarting at the origin for every sample.
    samples = [(2, 1, 2, 3), (0, 2, 1, 2)]
    pos0 = [(0, 0, 0), (0, 0, 1), (0, 0, 2), (0, 1, 0), (0, 1, 1), (0, 1, 2)]
    pos1 = [(0, 0, 0), (0, 0, 1), (1, 0, 0), (1, 0, 1)]
    split = (8, 8, 8)
    rng = np.random.default_rng(23)
    x = rng.standard_normal((1, 2 + 6 + 4, 2, 24))
    y = O.rope3d_packed_ref(x, samples, split)
    np.testing.assert_array_equal(y[0, :2], x[0, :2])                  # text untouched
    np.testing.assert_array_equal(y[0, 2], x[0, 2])                    # sample 0 origin
    np.testing.assert_array_equal(y[0, 8], x[0, 8])                    # sample 1 origin
    for base, pos in ((2, pos0), (8, pos1)):
        for r, (t, h, w) in enumerate(pos):
            # a 1D rotation per axis pair (RoFormer) checked through complex multiplication
            for c in range(0, 24, 2):
                axis, j = divmod(c, 8)
                p = (t, h, w)[axis]
                ang = p * 10000.0 ** (-(j / 2) * 2 / 8)
                for hd in range(2):
                    z = complex(x[0, base + r, hd, c], x[0, base + r, hd, c + 1]) * complex(math.cos(ang), math.sin(ang))
                    assert abs(y[0, base + r, hd, c] - z.real) < 1e-12
                    assert abs(y[0, base + r, hd, c + 1] - z.imag) < 1e-12


# ----------------------------------------------------------------------------------------------
# factorized (2D + 1D) and frame-causal masks
# ----------------------------------------------------------------------------------------------

def _coords(T, H, W):
    """(t, h, w) of every video token by nested loops (w fastest), written independently."""
    out = []
    for t in range(T):
        for h in range(H):
            for w in range(W):
                out.append((t, h, w))
    return out


@pytest.mark.parametrize("grid", [(3, 2, 2), (2, 1, 3)])
def test_spatial_and_temporal_attention_brute_force(grid):
    T, H, W = grid
    N = T * H * W
    c = _coords(T, H, W)
    rng = np.random.default_rng(40)
    q, k, v = (rng.standard_normal((1, N, 2, 3)) for _ in range(3))
    sp = O.spatial_attn_ref(q, k, v, grid)
    te = O.temporal_attn_ref(q, k, v, grid)
    tc = O.temporal_attn_ref(q, k, v, grid, causal=True)
    for h in range(2):
        args = (q[0, :, h].tolist(), k[0, :, h].tolist(), v[0, :, h].tolist())
        np.testing.assert_allclose(sp[0, :, h], _brute_masked_attention(*args, lambda i, j: c[i][0] == c[j][0],
                                                                         1 / math.sqrt(3)), rtol=1e-12, atol=1e-13)
        same_pos = lambda i, j: c[i][1:] == c[j][1:]
        np.testing.assert_allclose(te[0, :, h], _brute_masked_attention(*args, same_pos, 1 / math.sqrt(3)),
                                   rtol=1e-12, atol=1e-13)
        np.testing.assert_allclose(tc[0, :, h], _brute_masked_attention(
            *args, lambda i, j: same_pos(i, j) and c[j][0] <= c[i][0], 1 / math.sqrt(3)), rtol=1e-12, atol=1e-13)
    # causal: the first frame sees only itself -> its own value
    HW = H * W
    np.testing.assert_allclose(tc[0, :HW], v[0, :HW], atol=1e-15)


def test_factorized_special_cases():
    rng = np.random.default_rng(41)
    q, k, v = (rng.standard_normal((2, 12, 2, 4)) for _ in range(3))
    # one frame: spatial = full attention, temporal = each token alone (its own value)
    np.testing.assert_allclose(O.spatial_attn_ref(q, k, v, (1, 3, 4)), O.attn_ref(q, k, v), rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(O.temporal_attn_ref(q, k, v, (1, 3, 4)), v, atol=1e-15)
    # one position per frame: temporal = full attention, spatial = each token alone
    np.testing.assert_allclose(O.temporal_attn_ref(q, k, v, (12, 1, 1)), O.attn_ref(q, k, v), rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(O.spatial_attn_ref(q, k, v, (12, 1, 1)), v, atol=1e-15)


def test_frame_causal_limit_values():
    # text_len 3, frames of 4 tokens: text -> 3; frame 0 (tokens 3..6) -> 7; frame 1 -> 11
    assert [O.frame_causal_limit(r, 3, 4) for r in range(11)] == [3, 3, 3, 7, 7, 7, 7, 11, 11, 11, 11]
    assert [O.frame_causal_limit(r, 0, 2) for r in range(6)] == [2, 2, 4, 4, 6, 6]


def test_frame_causal_attention_brute_force():
    T, H, W, L = 3, 1, 2, 2
    N = L + T * H * W
    # block of each token written out: text 0, frame t -> t + 1
    block = [0, 0, 1, 1, 2, 2, 3, 3]
    rng = np.random.default_rng(42)
    q, k, v = (rng.standard_normal((1, N, 2, 5)) for _ in range(3))
    got = O.frame_causal_attn_ref(q, k, v, (T, H, W), L)
    for h in range(2):
        ref = _brute_masked_attention(q[0, :, h].tolist(), k[0, :, h].tolist(), v[0, :, h].tolist(),
                                      lambda i, j: block[j] <= block[i], 1 / math.sqrt(5))
        np.testing.assert_allclose(got[0, :, h], ref, rtol=1e-12, atol=1e-13)
    # the last frame sees everything: full attention there
    full = O.attn_ref(q, k, v)
    np.testing.assert_allclose(got[:, -2:], full[:, -2:], rtol=1e-13, atol=1e-14)
    # rows / heads subsets
    np.testing.assert_allclose(O.frame_causal_attn_ref(q, k, v, (T, H, W), L, rows=[7, 2, 0], heads=[1]),
                               got[:, [7, 2, 0]][:, :, [1]], rtol=0, atol=1e-15)
    # one frame, no text: plain full attention
    np.testing.assert_allclose(O.frame_causal_attn_ref(q[:, :6], k[:, :6], v[:, :6], (1, 2, 3), 0),
                               O.attn_ref(q[:, :6], k[:, :6], v[:, :6]), rtol=1e-13, atol=1e-14)


# ----------------------------------------------------------------------------------------------
# Skiparse with a joined text prefix (global text tokens)
# ----------------------------------------------------------------------------------------------

@pytest.mark.parametrize("mode", [O.SKIP_SINGLE, O.SKIP_GROUP])
def test_skiparse_text_brute_force(mode):
    L, nv, kr = 3, 8, 2
    N = L + nv
    # set of video token u (0-based among the video tokens), from the mode's definition
    set_of = (lambda u: u % kr) if mode == O.SKIP_SINGLE else (lambda u: (u // kr) % kr)

    def allowed(i, j):
        if i < L or j < L:
            return True          # text queries see all; every query sees the text
        return set_of(i - L) == set_of(j - L)

    rng = np.random.default_rng(60)
    q, k, v = (rng.standard_normal((1, N, 2, 3)) for _ in range(3))
    got = O.skiparse_text_attn_ref(q, k, v, L, kr, mode)
    for h in range(2):
        ref = _brute_masked_attention(q[0, :, h].tolist(), k[0, :, h].tolist(), v[0, :, h].tolist(), allowed,
                                      1 / math.sqrt(3))
        np.testing.assert_allclose(got[0, :, h], ref, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(O.skiparse_text_attn_ref(q, k, v, L, kr, mode, rows=[10, 1, 4], heads=[1]),
                               got[:, [10, 1, 4]][:, :, [1]], rtol=0, atol=1e-15)


def test_skiparse_text_special_cases():
    rng = np.random.default_rng(61)
    q, k, v = (rng.standard_normal((2, 16, 2, 4)) for _ in range(3))
    # no text: plain Skiparse; k = 1: full attention
    np.testing.assert_allclose(O.skiparse_text_attn_ref(q, k, v, 0, 4, O.SKIP_GROUP),
                               O.skiparse_attn_ref(q, k, v, 4, O.SKIP_GROUP), rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(O.skiparse_text_attn_ref(q, k, v, 5, 1, O.SKIP_SINGLE), O.attn_ref(q, k, v),
                               rtol=1e-13, atol=1e-14)


# ----------------------------------------------------------------------------------------------
# backward pass: central finite differences of a scalar loss through the forward oracle
# ----------------------------------------------------------------------------------------------

def _fd_grad(f, x, eps=1e-6):
    g = np.zeros_like(x)
    it = np.nditer(x, flags=["multi_index"])
    for _ in it:
        i = it.multi_index
        xp, xm = x.copy(), x.copy()
        xp[i] += eps
        xm[i] -= eps
        g[i] = (f(xp) - f(xm)) / (2 * eps)
    return g


def test_dense_backward_matches_finite_differences():
    rng = np.random.default_rng(80)
    q, k, v = (rng.standard_normal((1, 5, 2, 3)) for _ in range(3))
    G = rng.standard_normal((1, 5, 2, 3))           # loss = sum(O * G), so dO = G
    loss = lambda q_, k_, v_: float((O.attn_ref(q_, k_, v_, scale=0.7) * G).sum())
    dq, dk, dv = O.attn_backward_ref(q, k, v, G, scale=0.7)
    np.testing.assert_allclose(dq, _fd_grad(lambda x: loss(x, k, v), q), rtol=1e-6, atol=1e-8)
    np.testing.assert_allclose(dk, _fd_grad(lambda x: loss(q, x, v), k), rtol=1e-6, atol=1e-8)
    np.testing.assert_allclose(dv, _fd_grad(lambda x: loss(q, k, x), v), rtol=1e-6, atol=1e-8)


@pytest.mark.parametrize("mode", [O.SKIP_SINGLE, O.SKIP_GROUP])
def test_skiparse_backward_matches_finite_differences(mode):
    rng = np.random.default_rng(81)
    q, k, v = (rng.standard_normal((1, 8, 1, 3)) for _ in range(3))
    G = rng.standard_normal((1, 8, 1, 3))
    loss = lambda q_, k_, v_: float((O.skiparse_attn_ref(q_, k_, v_, 2, mode) * G).sum())
    dq, dk, dv = O.skiparse_backward_ref(q, k, v, G, 2, mode)
    np.testing.assert_allclose(dq, _fd_grad(lambda x: loss(x, k, v), q), rtol=1e-6, atol=1e-8)
    np.testing.assert_allclose(dk, _fd_grad(lambda x: loss(q, x, v), k), rtol=1e-6, atol=1e-8)
    np.testing.assert_allclose(dv, _fd_grad(lambda x: loss(q, k, x), v), rtol=1e-6, atol=1e-8)


def test_backward_closed_forms_and_lse():
    rng = np.random.default_rng(82)
    q, k, v = (rng.standard_normal((4, 3)) for _ in range(3))
    # dO = 0: every gradient vanishes; equal keys: dQ = 0 (softmax is flat in q)
    dq, dk, dv = O.attention_head_backward_ref(q, k, v, np.zeros((4, 3)), 0.5)
    assert not dq.any() and not dk.any() and not dv.any()
    kk = np.tile(k[:1], (4, 1))
    dq, _, dv = O.attention_head_backward_ref(q, kk, v, rng.standard_normal((4, 3)), 0.5)
    np.testing.assert_allclose(dq, 0, atol=1e-14)
    # dV = P^T dO with uniform P = 1/4 when all keys are equal
    do = rng.standard_normal((4, 3))
    _, _, dv = O.attention_head_backward_ref(q, kk, v, do, 0.5)
    np.testing.assert_allclose(dv, np.tile(do.sum(0) / 4, (4, 1)), rtol=1e-13)
    # lse: two keys with scores 0 and ln 3 -> ln 4
    lse = O.attention_head_lse_ref(np.array([[1.0, 0.0]]), np.array([[0.0, 0.0], [math.log(3.0), 0.0]]), 1.0)
    np.testing.assert_allclose(lse, [math.log(4.0)], rtol=1e-15)


def test_backward_rows_agree_with_full_backward():
    # the sampled-row form is the same chain rule evaluated row by row (pinned above by finite
    # differences through the full form)
    rng = np.random.default_rng(83)
    q, k, v, do = (rng.standard_normal((40, 8)) for _ in range(4))
    dq, dk, dv = O.attention_head_backward_ref(q, k, v, do, 0.3)
    rq, rk = [0, 7, 39], [3, 4, 38]
    sq, sk, sv = O.attention_head_backward_rows_ref(q, k, v, do, 0.3, rq, rk, chunk=16)
    np.testing.assert_allclose(sq, dq[rq], rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(sk, dk[rk], rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(sv, dv[rk], rtol=1e-12, atol=1e-13)


def test_frame_causal_backward_matches_finite_differences():
    rng = np.random.default_rng(84)
    grid, L = (3, 1, 2), 1                       # 7 tokens: text, then three frames of two
    q, k, v = (rng.standard_normal((1, 7, 1, 3)) for _ in range(3))
    G = rng.standard_normal((1, 7, 1, 3))
    loss = lambda q_, k_, v_: float((O.frame_causal_attn_ref(q_, k_, v_, grid, L) * G).sum())
    dq, dk, dv = O.frame_causal_backward_ref(q, k, v, G, grid, L)
    np.testing.assert_allclose(dq, _fd_grad(lambda x: loss(x, k, v), q), rtol=1e-6, atol=1e-8)
    np.testing.assert_allclose(dk, _fd_grad(lambda x: loss(q, x, v), k), rtol=1e-6, atol=1e-8)
    np.testing.assert_allclose(dv, _fd_grad(lambda x: loss(q, k, x), v), rtol=1e-6, atol=1e-8)
    # keys of the last frame are seen only by the last frame's queries: their dV is P^T dO of those
    assert not np.allclose(dv[0, 5:], 0)


def test_spatial_backward_matches_finite_differences_and_reduces_to_dense():
    rng = np.random.default_rng(85)
    grid = (2, 1, 3)                             # two frames of three tokens
    q, k, v = (rng.standard_normal((1, 6, 2, 3)) for _ in range(3))
    G = rng.standard_normal((1, 6, 2, 3))
    loss = lambda q_, k_, v_: float((O.spatial_attn_ref(q_, k_, v_, grid, scale=0.6) * G).sum())
    dq, dk, dv = O.spatial_backward_ref(q, k, v, G, grid, scale=0.6)
    np.testing.assert_allclose(dq, _fd_grad(lambda x: loss(x, k, v), q), rtol=1e-6, atol=1e-8)
    np.testing.assert_allclose(dk, _fd_grad(lambda x: loss(q, x, v), k), rtol=1e-6, atol=1e-8)
    np.testing.assert_allclose(dv, _fd_grad(lambda x: loss(q, k, x), v), rtol=1e-6, atol=1e-8)
    # one frame: spatial attention is full attention over the frame
    for a, b in zip(O.spatial_backward_ref(q, k, v, G, (1, 2, 3), scale=0.6),
                    O.attn_backward_ref(q, k, v, G, scale=0.6)):
        np.testing.assert_allclose(a, b, rtol=1e-12, atol=1e-13)


@pytest.mark.parametrize("causal", [False, True])
def test_temporal_backward_matches_finite_differences(causal):
    rng = np.random.default_rng(86 + causal)
    grid = (3, 1, 2)                             # three frames, two positions
    q, k, v = (rng.standard_normal((1, 6, 1, 3)) for _ in range(3))
    G = rng.standard_normal((1, 6, 1, 3))
    loss = lambda q_, k_, v_: float((O.temporal_attn_ref(q_, k_, v_, grid, causal=causal) * G).sum())
    dq, dk, dv = O.temporal_backward_ref(q, k, v, G, grid, causal=causal)
    np.testing.assert_allclose(dq, _fd_grad(lambda x: loss(x, k, v), q), rtol=1e-6, atol=1e-8)
    np.testing.assert_allclose(dk, _fd_grad(lambda x: loss(q, x, v), k), rtol=1e-6, atol=1e-8)
    np.testing.assert_allclose(dv, _fd_grad(lambda x: loss(q, k, x), v), rtol=1e-6, atol=1e-8)
    if causal:   # a first-frame query sees its own key only: softmax over one key, dQ = 0
        np.testing.assert_allclose(dq[0, :2], 0, atol=1e-14)
        assert np.abs(dq[0, 2:]).max() > 1e-3


def test_temporal_backward_special_cases():
    rng = np.random.default_rng(88)
    q, k, v, G = (rng.standard_normal((2, 5, 2, 4)) for _ in range(4))
    # one position: attention over the T tokens (full), frame-causal with one-token frames (causal)
    for a, b in zip(O.temporal_backward_ref(q, k, v, G, (5, 1, 1)), O.attn_backward_ref(q, k, v, G)):
        np.testing.assert_allclose(a, b, rtol=1e-12, atol=1e-13)
    for a, b in zip(O.temporal_backward_ref(q, k, v, G, (5, 1, 1), causal=True),
                    O.frame_causal_backward_ref(q, k, v, G, (5, 1, 1), 0)):
        np.testing.assert_allclose(a, b, rtol=1e-12, atol=1e-13)
    # a position's tokens t*H*W + pos are the Single Skip set pos with k = H*W
    q, k, v, G = (rng.standard_normal((1, 12, 1, 4)) for _ in range(4))
    for a, b in zip(O.temporal_backward_ref(q, k, v, G, (3, 2, 2)),
                    O.skiparse_backward_ref(q, k, v, G, 4, O.SKIP_SINGLE)):
        np.testing.assert_allclose(a, b, rtol=1e-12, atol=1e-13)


def test_packed_backward_matches_finite_differences_and_reduces_to_dense():
    # three samples of 4, 0 and 1 tokens, then 3: the empty and one-token samples included
    rng = np.random.default_rng(83)
    bounds = [0, 4, 4, 5, 8]
    q, k, v = (rng.standard_normal((1, 8, 2, 3)) for _ in range(3))
    G = rng.standard_normal((1, 8, 2, 3))
    loss = lambda q_, k_, v_: float((O.packed_attn_ref(q_, k_, v_, bounds, scale=0.6) * G).sum())
    dq, dk, dv = O.packed_backward_ref(q, k, v, G, bounds, scale=0.6)
    np.testing.assert_allclose(dq, _fd_grad(lambda x: loss(x, k, v), q), rtol=1e-6, atol=1e-8)
    np.testing.assert_allclose(dk, _fd_grad(lambda x: loss(q, x, v), k), rtol=1e-6, atol=1e-8)
    np.testing.assert_allclose(dv, _fd_grad(lambda x: loss(q, k, x), v), rtol=1e-6, atol=1e-8)
    # a one-token sample sees only itself (P = 1): its dq and dk vanish, its dv is its dO
    assert np.abs(dq[0, 4]).max() <= 1e-15 and np.abs(dk[0, 4]).max() <= 1e-15   # zero up to fp64 rounding
    np.testing.assert_array_equal(dv[0, 4], G[0, 4])
    # one sample spanning the batch is the dense backward
    one = O.packed_backward_ref(q, k, v, G, [0, 8], scale=0.6)
    dense = O.attn_backward_ref(q, k, v, G, scale=0.6)
    for a, b in zip(one, dense):
        np.testing.assert_allclose(a, b, rtol=1e-13, atol=1e-14)


@pytest.mark.parametrize("mode", [O.SKIP_SINGLE, O.SKIP_GROUP])
def test_skiparse_text_backward_matches_finite_differences(mode):
    # 3 text tokens + 8 video tokens in k = 2 sets
    rng = np.random.default_rng(84 + mode)
    q, k, v = (rng.standard_normal((1, 11, 2, 3)) for _ in range(3))
    G = rng.standard_normal((1, 11, 2, 3))
    loss = lambda q_, k_, v_: float((O.skiparse_text_attn_ref(q_, k_, v_, 3, 2, mode, scale=0.8) * G).sum())
    dq, dk, dv = O.skiparse_text_backward_ref(q, k, v, G, 3, 2, mode, scale=0.8)
    np.testing.assert_allclose(dq, _fd_grad(lambda x: loss(x, k, v), q), rtol=1e-6, atol=1e-8)
    np.testing.assert_allclose(dk, _fd_grad(lambda x: loss(q, x, v), k), rtol=1e-6, atol=1e-8)
    np.testing.assert_allclose(dv, _fd_grad(lambda x: loss(q, k, x), v), rtol=1e-6, atol=1e-8)


def test_skiparse_text_backward_reduces_to_skiparse_and_dense():
    rng = np.random.default_rng(86)
    q, k, v, G = (rng.standard_normal((2, 12, 2, 3)) for _ in range(4))
    # no text: the Skiparse backward
    for a, b in zip(O.skiparse_text_backward_ref(q, k, v, G, 0, 3, O.SKIP_SINGLE),
                    O.skiparse_backward_ref(q, k, v, G, 3, O.SKIP_SINGLE)):
        np.testing.assert_allclose(a, b, rtol=1e-12, atol=1e-13)
    # one set: every token sees every token, the dense backward
    for a, b in zip(O.skiparse_text_backward_ref(q, k, v, G, 4, 1, O.SKIP_GROUP), O.attn_backward_ref(q, k, v, G)):
        np.testing.assert_allclose(a, b, rtol=1e-12, atol=1e-13)


@pytest.mark.parametrize("text_len,text_rows", [(0, False), (3, True), (3, False)])
def test_skiparse_text_backward_rows_match_finite_differences(text_len, text_rows):
    # 3 (or no) text tokens + 12 video tokens in k = 2 Group Skip sets (groups of 2), B = 2; the
    # selected rows are text and video tokens of both sets, or video tokens of one set only (the
    # other set's row statistics are then not computed)
    rng = np.random.default_rng(87 + text_len)
    N = text_len + 12
    q, k, v = (rng.standard_normal((2, N, 3, 4)) for _ in range(3))
    G = rng.standard_normal((2, N, 3, 4))
    rows = sorted({0, 1, N - 1, text_len, text_len + 3}) if text_rows or not text_len else \
        [text_len, text_len + 1, text_len + 4, text_len + 9]
    heads = [0, 2]
    loss = lambda q_, k_, v_: float((O.skiparse_text_attn_ref(q_, k_, v_, text_len, 2, O.SKIP_GROUP, scale=0.7)
                                     * G).sum())
    dq, dk, dv = O.skiparse_text_backward_rows_ref(q, k, v, G, text_len, 2, O.SKIP_GROUP, rows, rows, heads=heads,
                                                   scale=0.7, chunk=5)
    fq = _fd_grad(lambda x: loss(x, k, v), q)
    fk = _fd_grad(lambda x: loss(q, x, v), k)
    fv = _fd_grad(lambda x: loss(q, k, x), v)
    sel = np.ix_(range(2), rows, heads, range(4))
    np.testing.assert_allclose(dq, fq[sel], rtol=1e-6, atol=1e-8)
    np.testing.assert_allclose(dk, fk[sel], rtol=1e-6, atol=1e-8)
    np.testing.assert_allclose(dv, fv[sel], rtol=1e-6, atol=1e-8)


def test_frame_causal_backward_rows_match_finite_differences():
    # 2 text tokens + 3 frames of 2 x 2, B = 2; selected rows: text, first and last frame
    rng = np.random.default_rng(91)
    grid, L = (3, 2, 2), 2
    N = L + 12
    q, k, v = (rng.standard_normal((2, N, 3, 4)) for _ in range(3))
    G = rng.standard_normal((2, N, 3, 4))
    rows = [0, 1, 2, 5, 9, 13]
    heads = [1, 2]
    loss = lambda q_, k_, v_: float((O.frame_causal_attn_ref(q_, k_, v_, grid, L, scale=0.6) * G).sum())
    dq, dk, dv = O.frame_causal_backward_rows_ref(q, k, v, G, grid, L, rows, rows, heads=heads, scale=0.6, chunk=3)
    sel = np.ix_(range(2), rows, heads, range(4))
    np.testing.assert_allclose(dq, _fd_grad(lambda x: loss(x, k, v), q)[sel], rtol=1e-6, atol=1e-8)
    np.testing.assert_allclose(dk, _fd_grad(lambda x: loss(q, x, v), k)[sel], rtol=1e-6, atol=1e-8)
    np.testing.assert_allclose(dv, _fd_grad(lambda x: loss(q, k, x), v)[sel], rtol=1e-6, atol=1e-8)
