"""GPU parity of 3D RoPE, the Skiparse index map and the k-fold gather / scatter.

Index maps and pure copies: bit-exact.  RoPE outputs: the kernel rotates in fp64 and rounds
once to bf16, so it is compared with the fp64 oracle correctly rounded to bf16: at most 1 ulp
apart anywhere (fp64 cos/sin of the two sides may differ in the last bits, which can flip a
rounding that sits on a tie boundary) and identical in all but a 1e-4 fraction of elements."""

import numpy as np
import pytest
import torch

import oracle as O
from spacetime_attention_b200 import ops, synthetic as syn
from tests.gpu_common import gpu  # noqa: F401
from tests.helpers import assert_bf16_close, bf16_round, to_f64

pytestmark = pytest.mark.gpu

ROPE_CASES = [
    # name, B, heads, d, grid, text_len, split
    ("tiny", 1, 2, 64, (4, 8, 8), 0, (16, 24, 24)),
    ("ragged_text", 2, 3, 64, (3, 5, 7), 7, (16, 24, 24)),
    ("d96", 1, 5, 96, (5, 6, 7), 0, (32, 32, 32)),
    ("d128_text", 1, 4, 128, (2, 9, 11), 13, (32, 48, 48)),
    ("uneven_split", 1, 2, 64, (6, 5, 4), 3, (20, 22, 22)),
    ("one_token", 1, 1, 64, (1, 1, 1), 0, (16, 24, 24)),
    ("text_heavy", 1, 2, 64, (1, 2, 2), 300, (16, 24, 24)),
]


def _rope_case(dev, B, heads, d, grid, L, split, seed=7, inplace=False):
    w = syn.custom("c", B, heads, d, grid, L, split)
    q, k, _ = syn.make_qkv(w, seed)
    qg, kg = q.to(dev), k.to(dev)
    if inplace:
        qo, ko = ops.rope3d(qg, kg, grid, L, split, q_out=qg, k_out=kg)
    else:
        qo, ko = ops.rope3d(qg, kg, grid, L, split)
    torch.cuda.synchronize()
    for x, xo in ((q, qo), (k, ko)):
        ref = bf16_round(O.rope3d_ref(to_f64(x), grid, L, split))
        assert_bf16_close(xo, ref, "rope3d")
        # text tokens are bit-exact copies
        assert torch.equal(xo[:, :L].cpu(), x[:, :L])


@pytest.mark.parametrize("case", ROPE_CASES, ids=[c[0] for c in ROPE_CASES])
def test_rope3d_matches_oracle(gpu, case):
    _, B, heads, d, grid, L, split = case
    _rope_case(gpu, B, heads, d, grid, L, split)


def test_rope3d_in_place(gpu):
    _rope_case(gpu, 2, 3, 64, (3, 5, 7), 7, (16, 24, 24), inplace=True)


@pytest.mark.parametrize("name", ["cogvideox_2b", "open_sora_plan", "long_video"])
def test_rope3d_full_size(gpu, name):
    w = syn.WORKLOADS[name]
    q, k, _ = syn.make_qkv(w)
    qo, ko = ops.rope3d(q.to(gpu), k.to(gpu), w.grid, w.text_len, w.split)
    torch.cuda.synchronize()
    # every token of a spread of heads (the oracle is vectorised over tokens)
    heads = sorted({0, w.heads // 2, w.heads - 1})
    for x, xo in ((q, qo), (k, ko)):
        ref = bf16_round(O.rope3d_ref(to_f64(x[:, :, heads]), w.grid, w.text_len, w.split))
        assert_bf16_close(xo[:, :, heads], ref, name)


@pytest.mark.parametrize("n,k,mode", [(256, 2, 0), (256, 2, 1), (28800, 4, 0), (28800, 4, 1), (36864, 4, 0),
                                      (36864, 4, 1), (17550, 3, 0), (18, 3, 1), (7, 1, 0), (64, 8, 1)])
def test_index_map_bit_exact(gpu, n, k, mode):
    got = ops.skiparse_index_map(n, k, mode, device=gpu).cpu().numpy()
    assert np.array_equal(got, O.skiparse_index_map(n, k, mode))


GATHER_CASES = [
    ("tiny_k2", 1, 2, 64, (4, 8, 8), 2),
    ("ragged_k3", 2, 3, 64, (3, 6, 3), 3),
    ("d96_k4", 1, 2, 96, (4, 4, 8), 4),
    ("d128_k2", 2, 2, 128, (2, 4, 6), 2),
]


@pytest.mark.parametrize("case", GATHER_CASES, ids=[c[0] for c in GATHER_CASES])
@pytest.mark.parametrize("mode", [0, 1])
def test_gather_scatter(gpu, case, mode):
    _, B, heads, d, grid, k = case
    split = {64: (16, 24, 24), 96: (32, 32, 32), 128: (32, 48, 48)}[d]
    w = syn.custom("g", B, heads, d, grid, 0, split)
    q, kk, v = syn.make_qkv(w, 11)
    qg, kg, vg = q.to(gpu), kk.to(gpu), v.to(gpu)
    # without RoPE: exact permutation of all three
    qo, ko, vo = ops.skiparse_gather(qg, kg, vg, grid, k, mode)
    for x, xo in ((q, qo), (kk, ko), (v, vo)):
        ref = O.skiparse_gather_ref(to_f64(x), k, mode)
        assert np.array_equal(to_f64(xo), ref)
    # scatter inverts it bit-exactly
    assert torch.equal(ops.skiparse_scatter(vo, grid, k, mode), vg)
    # with RoPE on q, k (positions of the source tokens), v copied exactly
    qr, kr, vr = ops.skiparse_gather(qg, kg, vg, grid, k, mode, split=split)
    torch.cuda.synchronize()
    assert torch.equal(vr, vo)
    for x, xr in ((q, qr), (kk, kr)):
        ref = bf16_round(O.skiparse_gather_ref(O.rope3d_ref(to_f64(x), grid, 0, split), k, mode))
        assert_bf16_close(xr, ref, "gather+rope")
    # q only
    q_only, none_k, none_v = ops.skiparse_gather(qg, None, None, grid, k, mode, split=split)
    assert none_k is None and none_v is None and torch.equal(q_only, qr)


def test_gather_full_size_open_sora_plan(gpu):
    w = syn.WORKLOADS["open_sora_plan"]
    q, k, v = syn.make_qkv(w)
    for mode in (0, 1):
        qo, ko, vo = ops.skiparse_gather(q.to(gpu), k.to(gpu), v.to(gpu), w.grid, 4, mode, split=w.split)
        torch.cuda.synchronize()
        ref_v = O.skiparse_gather_ref(to_f64(v[:, :, :2]), 4, mode)
        assert np.array_equal(to_f64(vo[:, :, :2]), ref_v)
        ref_q = bf16_round(O.skiparse_gather_ref(O.rope3d_ref(to_f64(q[:, :, :2]), w.grid, 0, w.split), 4, mode))
        assert_bf16_close(qo[:, :, :2], ref_q, "gather+rope full size")
        assert torch.equal(ops.skiparse_scatter(vo, w.grid, 4, mode).cpu(), v)
