"""Plain fp64 CPU oracle for spacetime attention (3D RoPE, 3D full attention, Skiparse).

TEST INFRASTRUCTURE ONLY.  Only the test suite, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this module.  It shares
no code with the CUDA library and never calls it; the library never calls this module.

Everything here is the written-out definition of what the method computes, in float64,
starting from the exact values of the (bf16) inputs.  Library primitives (a matmul, exp) are
used as single steps; there is no blocking, fusion or reordering beyond splitting query rows
into chunks to bound memory, which does not change any value.

Sources (page title, section):
  * "CogVideoX: Text-to-Video Diffusion Models with an Expert Transformer", section 2
    (latents are patchified and unfolded into one sequence; text embeddings are concatenated
    with it along the sequence axis), section 2.2 "Patchify" (sequence length), "3D-RoPE"
    (independent 1D RoPE per coordinate axis over channel shares, concatenated along the
    channel axis), "3D Full Attention"; section 3.1 and the appendix on RoPE interpolation
    (positions are raw indices, extrapolated, never rescaled).
  * "Open Video Models", The Breakthrough (HunyuanVideo's 3D RoPE: separate rotation
    frequencies along time, height and width).
  * RoFormer (reference [14] of the CogVideoX paper): rotation of channel pairs by
    position times a geometric frequency series with base 10000.
  * "Open-Sora Plan: Open-Source Large Video Generation Model", section 2.2.2 "Skiparse
    Attention" (sequence cut to 1/k with the batch grown k-fold; Single Skip; Group Skip
    groups adjacent tokens and connects groups that are k-1 groups apart; THW mod k = 0).
  * "Attention is all you need" (reference [1]): softmax(q k^T / sqrt(d)) v.

Readings where the pages are silent (each also listed in the design notes):
  * flattening order of the (t, h, w) grid is row-major, w fastest; text tokens come first;
  * channel chunks are ordered t, h, w; pairs inside a chunk are interleaved (2j, 2j+1);
    the frequency of pair j in a chunk of size d_a is theta^(-2j/d_a);
  * text tokens are not rotated;
  * Single Skip set g = tokens {s*k + g}; Group Skip uses groups of k adjacent tokens and
    set g = groups whose index is congruent to g mod k, i.e. slot s = o*k + r maps to token
    o*k*k + g*k + r; each set lists its tokens in ascending order;
  * the k-fold batch produced by the gather is ordered b*k + g (b outer);
  * softmax scale 1/sqrt(head_dim) unless given.

Parity is pinned for every function here by ``tests/test_oracle_pins.py``.  Match to any
trained checkpoint is "parity unpinned": no weights or code exist to compare against, and the
pages do not fix the pairing convention of RoPE channels.
"""

from __future__ import annotations

import math
from typing import Sequence

import numpy as np

SKIP_SINGLE = 0
SKIP_GROUP = 1


# ----------------------------------------------------------------------------------------------
# Storage precision
# ----------------------------------------------------------------------------------------------

def round_to_bf16(x: np.ndarray) -> np.ndarray:
    """Round fp64 values to the nearest bf16 value, ties to even, returned as fp64.

    bf16 is the storage format of every tensor at the library's boundary (the pages run their
    models in bf16, CogVideoX Tables 7 and 8), so a RoPE output that feeds attention is rounded
    to bf16 once.  Done in two exact steps: fp64 -> fp32 rounded to odd (truncate toward zero,
    then set the lowest bit when anything was dropped), then fp32 -> bf16 to nearest even on the
    bit pattern.  fp32 keeps 16 more significand bits than bf16, so the result is the single
    correct rounding of x.  Finite inputs only.
    """
    x = np.ascontiguousarray(x, dtype=np.float64)
    f = x.astype(np.float32)
    over = np.abs(f.astype(np.float64)) > np.abs(x)
    f = np.where(over, np.nextafter(f, np.float32(0)), f).astype(np.float32)
    bits = f.view(np.uint32) | (f.astype(np.float64) != x).astype(np.uint32)
    lsb = (bits >> np.uint32(16)) & np.uint32(1)
    rounded = ((bits + np.uint32(0x7FFF) + lsb) >> np.uint32(16)) << np.uint32(16)
    return rounded.astype(np.uint32).view(np.float32).astype(np.float64)


# ----------------------------------------------------------------------------------------------
# Token positions
# ----------------------------------------------------------------------------------------------

def video_positions(T: int, H: int, W: int):
    """(t, h, w) integer coordinates of every video token, in sequence order.

    The latent grid T x H x W is unfolded into one sequence (CogVideoX section 2 and 2.2
    "Patchify"); reading: row-major, w fastest.  Token v has t = v div (H W),
    h = (v div W) mod H, w = v mod W.  Positions start at 0 and are not rescaled
    (CogVideoX section 3.1: extrapolation, not interpolation).
    """
    n = T * H * W
    v = np.arange(n, dtype=np.int64)
    t = v // (H * W)
    h = (v // W) % H
    w = v % W
    return t, h, w


# ----------------------------------------------------------------------------------------------
# 3D RoPE
# ----------------------------------------------------------------------------------------------

def rope_frequencies(d_axis: int, theta: float = 10000.0) -> np.ndarray:
    """Frequencies of one axis's 1D RoPE: omega_j = theta^(-2j/d_axis), j < d_axis/2.

    RoFormer's geometric series, applied per axis with the axis's own channel count
    ("Open Video Models": separate rotation frequencies along time, height and width).
    """
    if d_axis % 2:
        raise ValueError("each RoPE channel chunk must be even")
    j = np.arange(d_axis // 2, dtype=np.float64)
    return np.power(float(theta), -2.0 * j / float(d_axis))


def rope_rotate_chunk(x: np.ndarray, pos: np.ndarray, d_axis: int, theta: float) -> np.ndarray:
    """1D RoPE on one channel chunk.

    x: [..., n_tok, n_heads, d_axis] float64, pos: [n_tok] integer positions.
    Pair j = channels (2j, 2j+1) is rotated by angle pos * omega_j:
        x' = x cos(a) - y sin(a),  y' = x sin(a) + y cos(a).
    """
    omega = rope_frequencies(d_axis, theta)                      # [d_axis/2]
    ang = pos.astype(np.float64)[:, None] * omega[None, :]       # [n_tok, d_axis/2]
    c = np.cos(ang)[:, None, :]                                  # broadcast over heads
    s = np.sin(ang)[:, None, :]
    xe = x[..., 0::2]
    xo = x[..., 1::2]
    out = np.empty_like(x)
    out[..., 0::2] = xe * c - xo * s
    out[..., 1::2] = xe * s + xo * c
    return out


def rope3d_positions_ref(x: np.ndarray, pos_t, pos_h, pos_w, split: Sequence[int],
                         theta: float = 10000.0) -> np.ndarray:
    """3D RoPE of video tokens with explicit positions.

    x: [B, n_tok, n_heads, d] (values of the bf16 inputs); pos_*: [n_tok] integers.
    CogVideoX section 2.2 "3D-RoPE": an independent 1D RoPE per coordinate axis, each on its
    own share of the channels, the results concatenated along the channel axis.  Reading:
    chunk order t, h, w with sizes split = (d_t, d_h, d_w).
    """
    x = np.asarray(x, dtype=np.float64)
    d_t, d_h, d_w = (int(a) for a in split)
    if d_t + d_h + d_w != x.shape[-1]:
        raise ValueError("RoPE split must sum to head_dim")
    out = np.empty_like(x)
    out[..., 0:d_t] = rope_rotate_chunk(x[..., 0:d_t], np.asarray(pos_t), d_t, theta)
    out[..., d_t:d_t + d_h] = rope_rotate_chunk(x[..., d_t:d_t + d_h], np.asarray(pos_h), d_h, theta)
    out[..., d_t + d_h:] = rope_rotate_chunk(x[..., d_t + d_h:], np.asarray(pos_w), d_w, theta)
    return out


def rope3d_ref(x: np.ndarray, grid: Sequence[int], text_len: int, split: Sequence[int],
               theta: float = 10000.0) -> np.ndarray:
    """3D RoPE over a [B, text_len + T*H*W, n_heads, d] sequence.

    Text tokens (the first text_len; CogVideoX section 2 concatenates text before video) are
    left unrotated (reading: the pages give text no spatio-temporal position); video tokens
    are rotated by their (t, h, w) grid coordinates.
    """
    T, H, W = (int(a) for a in grid)
    x = np.asarray(x, dtype=np.float64)
    if x.shape[1] != text_len + T * H * W:
        raise ValueError("sequence length does not match text_len + T*H*W")
    out = x.copy()
    t, h, w = video_positions(T, H, W)
    out[:, text_len:] = rope3d_positions_ref(x[:, text_len:], t, h, w, split, theta)
    return out


# ----------------------------------------------------------------------------------------------
# Skiparse index maps
# ----------------------------------------------------------------------------------------------

def skiparse_sets(n_video: int, k: int, mode: int) -> list[list[int]]:
    """The k token sets of Skiparse attention, each as an explicit ascending list.

    Open-Sora Plan section 2.2.2: the sequence is cut to 1/k of its length and the batch
    grown k-fold.  Single Skip: set g holds every k-th token starting at g.  Group Skip:
    adjacent tokens form groups (of k tokens, reading) and a set joins groups that are
    k-1 groups apart, i.e. the groups whose index is congruent to g mod k.
    """
    if k < 1:
        raise ValueError("k must be >= 1")
    if mode == SKIP_SINGLE:
        if n_video % k:
            raise ValueError("Single Skip needs n_video mod k == 0")
        return [[s * k + g for s in range(n_video // k)] for g in range(k)]
    if mode == SKIP_GROUP:
        if n_video % (k * k):
            raise ValueError("Group Skip needs n_video mod k^2 == 0")
        n_groups = n_video // k
        sets = []
        for g in range(k):
            members = []
            for group in range(n_groups):
                if group % k == g:
                    members.extend(range(group * k, group * k + k))
            sets.append(members)
        return sets
    raise ValueError("mode must be SKIP_SINGLE or SKIP_GROUP")


def skiparse_index_map(n_video: int, k: int, mode: int) -> np.ndarray:
    """Concatenation of the k sets: entry g*(n_video/k) + s is the token at slot s of set g."""
    return np.asarray([tok for st in skiparse_sets(n_video, k, mode) for tok in st], dtype=np.int32)


# ----------------------------------------------------------------------------------------------
# Gather / scatter (the k-fold batch)
# ----------------------------------------------------------------------------------------------

def skiparse_gather_ref(x: np.ndarray, k: int, mode: int) -> np.ndarray:
    """[B, N, n_h, d] -> [B*k, N/k, n_h, d]: out[b*k + g, s] = x[b, set_g[s]]."""
    B, N = x.shape[0], x.shape[1]
    sets = skiparse_sets(N, k, mode)
    out = np.empty((B * k, N // k) + tuple(x.shape[2:]), dtype=x.dtype)
    for b in range(B):
        for g in range(k):
            out[b * k + g] = x[b, sets[g]]
    return out


def skiparse_scatter_ref(y: np.ndarray, k: int, mode: int) -> np.ndarray:
    """Inverse of the gather: out[b, set_g[s]] = y[b*k + g, s]."""
    Bk, n_set = y.shape[0], y.shape[1]
    B, N = Bk // k, n_set * k
    sets = skiparse_sets(N, k, mode)
    out = np.empty((B, N) + tuple(y.shape[2:]), dtype=y.dtype)
    for b in range(B):
        for g in range(k):
            out[b, sets[g]] = y[b * k + g]
    return out


# ----------------------------------------------------------------------------------------------
# Attention
# ----------------------------------------------------------------------------------------------

def softmax_rows(s: np.ndarray) -> np.ndarray:
    """Row softmax p_ij = exp(s_ij - max_j s_ij) / sum_j exp(s_ij - max_j s_ij)."""
    m = np.max(s, axis=-1, keepdims=True)
    e = np.exp(s - m)
    return e / np.sum(e, axis=-1, keepdims=True)


def attention_head_ref(q: np.ndarray, k: np.ndarray, v: np.ndarray, scale: float,
                       rows=None, chunk: int = 1024) -> np.ndarray:
    """Exact attention for one head: o_i = sum_j softmax_j(q_i . k_j * scale) v_j.

    q: [n_q, d], k: [n_kv, d], v: [n_kv, d] float64.  ``rows`` optionally selects query rows
    (the result then has len(rows) rows).  Query rows are processed ``chunk`` at a time.
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    if rows is not None:
        q = q[np.asarray(rows)]
    out = np.empty((q.shape[0], v.shape[1]), dtype=np.float64)
    for r0 in range(0, q.shape[0], chunk):
        s = (q[r0:r0 + chunk] @ k.T) * scale
        out[r0:r0 + chunk] = softmax_rows(s) @ v
    return out


def default_scale(d: int) -> float:
    return 1.0 / math.sqrt(d)


def attn_ref(q: np.ndarray, k: np.ndarray, v: np.ndarray, scale: float | None = None,
             rows=None, heads=None) -> np.ndarray:
    """3D full attention (CogVideoX "3D Full Attention"): every token of a sample attends to
    every token of the same sample (text and video), bidirectionally, per head.

    q, k, v: [B, N, n_h, d].  Returns [B, N, n_h, d] float64, or, with ``rows`` (query token
    indices) and/or ``heads``, only those rows/heads: [B, len(rows), len(heads), d].
    """
    B, N, nh, d = q.shape
    scale = default_scale(d) if scale is None else scale
    rows_ = np.arange(N) if rows is None else np.asarray(rows)
    heads_ = np.arange(nh) if heads is None else np.asarray(heads)
    out = np.empty((B, len(rows_), len(heads_), d), dtype=np.float64)
    for b in range(B):
        for hi, h in enumerate(heads_):
            out[b, :, hi] = attention_head_ref(q[b, :, h], k[b, :, h], v[b, :, h], scale, rows_)
    return out


def cross_attn_ref(q: np.ndarray, k: np.ndarray, v: np.ndarray, scale: float | None = None,
                   rows=None, heads=None) -> np.ndarray:
    """Video -> text cross-attention ("Open-Sora Plan" section 2.2.1: each block attends from the
    video tokens to the text embeddings): o_i = softmax_j(q_i . k_j * scale) v_j with queries from
    the video sequence and keys/values from the text sequence, per sample and head.

    q: [B, N_q, n_h, d]; k, v: [B, N_kv, n_h, d] (N_q and N_kv independent).  ``rows`` optionally
    selects query tokens; the result is [B, len(rows), len(heads), d].
    """
    B, Nq, nh, d = q.shape
    scale = default_scale(d) if scale is None else scale
    rows_ = np.arange(Nq) if rows is None else np.asarray(rows)
    heads_ = np.arange(nh) if heads is None else np.asarray(heads)
    out = np.empty((B, len(rows_), len(heads_), d), dtype=np.float64)
    for b in range(B):
        for hi, h in enumerate(heads_):
            out[b, :, hi] = attention_head_ref(q[b, :, h], k[b, :, h], v[b, :, h], scale, rows_)
    return out


def skiparse_attn_ref(q: np.ndarray, k: np.ndarray, v: np.ndarray, k_ratio: int, mode: int,
                      scale: float | None = None, rows=None, heads=None) -> np.ndarray:
    """Skiparse attention: each token attends only to the tokens of its own set
    (Open-Sora Plan section 2.2.2), output in natural token order.

    q, k, v: [B, N, n_h, d] with no text tokens.  ``rows`` optionally restricts the query
    tokens computed (natural indices); the result is then [B, len(rows), len(heads), d].
    """
    B, N, nh, d = q.shape
    scale = default_scale(d) if scale is None else scale
    sets = skiparse_sets(N, k_ratio, mode)
    set_of = np.empty(N, dtype=np.int64)
    slot_of = np.empty(N, dtype=np.int64)
    for g, st in enumerate(sets):
        set_of[st] = g
        slot_of[st] = np.arange(len(st))
    rows_ = np.arange(N) if rows is None else np.asarray(rows)
    heads_ = np.arange(nh) if heads is None else np.asarray(heads)
    out = np.empty((B, len(rows_), len(heads_), d), dtype=np.float64)
    for b in range(B):
        for hi, h in enumerate(heads_):
            for g, st in enumerate(sets):
                sel = np.nonzero(set_of[rows_] == g)[0]
                if sel.size == 0:
                    continue
                idx = np.asarray(st)
                out[b, sel, hi] = attention_head_ref(q[b, idx, h], k[b, idx, h], v[b, idx, h],
                                                     scale, slot_of[rows_[sel]])
    return out


# ----------------------------------------------------------------------------------------------
# Packed batches of videos of different shapes
# ----------------------------------------------------------------------------------------------
#
# "CogVideoX", section 3.1 "Multi-Resolution Frame Pack": videos of different durations and
# resolutions are placed into one batch (after Patch'n Pack / NaViT), and each video's 3D RoPE
# positions are its own grid coordinates (extrapolation: the front of one position table, never
# rescaled).  Readings: the packed sequence is the concatenation of samples; sample i is its own
# text_i tokens followed by its T_i*H_i*W_i video tokens; a token attends only to the tokens of its
# own sample (Patch'n Pack's example masking), i.e. attention is block-diagonal over samples.

def segment_bounds(lengths: Sequence[int]) -> np.ndarray:
    """Start offsets of consecutive segments: [0, l_0, l_0 + l_1, ...] (n_seg + 1 entries)."""
    out = np.zeros(len(lengths) + 1, dtype=np.int64)
    out[1:] = np.cumsum(np.asarray(lengths, dtype=np.int64))
    return out


def rope3d_packed_ref(x: np.ndarray, samples: Sequence[Sequence[int]], split: Sequence[int],
                      theta: float = 10000.0) -> np.ndarray:
    """3D RoPE over a packed [1, sum_i (text_i + T_i*H_i*W_i), n_h, d] sequence.

    ``samples`` lists (text_len, T, H, W) per packed sample.  Every sample is rotated exactly as
    ``rope3d_ref`` rotates it on its own: its video positions start at (0, 0, 0) and follow its
    own grid; its text tokens are left unrotated.
    """
    x = np.asarray(x, dtype=np.float64)
    lens = [int(L) + int(T) * int(H) * int(W) for L, T, H, W in samples]
    bounds = segment_bounds(lens)
    if x.shape[0] != 1 or x.shape[1] != bounds[-1]:
        raise ValueError("packed tensor must be [1, sum of sample lengths, heads, d]")
    out = np.empty_like(x)
    for i, (L, T, H, W) in enumerate(samples):
        a, b = bounds[i], bounds[i + 1]
        out[:, a:b] = rope3d_ref(x[:, a:b], (T, H, W), int(L), split, theta)
    return out


def packed_attn_ref(q: np.ndarray, k: np.ndarray, v: np.ndarray, q_bounds: Sequence[int],
                    kv_bounds: Sequence[int] | None = None, scale: float | None = None,
                    rows=None, heads=None) -> np.ndarray:
    """Block-diagonal attention over a packed batch: query token r of segment i attends to the
    key/value tokens of segment i only, per head.

    q: [1, N_q, n_h, d]; k, v: [1, N_kv, n_h, d].  Segment i owns query rows
    [q_bounds[i], q_bounds[i+1]) and key rows [kv_bounds[i], kv_bounds[i+1]) (the same rows
    when ``kv_bounds`` is None: self-attention within each sample).  ``rows`` optionally
    selects query rows (packed indices); the result is [1, len(rows), len(heads), d].
    """
    qb = np.asarray(q_bounds, dtype=np.int64)
    kb = qb if kv_bounds is None else np.asarray(kv_bounds, dtype=np.int64)
    _, Nq, nh, d = q.shape
    scale = default_scale(d) if scale is None else scale
    rows_ = np.arange(Nq) if rows is None else np.asarray(rows)
    heads_ = np.arange(nh) if heads is None else np.asarray(heads)
    seg_of = np.searchsorted(qb, rows_, side="right") - 1
    out = np.empty((1, len(rows_), len(heads_), d), dtype=np.float64)
    for i in range(len(qb) - 1):
        sel = np.nonzero(seg_of == i)[0]
        if sel.size == 0:
            continue
        kk = slice(kb[i], kb[i + 1])
        for hi, h in enumerate(heads_):
            out[0, sel, hi] = attention_head_ref(q[0, qb[i]:qb[i + 1], h], k[0, kk, h], v[0, kk, h], scale,
                                                 rows_[sel] - qb[i])
    return out


# ----------------------------------------------------------------------------------------------
# Factorized and frame-causal attention masks
# ----------------------------------------------------------------------------------------------
#
# "CogVideoX" section 2.2 and Table 8 compare 3D full attention with "2D + 1D" attention:
# separate spatial attention (within one frame) and temporal attention (across frames).  The
# Sora page ("Video DiT Diffusion Model") names Local Spatial Attention (patches of the same
# frame; a block-diagonal 0/1 mask over frames), Causal Time Attention (previous frames), and
# brute-force long-time attention (frame i attends to all earlier frames).  Readings: spatial
# and temporal attention act on the video tokens only (no text); temporal attention of token
# (t, h, w) covers the tokens (t', h, w) of the same spatial position, every t' (bidirectional)
# or t' <= t (causal); frame-causal attention lets a token of frame t attend to every token of
# frames 0..t, with a text prefix forming a block before frame 0 (text attends to text only,
# every video token attends to the text).

def spatial_attn_ref(q: np.ndarray, k: np.ndarray, v: np.ndarray, grid: Sequence[int],
                     scale: float | None = None) -> np.ndarray:
    """Per-frame attention: token (t, h, w) attends to the H*W tokens of frame t.
    q, k, v: [B, T*H*W, n_h, d] video tokens (no text)."""
    T, H, W = (int(a) for a in grid)
    B, N, nh, d = q.shape
    if N != T * H * W:
        raise ValueError("spatial attention takes the T*H*W video tokens only")
    scale = default_scale(d) if scale is None else scale
    out = np.empty((B, N, nh, d), dtype=np.float64)
    HW = H * W
    for b in range(B):
        for t in range(T):
            f = slice(t * HW, (t + 1) * HW)
            for h in range(nh):
                out[b, f, h] = attention_head_ref(q[b, f, h], k[b, f, h], v[b, f, h], scale)
    return out


def temporal_attn_ref(q: np.ndarray, k: np.ndarray, v: np.ndarray, grid: Sequence[int],
                      causal: bool = False, scale: float | None = None) -> np.ndarray:
    """Per-position attention over time: token (t, h, w) attends to the tokens (t', h, w),
    all t' or (causal) t' <= t.  q, k, v: [B, T*H*W, n_h, d] video tokens (no text)."""
    T, H, W = (int(a) for a in grid)
    B, N, nh, d = q.shape
    if N != T * H * W:
        raise ValueError("temporal attention takes the T*H*W video tokens only")
    scale = default_scale(d) if scale is None else scale
    HW = H * W
    out = np.empty((B, N, nh, d), dtype=np.float64)
    for b in range(B):
        for pos in range(HW):
            idx = pos + HW * np.arange(T)          # the position's token in every frame
            for h in range(nh):
                if not causal:
                    out[b, idx, h] = attention_head_ref(q[b, idx, h], k[b, idx, h], v[b, idx, h], scale)
                else:
                    for t in range(T):
                        sub = idx[:t + 1]
                        out[b, idx[t], h] = attention_head_ref(q[b, idx[t:t + 1], h], k[b, sub, h], v[b, sub, h],
                                                               scale)[0]
    return out


def frame_causal_limit(token: int, text_len: int, HW: int) -> int:
    """Number of leading tokens a query token may attend to under the frame-causal mask: the
    text block for a text token, the text and frames 0..t for a token of frame t."""
    if token < text_len:
        return text_len
    return text_len + ((token - text_len) // HW + 1) * HW


def frame_causal_attn_ref(q: np.ndarray, k: np.ndarray, v: np.ndarray, grid: Sequence[int], text_len: int,
                          scale: float | None = None, rows=None, heads=None) -> np.ndarray:
    """Frame-causal attention over [B, text_len + T*H*W, n_h, d]: query token r attends to the
    first frame_causal_limit(r) tokens.  ``rows`` / ``heads`` select a subset as in attn_ref."""
    T, H, W = (int(a) for a in grid)
    B, N, nh, d = q.shape
    if N != text_len + T * H * W:
        raise ValueError("sequence length does not match text_len + T*H*W")
    scale = default_scale(d) if scale is None else scale
    rows_ = np.arange(N) if rows is None else np.asarray(rows)
    heads_ = np.arange(nh) if heads is None else np.asarray(heads)
    lim = np.array([frame_causal_limit(int(r), text_len, H * W) for r in rows_])
    out = np.empty((B, len(rows_), len(heads_), d), dtype=np.float64)
    for b in range(B):
        for hi, h in enumerate(heads_):
            for L in np.unique(lim):
                sel = np.nonzero(lim == L)[0]
                out[b, sel, hi] = attention_head_ref(q[b, :L, h], k[b, :L, h], v[b, :L, h], scale, rows_[sel])
    return out


# ----------------------------------------------------------------------------------------------
# Skiparse with a text prefix joined to every set
# ----------------------------------------------------------------------------------------------
#
# Not on the pages (Open-Sora Plan feeds text through cross-attention; CogVideoX joins text and
# video in dense attention).  Reading for a joint text + video sequence under Skiparse: the text
# tokens are global tokens.  A video token of set g attends to every text token and to the video
# tokens of set g; a text token attends to every token of its sample.

def skiparse_text_attn_ref(q: np.ndarray, k: np.ndarray, v: np.ndarray, text_len: int, k_ratio: int, mode: int,
                           scale: float | None = None, rows=None, heads=None) -> np.ndarray:
    """q, k, v: [B, text_len + N_v, n_h, d].  ``rows`` (token indices) / ``heads`` select a
    subset as in attn_ref."""
    B, N, nh, d = q.shape
    L = int(text_len)
    scale = default_scale(d) if scale is None else scale
    sets = skiparse_sets(N - L, k_ratio, mode)
    set_of = np.empty(N - L, dtype=np.int64)
    for g, st in enumerate(sets):
        set_of[st] = g
    rows_ = np.arange(N) if rows is None else np.asarray(rows)
    heads_ = np.arange(nh) if heads is None else np.asarray(heads)
    out = np.empty((B, len(rows_), len(heads_), d), dtype=np.float64)
    text = np.arange(L)
    for b in range(B):
        for hi, h in enumerate(heads_):
            sel = np.nonzero(rows_ < L)[0]
            if sel.size:
                out[b, sel, hi] = attention_head_ref(q[b, :, h], k[b, :, h], v[b, :, h], scale, rows_[sel])
            for g, st in enumerate(sets):
                sel = np.nonzero((rows_ >= L) & (set_of[np.maximum(rows_ - L, 0)] == g))[0]
                if sel.size == 0:
                    continue
                keys = np.concatenate([text, L + np.asarray(st)])
                out[b, sel, hi] = attention_head_ref(q[b, rows_[sel], h], k[b, keys, h], v[b, keys, h], scale)
    return out


# ----------------------------------------------------------------------------------------------
# Backward pass (gradients of the attention output)
# ----------------------------------------------------------------------------------------------
#
# Open-Sora Plan trains with Skiparse attention (section 2.2.2 and the sparse-tuning stage), so
# the hot path has a backward pass.  For one head with S = q k^T * scale, P = softmax(S) (rows),
# O = P v and an upstream gradient dO, the chain rule gives
#   dV = P^T dO,   dP = dO v^T,   dS = P * (dP - rowsum(P * dP)),
#   dQ = dS k * scale,   dK = dS^T q * scale,
# and rowsum(P * dP) = rowsum(dO * O).  The log-sum-exp of a row, lse = log sum_j exp(S_ij), is
# what the forward pass keeps so that P can be rebuilt as exp(S - lse).

def attention_head_lse_ref(q: np.ndarray, k: np.ndarray, scale: float) -> np.ndarray:
    """Natural log-sum-exp of every row of q k^T * scale (one head), fp64."""
    s = (np.asarray(q, np.float64) @ np.asarray(k, np.float64).T) * scale
    m = s.max(axis=1)
    return m + np.log(np.exp(s - m[:, None]).sum(axis=1))


def attention_head_backward_ref(q, k, v, do, scale: float):
    """(dq, dk, dv) of one head by the chain rule above, fp64."""
    q, k, v, do = (np.asarray(a, np.float64) for a in (q, k, v, do))
    p = softmax_rows((q @ k.T) * scale)
    o = p @ v
    dv = p.T @ do
    dp = do @ v.T
    ds = p * (dp - (do * o).sum(axis=1, keepdims=True))
    return ds @ k * scale, ds.T @ q * scale, dv


def attn_backward_ref(q, k, v, do, scale: float | None = None):
    """Gradients of 3D full attention (attn_ref) for [B, N, n_h, d] inputs: (dq, dk, dv)."""
    B, N, nh, d = q.shape
    scale = default_scale(d) if scale is None else scale
    out = [np.empty((B, N, nh, d)) for _ in range(3)]
    for b in range(B):
        for h in range(nh):
            g = attention_head_backward_ref(q[b, :, h], k[b, :, h], v[b, :, h], do[b, :, h], scale)
            for o_, g_ in zip(out, g):
                o_[b, :, h] = g_
    return tuple(out)


def skiparse_backward_ref(q, k, v, do, k_ratio: int, mode: int, scale: float | None = None):
    """Gradients of Skiparse attention (skiparse_attn_ref, no text): each set's own backward,
    scattered back to natural token order."""
    B, N, nh, d = q.shape
    scale = default_scale(d) if scale is None else scale
    out = [np.empty((B, N, nh, d)) for _ in range(3)]
    for st in skiparse_sets(N, k_ratio, mode):
        idx = np.asarray(st)
        for b in range(B):
            for h in range(nh):
                g = attention_head_backward_ref(q[b, idx, h], k[b, idx, h], v[b, idx, h], do[b, idx, h], scale)
                for o_, g_ in zip(out, g):
                    o_[b, idx, h] = g_
    return tuple(out)


def attention_head_backward_rows_ref(q, k, v, do, scale: float, q_rows, k_rows, chunk: int = 2048):
    """Selected rows of (dq, dk, dv) of one head, without forming the full score matrix: dq for
    query rows ``q_rows``, dk and dv for key rows ``k_rows``.  Same chain rule as
    attention_head_backward_ref; the row log-sum-exp and rowsum(dO * O) of every query come first
    (query chunks of ``chunk`` rows)."""
    q, k, v, do = (np.asarray(a, np.float64) for a in (q, k, v, do))
    n = q.shape[0]
    lse = np.empty(n)
    dsum = np.empty(n)
    for r0 in range(0, n, chunk):
        s = (q[r0:r0 + chunk] @ k.T) * scale
        m = s.max(axis=1)
        e = np.exp(s - m[:, None])
        z = e.sum(axis=1)
        lse[r0:r0 + chunk] = m + np.log(z)
        o = (e / z[:, None]) @ v
        dsum[r0:r0 + chunk] = (do[r0:r0 + chunk] * o).sum(axis=1)
    qr = np.asarray(q_rows)
    p = np.exp((q[qr] @ k.T) * scale - lse[qr][:, None])
    ds = p * (do[qr] @ v.T - dsum[qr][:, None])
    dq = ds @ k * scale
    kr = np.asarray(k_rows)
    pt = np.exp((q @ k[kr].T) * scale - lse[:, None])              # [n, len(k_rows)]
    dst = pt * (do @ v[kr].T - dsum[:, None])
    dk = dst.T @ q * scale
    dv = pt.T @ do
    return dq, dk, dv


def frame_causal_backward_ref(q, k, v, do, grid: Sequence[int], text_len: int, scale: float | None = None):
    """Gradients of frame-causal attention (frame_causal_attn_ref): the backward chain rule above
    with P zero outside the mask (query token r sees the first frame_causal_limit(r) keys)."""
    T, H, W = (int(a) for a in grid)
    B, N, nh, d = q.shape
    scale = default_scale(d) if scale is None else scale
    lim = np.array([frame_causal_limit(r, text_len, H * W) for r in range(N)])
    allowed = np.arange(N)[None, :] < lim[:, None]
    out = [np.empty((B, N, nh, d)) for _ in range(3)]
    for b in range(B):
        for h in range(nh):
            qh, kh, vh, dh = (np.asarray(a[b, :, h], np.float64) for a in (q, k, v, do))
            s = np.where(allowed, (qh @ kh.T) * scale, -np.inf)
            p = softmax_rows(s)
            o = p @ vh
            ds = p * (dh @ vh.T - (dh * o).sum(axis=1, keepdims=True))
            out[0][b, :, h] = ds @ kh * scale
            out[1][b, :, h] = ds.T @ qh * scale
            out[2][b, :, h] = p.T @ dh
    return tuple(out)


def spatial_backward_ref(q, k, v, do, grid: Sequence[int], scale: float | None = None):
    """Gradients of per-frame attention (spatial_attn_ref): every frame's own backward by the
    chain rule above.  q, k, v, do: [B, T*H*W, n_h, d] video tokens."""
    T, H, W = (int(a) for a in grid)
    B, N, nh, d = q.shape
    if N != T * H * W:
        raise ValueError("spatial attention takes the T*H*W video tokens only")
    scale = default_scale(d) if scale is None else scale
    HW = H * W
    out = [np.empty((B, N, nh, d)) for _ in range(3)]
    for b in range(B):
        for t in range(T):
            f = slice(t * HW, (t + 1) * HW)
            for h in range(nh):
                g = attention_head_backward_ref(q[b, f, h], k[b, f, h], v[b, f, h], do[b, f, h], scale)
                for o_, g_ in zip(out, g):
                    o_[b, f, h] = g_
    return tuple(out)


def temporal_backward_ref(q, k, v, do, grid: Sequence[int], causal: bool = False, scale: float | None = None):
    """Gradients of per-position attention over time (temporal_attn_ref): for each spatial
    position, the chain rule above over its T tokens, with P zero where t' > t when causal."""
    T, H, W = (int(a) for a in grid)
    B, N, nh, d = q.shape
    if N != T * H * W:
        raise ValueError("temporal attention takes the T*H*W video tokens only")
    scale = default_scale(d) if scale is None else scale
    HW = H * W
    allowed = np.tril(np.ones((T, T), dtype=bool)) if causal else np.ones((T, T), dtype=bool)
    out = [np.empty((B, N, nh, d)) for _ in range(3)]
    for b in range(B):
        for pos in range(HW):
            idx = pos + HW * np.arange(T)
            for h in range(nh):
                qh, kh, vh, dh = (np.asarray(a[b, idx, h], np.float64) for a in (q, k, v, do))
                p = softmax_rows(np.where(allowed, (qh @ kh.T) * scale, -np.inf))
                o = p @ vh
                ds = p * (dh @ vh.T - (dh * o).sum(axis=1, keepdims=True))
                out[0][b, idx, h] = ds @ kh * scale
                out[1][b, idx, h] = ds.T @ qh * scale
                out[2][b, idx, h] = p.T @ dh
    return tuple(out)



def packed_backward_ref(q, k, v, do, q_bounds: Sequence[int], scale: float | None = None):
    """Gradients of block-diagonal self-attention over a packed batch (packed_attn_ref with
    kv_bounds = q_bounds; CogVideoX section 3.1, Multi-Resolution Frame Pack): each sample's own
    backward by the chain rule above, per head, written at the sample's rows.

    q, k, v, do: [1, N, n_h, d] packed tensors; sample i owns rows [q_bounds[i], q_bounds[i+1])."""
    qb = np.asarray(q_bounds, dtype=np.int64)
    _, N, nh, d = q.shape
    scale = default_scale(d) if scale is None else scale
    out = [np.zeros((1, N, nh, d)) for _ in range(3)]
    for i in range(len(qb) - 1):
        r = slice(qb[i], qb[i + 1])
        if qb[i + 1] <= qb[i]:
            continue
        for h in range(nh):
            g = attention_head_backward_ref(q[0, r, h], k[0, r, h], v[0, r, h], do[0, r, h], scale)
            for o_, g_ in zip(out, g):
                o_[0, r, h] = g_
    return tuple(out)


def skiparse_text_backward_ref(q, k, v, do, text_len: int, k_ratio: int, mode: int, scale: float | None = None):
    """Gradients of Skiparse attention with a joined text prefix (skiparse_text_attn_ref): per
    sample and head, the chain rule above on the masked score matrix whose row for a text token
    sees every token and whose row for a video token of set g sees the text tokens and set g."""
    B, N, nh, d = q.shape
    L = int(text_len)
    scale = default_scale(d) if scale is None else scale
    visible = np.zeros((N, N), dtype=bool)
    visible[:L, :] = True
    for st in skiparse_sets(N - L, k_ratio, mode):
        rows = L + np.asarray(st)
        visible[np.ix_(rows, np.arange(L))] = True
        visible[np.ix_(rows, rows)] = True
    out = [np.empty((B, N, nh, d)) for _ in range(3)]
    for b in range(B):
        for h in range(nh):
            qh, kh, vh, dh = (np.asarray(a[b, :, h], np.float64) for a in (q, k, v, do))
            p = softmax_rows(np.where(visible, (qh @ kh.T) * scale, -np.inf))
            o = p @ vh
            ds = p * (dh @ vh.T - (dh * o).sum(axis=1, keepdims=True))
            out[0][b, :, h] = ds @ kh * scale
            out[1][b, :, h] = ds.T @ qh * scale
            out[2][b, :, h] = p.T @ dh
    return tuple(out)


def skiparse_text_backward_rows_ref(q, k, v, do, text_len: int, k_ratio: int, mode: int, q_rows, k_rows,
                                    heads=None, scale: float | None = None, chunk: int = 2048):
    """Selected rows of the gradients of skiparse_text_attn_ref (text_len = 0: of
    skiparse_attn_ref), without forming the N x N score matrix: dq for tokens ``q_rows``, dk and
    dv for tokens ``k_rows``, for heads ``heads`` (all by default); each [B, rows, heads, d].
    The same chain rule as skiparse_text_backward_ref on the masked score matrix: row r of a text
    token sees every token, row r of a video token of set g the text tokens and set g.  The
    row log-sum-exp and rowsum(dO * O) of every query come first, per group of rows that see the
    same keys (the text rows; each set's rows), in chunks of ``chunk`` rows."""
    B, N, nh, d = q.shape
    L = int(text_len)
    scale = default_scale(d) if scale is None else scale
    sets = [L + np.asarray(st, dtype=np.int64) for st in skiparse_sets(N - L, k_ratio, mode)]
    text = np.arange(L)
    set_of = np.empty(N, dtype=np.int64)
    set_of[:L] = -1
    for g, st in enumerate(sets):
        set_of[st] = g
    # (rows, their keys) per group of rows that see the same keys
    groups = ([(text, np.arange(N))] if L else []) + [(st, np.concatenate([text, st])) for st in sets]
    heads_ = np.arange(nh) if heads is None else np.asarray(heads)
    qr, kr = np.asarray(q_rows, dtype=np.int64), np.asarray(k_rows, dtype=np.int64)
    # only the groups whose rows are read: the text rows (they see every key), the sets of the
    # selected video rows and keys, and every set if a text key is selected
    need = {int(set_of[r]) for r in np.concatenate([qr, kr]) if r >= L}
    if (kr < L).any():
        need = set(range(len(sets)))
    groups = ([groups[0]] if L else []) + [groups[(1 if L else 0) + g] for g in sorted(need)]
    out = [np.empty((B, len(qr), len(heads_), d)), np.empty((B, len(kr), len(heads_), d)),
           np.empty((B, len(kr), len(heads_), d))]
    for b in range(B):
        for hi, h in enumerate(heads_):
            qh, kh, vh, dh = (np.asarray(a[b, :, h], np.float64) for a in (q, k, v, do))
            lse = np.empty(N)
            dsum = np.empty(N)
            for rows, keys in groups:
                for r0 in range(0, len(rows), chunk):
                    rr = rows[r0:r0 + chunk]
                    s = (qh[rr] @ kh[keys].T) * scale
                    m = s.max(axis=1)
                    e = np.exp(s - m[:, None])
                    z = e.sum(axis=1)
                    lse[rr] = m + np.log(z)
                    dsum[rr] = (dh[rr] * ((e / z[:, None]) @ vh[keys])).sum(axis=1)
            # dq of the selected query rows, over the keys each row sees
            for i, r in enumerate(qr):
                keys = np.arange(N) if r < L else np.concatenate([text, sets[set_of[r]]])
                p = np.exp((kh[keys] @ qh[r]) * scale - lse[r])
                ds = p * (vh[keys] @ dh[r] - dsum[r])
                out[0][b, i, hi] = ds @ kh[keys] * scale
            # dk, dv of the selected key rows, over the query rows that see each key
            for i, j in enumerate(kr):
                rows = np.arange(N) if j < L else np.concatenate([text, sets[set_of[j]]])
                p = np.exp((qh[rows] @ kh[j]) * scale - lse[rows])
                ds = p * (dh[rows] @ vh[j] - dsum[rows])
                out[1][b, i, hi] = ds @ qh[rows] * scale
                out[2][b, i, hi] = p @ dh[rows]
    return tuple(out)


def frame_causal_backward_rows_ref(q, k, v, do, grid: Sequence[int], text_len: int, q_rows, k_rows, heads=None,
                                   scale: float | None = None, chunk: int = 2048):
    """Selected rows of the gradients of frame_causal_attn_ref without forming the N x N score
    matrix: dq for tokens ``q_rows``, dk and dv for tokens ``k_rows``, for heads ``heads`` (all by
    default); each [B, rows, heads, d].  Row r sees the first frame_causal_limit(r) tokens; the
    row log-sum-exp and rowsum(dO * O) of every row come first, per group of rows with the same
    limit (the text block; each frame), in chunks of ``chunk`` rows."""
    T, H, W = (int(a) for a in grid)
    B, N, nh, d = q.shape
    L = int(text_len)
    HW = H * W
    scale = default_scale(d) if scale is None else scale
    lim = np.array([frame_causal_limit(r, L, HW) for r in range(N)])
    groups = ([np.arange(L)] if L else []) + [L + t * HW + np.arange(HW) for t in range(T)]
    heads_ = np.arange(nh) if heads is None else np.asarray(heads)
    qr, kr = np.asarray(q_rows, dtype=np.int64), np.asarray(k_rows, dtype=np.int64)
    out = [np.empty((B, len(qr), len(heads_), d)), np.empty((B, len(kr), len(heads_), d)),
           np.empty((B, len(kr), len(heads_), d))]
    for b in range(B):
        for hi, h in enumerate(heads_):
            qh, kh, vh, dh = (np.asarray(a[b, :, h], np.float64) for a in (q, k, v, do))
            lse = np.empty(N)
            dsum = np.empty(N)
            for rows in groups:
                n_keys = lim[rows[0]]
                for r0 in range(0, len(rows), chunk):
                    rr = rows[r0:r0 + chunk]
                    s = (qh[rr] @ kh[:n_keys].T) * scale
                    m = s.max(axis=1)
                    e = np.exp(s - m[:, None])
                    z = e.sum(axis=1)
                    lse[rr] = m + np.log(z)
                    dsum[rr] = (dh[rr] * ((e / z[:, None]) @ vh[:n_keys])).sum(axis=1)
            for i, r in enumerate(qr):
                keys = np.arange(lim[r])
                p = np.exp((kh[keys] @ qh[r]) * scale - lse[r])
                ds = p * (vh[keys] @ dh[r] - dsum[r])
                out[0][b, i, hi] = ds @ kh[keys] * scale
            for i, j in enumerate(kr):
                rows = np.nonzero(lim > j)[0]          # the rows whose limit covers key j
                p = np.exp((qh[rows] @ kh[j]) * scale - lse[rows])
                ds = p * (dh[rows] @ vh[j] - dsum[rows])
                out[1][b, i, hi] = ds @ qh[rows] * scale
                out[2][b, i, hi] = p @ dh[rows]
    return tuple(out)
