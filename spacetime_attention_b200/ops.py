"""ctypes binding over libosp.so (declared in include/osp.h).

Argument marshalling only: every function takes torch CUDA tensors, checks dtype/layout/device,
passes raw device pointers, the shape structs and the current CUDA stream to the C entry point
of the same name, and raises on a non-zero status.  All computation happens in the library's
CUDA kernels; there is no fallback of any kind.  If the library is missing or cannot be loaded,
every call raises.
"""

from __future__ import annotations

import ctypes
import math
import os
from typing import Optional, Sequence

import torch

# OSP_LIBRARY=debug selects the debug build (libosp_debug.so: device-side index checks that report
# OSP_ERR_BOUNDS); any other value is taken as a path.
_LIB_DIR = os.path.dirname(os.path.abspath(__file__))
_LIB_SEL = os.environ.get("OSP_LIBRARY", "")
LIB_PATH = (os.path.join(_LIB_DIR, "libosp_debug.so") if _LIB_SEL == "debug"
            else (_LIB_SEL or os.path.join(_LIB_DIR, "libosp.so")))

OSP_SKIP_SINGLE = 0
OSP_SKIP_GROUP = 1

STATUS_NAMES = {0: "OSP_OK", 1: "OSP_ERR_INVALID_ARG", 2: "OSP_ERR_UNSUPPORTED", 3: "OSP_ERR_DIVISIBILITY",
                4: "OSP_ERR_CUDA", 5: "OSP_ERR_TIMEOUT", 6: "OSP_ERR_BOUNDS"}

# Every symbol include/osp.h declares (tests check the library exports all of them).
EXPORTED = ("osp_rope3d", "osp_attn_full", "osp_skiparse_gather", "osp_skiparse_scatter", "osp_skiparse_attn",
            "osp_skiparse_index_map", "osp_check_status", "osp_get_last_error", "osp_version",
            "osp_attn_full_noalloc", "osp_attn_cross", "osp_rope3d_packed", "osp_attn_packed",
            "osp_attn_spatial", "osp_attn_temporal", "osp_attn_frame_causal", "osp_attn_forward_train",
            "osp_attn_backward", "osp_attn_frame_causal_train", "osp_attn_frame_causal_backward",
            "osp_attn_spatial_train", "osp_attn_spatial_backward", "osp_attn_temporal_train",
            "osp_attn_temporal_backward", "osp_attn_packed_lse_rows", "osp_attn_packed_train",
            "osp_attn_packed_backward")

MAX_SEGMENTS = 256   # OSP_MAX_SEGMENTS


class OspShape(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int32), ("text_len", ctypes.c_int32), ("T", ctypes.c_int32),
                ("H", ctypes.c_int32), ("W", ctypes.c_int32), ("heads", ctypes.c_int32),
                ("head_dim", ctypes.c_int32)]


class OspRope(ctypes.Structure):
    _fields_ = [("d_t", ctypes.c_int32), ("d_h", ctypes.c_int32), ("d_w", ctypes.c_int32),
                ("theta", ctypes.c_double)]


class OspSampleGrid(ctypes.Structure):
    _fields_ = [("text_len", ctypes.c_int32), ("T", ctypes.c_int32), ("H", ctypes.c_int32), ("W", ctypes.c_int32)]


class OspError(RuntimeError):
    def __init__(self, fn: str, code: int, msg: str):
        super().__init__(f"{fn} -> {STATUS_NAMES.get(code, code)}: {msg}")
        self.code = code


_lib = None


def library() -> ctypes.CDLL:
    """Load libosp.so (once).  Raises if it is missing: there is no fallback path."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m spacetime_attention_b200.build`")
        lib = ctypes.CDLL(LIB_PATH)
        vp, i32, sp, rp = ctypes.c_void_p, ctypes.c_int32, ctypes.POINTER(OspShape), ctypes.POINTER(OspRope)
        sig = {
            "osp_rope3d": [vp, vp, vp, vp, sp, rp, vp],
            "osp_attn_full": [vp, vp, vp, vp, sp, ctypes.c_float, vp],
            "osp_attn_full_noalloc": [vp, vp, vp, vp, sp, ctypes.c_float, vp],
            "osp_attn_cross": [vp, vp, vp, vp, sp, ctypes.c_float, vp],
            "osp_attn_spatial": [vp, vp, vp, vp, sp, ctypes.c_float, vp],
            "osp_attn_forward_train": [vp, vp, vp, vp, vp, sp, i32, i32, ctypes.c_float, vp],
            "osp_attn_backward": [vp, vp, vp, vp, vp, vp, vp, vp, vp, sp, i32, i32, ctypes.c_float, vp],
            "osp_attn_frame_causal_train": [vp, vp, vp, vp, vp, sp, ctypes.c_float, vp],
            "osp_attn_frame_causal_backward": [vp, vp, vp, vp, vp, vp, vp, vp, vp, sp, ctypes.c_float, vp],
            "osp_attn_temporal": [vp, vp, vp, vp, sp, i32, ctypes.c_float, vp],
            "osp_attn_spatial_train": [vp, vp, vp, vp, vp, sp, ctypes.c_float, vp],
            "osp_attn_spatial_backward": [vp, vp, vp, vp, vp, vp, vp, vp, vp, sp, ctypes.c_float, vp],
            "osp_attn_temporal_train": [vp, vp, vp, vp, vp, sp, i32, ctypes.c_float, vp],
            "osp_attn_temporal_backward": [vp, vp, vp, vp, vp, vp, vp, vp, vp, sp, i32, ctypes.c_float, vp],
            "osp_attn_frame_causal": [vp, vp, vp, vp, sp, ctypes.c_float, vp],
            "osp_rope3d_packed": [vp, vp, vp, vp, ctypes.POINTER(OspSampleGrid), i32, i32, i32, rp, vp],
            "osp_attn_packed": [vp, vp, vp, vp, ctypes.POINTER(ctypes.c_int32), ctypes.POINTER(ctypes.c_int32), i32,
                                i32, i32, ctypes.c_float, vp],
            "osp_attn_packed_lse_rows": [ctypes.POINTER(ctypes.c_int32), i32],
            "osp_attn_packed_train": [vp, vp, vp, vp, vp, ctypes.POINTER(ctypes.c_int32), i32, i32, i32,
                                      ctypes.c_float, vp],
            "osp_attn_packed_backward": [vp, vp, vp, vp, vp, vp, vp, vp, vp, ctypes.POINTER(ctypes.c_int32), i32,
                                         i32, i32, ctypes.c_float, vp],
            "osp_skiparse_gather": [vp, vp, vp, vp, vp, vp, sp, i32, i32, rp, vp],
            "osp_skiparse_scatter": [vp, vp, sp, i32, i32, vp],
            "osp_skiparse_attn": [vp, vp, vp, vp, sp, i32, i32, ctypes.c_float, vp],
            "osp_skiparse_index_map": [i32, i32, i32, vp, vp],
            "osp_check_status": [vp],
            "osp_get_last_error": [],
            "osp_version": [],
        }
        for name, args in sig.items():
            f = getattr(lib, name)
            f.argtypes = args
            f.restype = ctypes.c_char_p if name == "osp_get_last_error" else ctypes.c_int
        _lib = lib
    return _lib


def _check(fn: str, rc: int):
    if rc != 0:
        raise OspError(fn, rc, library().osp_get_last_error().decode())


def _stream_handle(t: torch.Tensor):
    return ctypes.c_void_p(torch.cuda.current_stream(t.device).cuda_stream)


def _ptr(t: Optional[torch.Tensor]):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else ctypes.c_void_p(0)


def _bshd(t: torch.Tensor, name: str):
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != torch.bfloat16:
        raise ValueError(f"{name} must be bfloat16")
    if t.dim() != 4 or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous [B, N, heads, head_dim] tensor")


def make_shape(B: int, text_len: int, grid: Sequence[int], heads: int, head_dim: int) -> OspShape:
    T, H, W = (int(x) for x in grid)
    return OspShape(int(B), int(text_len), T, H, W, int(heads), int(head_dim))


def make_rope(split: Sequence[int], theta: float = 10000.0) -> OspRope:
    d_t, d_h, d_w = (int(x) for x in split)
    return OspRope(d_t, d_h, d_w, float(theta))


def _shape_of(t: torch.Tensor, grid, text_len: int) -> OspShape:
    """The call's shape from q's [B, N, heads, d]; N must be text_len + T*H*W, since the library
    sizes every access from the shape alone."""
    B, N, heads, d = t.shape
    T, H, W = (int(x) for x in grid)
    if N != int(text_len) + T * H * W:
        raise ValueError(f"q has {N} tokens per sample, but text_len + T*H*W = {int(text_len)} + "
                         f"{T}*{H}*{W} = {int(text_len) + T * H * W}")
    return make_shape(B, text_len, grid, heads, d)


def _same(t: torch.Tensor, ref: torch.Tensor, name: str) -> torch.Tensor:
    """t, checked to have ref's shape and device (the library reads or writes it with ref's
    layout), and to be a contiguous bf16 CUDA tensor."""
    if tuple(t.shape) != tuple(ref.shape) or t.device != ref.device:
        raise ValueError(f"{name} must have shape {tuple(ref.shape)} on {ref.device} "
                         f"(got {tuple(t.shape)} on {t.device})")
    _bshd(t, name)
    return t


def _out(t: Optional[torch.Tensor], ref: torch.Tensor, name: str) -> torch.Tensor:
    """A caller's output tensor, checked like ref, or a new one."""
    return torch.empty_like(ref) if t is None else _same(t, ref, name)


def _heads_match(t: torch.Tensor, ref: torch.Tensor, name: str) -> None:
    """t has ref's batch, heads and head_dim (its token count may differ)."""
    if t.dim() != 4 or t.shape[0] != ref.shape[0] or tuple(t.shape[2:]) != tuple(ref.shape[2:]) \
            or t.device != ref.device:
        raise ValueError(f"{name} must be [{ref.shape[0]}, n, {ref.shape[2]}, {ref.shape[3]}] on {ref.device} "
                         f"(got {tuple(t.shape)} on {t.device})")
    _bshd(t, name)


def _packed_rows(samples) -> int:
    """Rows of a packed batch: the sum of text_len + T*H*W over its samples."""
    return sum(int(L) + int(T) * int(H) * int(W) for L, T, H, W in samples)


def rope3d(q: torch.Tensor, k: torch.Tensor, grid, text_len: int, split, theta: float = 10000.0,
           q_out: Optional[torch.Tensor] = None, k_out: Optional[torch.Tensor] = None):
    """osp_rope3d: 3D RoPE of q and k; returns (q_out, k_out) (new tensors unless given)."""
    _bshd(q, "q"); _same(k, q, "k")
    shp, rp = _shape_of(q, grid, text_len), make_rope(split, theta)
    q_out, k_out = _out(q_out, q, "q_out"), _out(k_out, k, "k_out")
    _check("osp_rope3d", library().osp_rope3d(_ptr(q), _ptr(k), _ptr(q_out), _ptr(k_out), ctypes.byref(shp),
                                              ctypes.byref(rp), _stream_handle(q)))
    return q_out, k_out


def attn_full(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, grid, text_len: int, scale: float = 0.0,
              o: Optional[torch.Tensor] = None) -> torch.Tensor:
    """osp_attn_full: dense 3D full attention over text_len + T*H*W tokens."""
    _bshd(q, "q"); _same(k, q, "k"); _same(v, q, "v")
    shp = _shape_of(q, grid, text_len)
    o = _out(o, q, "o")
    _check("osp_attn_full", library().osp_attn_full(_ptr(q), _ptr(k), _ptr(v), _ptr(o), ctypes.byref(shp),
                                                    ctypes.c_float(scale), _stream_handle(q)))
    return o


def attn_cross(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, grid, scale: float = 0.0,
               o: Optional[torch.Tensor] = None) -> torch.Tensor:
    """osp_attn_cross: video queries q [B, T*H*W, heads, d] attend to text keys/values
    k, v [B, text_len, heads, d]."""
    _bshd(q, "q"); _heads_match(k, q, "k"); _same(v, k, "v")
    B, N, heads, d = q.shape
    T, H, W = (int(x) for x in grid)
    if N != T * H * W:
        raise ValueError(f"q has {N} tokens per sample, the grid {T}x{H}x{W} has {T * H * W}")
    shp = make_shape(B, k.shape[1], grid, heads, d)
    o = _out(o, q, "o")
    _check("osp_attn_cross", library().osp_attn_cross(_ptr(q), _ptr(k), _ptr(v), _ptr(o), ctypes.byref(shp),
                                                      ctypes.c_float(scale), _stream_handle(q)))
    return o


def _attn3(fn: str, q, k, v, grid, text_len, scale, o, *extra):
    _bshd(q, "q"); _same(k, q, "k"); _same(v, q, "v")
    shp = _shape_of(q, grid, text_len)
    o = _out(o, q, "o")
    f = getattr(library(), fn)
    args = [_ptr(q), _ptr(k), _ptr(v), _ptr(o), ctypes.byref(shp), *extra, ctypes.c_float(scale), _stream_handle(q)]
    _check(fn, f(*args))
    return o


def attn_spatial(q, k, v, grid, scale: float = 0.0, o=None) -> torch.Tensor:
    """osp_attn_spatial: per-frame attention over the H*W tokens of each frame (no text)."""
    return _attn3("osp_attn_spatial", q, k, v, grid, 0, scale, o)


def attn_temporal(q, k, v, grid, causal: bool = False, scale: float = 0.0, o=None) -> torch.Tensor:
    """osp_attn_temporal: per-position attention over the T frames (causal: t' <= t)."""
    return _attn3("osp_attn_temporal", q, k, v, grid, 0, scale, o, int(bool(causal)))


def attn_frame_causal(q, k, v, grid, text_len: int, scale: float = 0.0, o=None) -> torch.Tensor:
    """osp_attn_frame_causal: token of frame t attends to the text and frames 0..t."""
    return _attn3("osp_attn_frame_causal", q, k, v, grid, text_len, scale, o)


def lse_shape(q: torch.Tensor, sparse_k: int = 1, text_len: int = 0):
    """Shape of the lse buffer of osp_attn_forward_train: [B*G, heads, ceil(n/128)*128]; with a
    joined text prefix (Skiparse, text_len > 0) one flat run: the video rows' block, then the
    text rows' [B, heads, ceil(text_len/128)*128]."""
    B, N, heads, _ = q.shape
    if sparse_k > 1 and text_len > 0:
        n = (N - text_len) // sparse_k
        return (B * sparse_k * heads * ((n + 127) // 128 * 128) + B * heads * ((text_len + 127) // 128 * 128),)
    G = 1 if sparse_k == 1 else sparse_k
    n = N // G
    return (B * G, heads, (n + 127) // 128 * 128)


def _lse_buffer(lse, shape, q: torch.Tensor) -> torch.Tensor:
    """The caller's lse buffer, checked against the shape the call writes, or a new one."""
    if lse is None:
        return torch.empty(shape, dtype=torch.float32, device=q.device)
    if lse.dtype != torch.float32 or lse.device != q.device or not lse.is_contiguous():
        raise ValueError("lse must be a contiguous float32 tensor on q's device")
    if lse.numel() < math.prod(shape):
        raise ValueError(f"lse holds {lse.numel()} values, the call writes {shape}")
    return lse


def attn_forward_train(q, k, v, grid, text_len: int = 0, sparse_k: int = 1, mode: int = 0, scale: float = 0.0,
                       o=None, lse=None):
    """osp_attn_forward_train: returns (o, lse)."""
    _bshd(q, "q"); _same(k, q, "k"); _same(v, q, "v")
    shp = _shape_of(q, grid, text_len)
    o = _out(o, q, "o")
    lse = _lse_buffer(lse, lse_shape(q, sparse_k, text_len), q)
    _check("osp_attn_forward_train",
           library().osp_attn_forward_train(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), ctypes.byref(shp),
                                            int(sparse_k), int(mode), ctypes.c_float(scale), _stream_handle(q)))
    return o, lse


def attn_backward(q, k, v, o, dout, lse, grid, text_len: int = 0, sparse_k: int = 1, mode: int = 0,
                  scale: float = 0.0, dq=None, dk=None, dv=None):
    """osp_attn_backward: returns (dq, dk, dv)."""
    _bshd(q, "q")
    for t, n in ((k, "k"), (v, "v"), (o, "o"), (dout, "dout")):
        _same(t, q, n)
    dq, dk, dv = _out(dq, q, "dq"), _out(dk, q, "dk"), _out(dv, q, "dv")
    lse = _lse_buffer(lse, lse_shape(q, sparse_k, text_len), q)
    shp = _shape_of(q, grid, text_len)
    _check("osp_attn_backward",
           library().osp_attn_backward(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(dout), _ptr(lse), _ptr(dq), _ptr(dk),
                                       _ptr(dv), ctypes.byref(shp), int(sparse_k), int(mode), ctypes.c_float(scale),
                                       _stream_handle(q)))
    return dq, dk, dv


def attn_frame_causal_train(q, k, v, grid, text_len: int = 0, scale: float = 0.0, o=None, lse=None):
    """osp_attn_frame_causal_train: returns (o, lse)."""
    _bshd(q, "q"); _same(k, q, "k"); _same(v, q, "v")
    shp = _shape_of(q, grid, text_len)
    o = _out(o, q, "o")
    lse = _lse_buffer(lse, lse_shape(q, 1), q)
    _check("osp_attn_frame_causal_train",
           library().osp_attn_frame_causal_train(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), ctypes.byref(shp),
                                                 ctypes.c_float(scale), _stream_handle(q)))
    return o, lse


def attn_frame_causal_backward(q, k, v, o, dout, lse, grid, text_len: int = 0, scale: float = 0.0, dq=None, dk=None,
                               dv=None):
    """osp_attn_frame_causal_backward: returns (dq, dk, dv)."""
    _bshd(q, "q")
    for t, n in ((k, "k"), (v, "v"), (o, "o"), (dout, "dout")):
        _same(t, q, n)
    dq, dk, dv = _out(dq, q, "dq"), _out(dk, q, "dk"), _out(dv, q, "dv")
    lse = _lse_buffer(lse, lse_shape(q, 1), q)
    shp = _shape_of(q, grid, text_len)
    _check("osp_attn_frame_causal_backward",
           library().osp_attn_frame_causal_backward(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(dout), _ptr(lse),
                                                    _ptr(dq), _ptr(dk), _ptr(dv), ctypes.byref(shp),
                                                    ctypes.c_float(scale), _stream_handle(q)))
    return dq, dk, dv


def factorized_lse_shape(q: torch.Tensor, grid, temporal: bool):
    """Shape of the lse buffer of the factorized training calls: [B*T, heads, ceil(H*W/128)*128]
    (spatial, one set per frame) or [B*H*W, heads, ceil(T/128)*128] (temporal, one per position)."""
    B, _, heads, _ = q.shape
    T, H, W = (int(a) for a in grid)
    sets, n = (B * H * W, T) if temporal else (B * T, H * W)
    return (sets, heads, (n + 127) // 128 * 128)


def _factorized_train(fn: str, q, k, v, grid, temporal: bool, extra, scale, o, lse):
    _bshd(q, "q"); _same(k, q, "k"); _same(v, q, "v")
    shp = _shape_of(q, grid, 0)
    o = _out(o, q, "o")
    lse = _lse_buffer(lse, factorized_lse_shape(q, grid, temporal), q)
    _check(fn, getattr(library(), fn)(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), ctypes.byref(shp), *extra,
                                      ctypes.c_float(scale), _stream_handle(q)))
    return o, lse


def _factorized_backward(fn: str, q, k, v, o, dout, lse, grid, temporal: bool, extra, scale, dq, dk, dv):
    _bshd(q, "q")
    for t, n in ((k, "k"), (v, "v"), (o, "o"), (dout, "dout")):
        _same(t, q, n)
    dq, dk, dv = _out(dq, q, "dq"), _out(dk, q, "dk"), _out(dv, q, "dv")
    shp = _shape_of(q, grid, 0)
    lse = _lse_buffer(lse, factorized_lse_shape(q, grid, temporal), q)
    _check(fn, getattr(library(), fn)(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(dout), _ptr(lse), _ptr(dq), _ptr(dk),
                                      _ptr(dv), ctypes.byref(shp), *extra, ctypes.c_float(scale), _stream_handle(q)))
    return dq, dk, dv


def attn_spatial_train(q, k, v, grid, scale: float = 0.0, o=None, lse=None):
    """osp_attn_spatial_train: per-frame attention with its saved lse; returns (o, lse)."""
    return _factorized_train("osp_attn_spatial_train", q, k, v, grid, False, (), scale, o, lse)


def attn_spatial_backward(q, k, v, o, dout, lse, grid, scale: float = 0.0, dq=None, dk=None, dv=None):
    """osp_attn_spatial_backward: returns (dq, dk, dv)."""
    return _factorized_backward("osp_attn_spatial_backward", q, k, v, o, dout, lse, grid, False, (), scale,
                                dq, dk, dv)


def attn_temporal_train(q, k, v, grid, causal: bool = False, scale: float = 0.0, o=None, lse=None):
    """osp_attn_temporal_train: per-position attention over time with its saved lse; returns (o, lse)."""
    return _factorized_train("osp_attn_temporal_train", q, k, v, grid, True, (int(bool(causal)),), scale, o, lse)


def attn_temporal_backward(q, k, v, o, dout, lse, grid, causal: bool = False, scale: float = 0.0, dq=None, dk=None,
                           dv=None):
    """osp_attn_temporal_backward: returns (dq, dk, dv)."""
    return _factorized_backward("osp_attn_temporal_backward", q, k, v, o, dout, lse, grid, True,
                                (int(bool(causal)),), scale, dq, dk, dv)


def _bounds(b) -> ctypes.Array:
    vals = [int(x) for x in b]
    return (ctypes.c_int32 * len(vals))(*vals)


def rope3d_packed(q: torch.Tensor, k: torch.Tensor, samples, split, theta: float = 10000.0,
                  q_out: Optional[torch.Tensor] = None, k_out: Optional[torch.Tensor] = None):
    """osp_rope3d_packed: 3D RoPE of a packed batch [1, total, heads, d]; ``samples`` lists
    (text_len, T, H, W) per sample.  Returns (q_out, k_out)."""
    _bshd(q, "q"); _same(k, q, "k")
    if q.shape[0] != 1 or q.shape[1] != _packed_rows(samples):
        raise ValueError(f"a packed batch is [1, {_packed_rows(samples)}, heads, d] for these samples "
                         f"(got {tuple(q.shape)})")
    q_out, k_out = _out(q_out, q, "q_out"), _out(k_out, k, "k_out")
    arr = (OspSampleGrid * max(1, len(samples)))(*[OspSampleGrid(*(int(x) for x in s)) for s in samples])
    rp = make_rope(split, theta)
    _, _, heads, d = q.shape
    _check("osp_rope3d_packed", library().osp_rope3d_packed(_ptr(q), _ptr(k), _ptr(q_out), _ptr(k_out), arr,
                                                            len(samples), heads, d, ctypes.byref(rp),
                                                            _stream_handle(q)))
    return q_out, k_out


def attn_packed(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, q_bounds, kv_bounds=None, scale: float = 0.0,
                o: Optional[torch.Tensor] = None) -> torch.Tensor:
    """osp_attn_packed: block-diagonal attention over a packed batch q [1, total_q, heads, d],
    k, v [1, total_kv, heads, d]; sample i owns rows [bounds[i], bounds[i+1])."""
    _bshd(q, "q"); _heads_match(k, q, "k"); _same(v, k, "v")
    if q.shape[0] != 1:
        raise ValueError(f"a packed batch has B = 1 (got {q.shape[0]})")
    _, _, heads, d = q.shape
    qb = _bounds(q_bounds)
    kb = _bounds(kv_bounds) if kv_bounds is not None else None
    if len(qb) < 1 or qb[len(qb) - 1] != q.shape[1]:
        raise ValueError(f"the last query bound must be q's {q.shape[1]} rows")
    kv_end = kb[len(kb) - 1] if kb is not None and len(kb) else (qb[len(qb) - 1] if len(qb) else -1)
    if kv_end != k.shape[1]:
        raise ValueError(f"the last key bound must be k's {k.shape[1]} rows (got {kv_end})")
    o = _out(o, q, "o")
    _check("osp_attn_packed", library().osp_attn_packed(_ptr(q), _ptr(k), _ptr(v), _ptr(o), qb, kb, len(qb) - 1,
                                                        heads, d, ctypes.c_float(scale), _stream_handle(q)))
    return o


def packed_lse_rows(bounds) -> int:
    """osp_attn_packed_lse_rows: lse rows per head of a packed batch (each sample's 256-row blocks)."""
    b = _bounds(bounds)
    n = library().osp_attn_packed_lse_rows(b, len(b) - 1)
    if n < 0:
        _check("osp_attn_packed_lse_rows", -n)
    return n


def _packed_self(q: torch.Tensor, bounds):
    _bshd(q, "q")
    if q.shape[0] != 1:
        raise ValueError(f"a packed batch has B = 1 (got {q.shape[0]})")
    b = _bounds(bounds)
    if len(b) < 2 or b[len(b) - 1] != q.shape[1]:
        raise ValueError(f"the last bound must be the batch's {q.shape[1]} rows")
    return b


def attn_packed_train(q, k, v, bounds, scale: float = 0.0, o=None, lse=None):
    """osp_attn_packed_train: packed self-attention with the saved lse; returns (o, lse), lse
    [heads, packed_lse_rows(bounds)] fp32."""
    b = _packed_self(q, bounds); _same(k, q, "k"); _same(v, q, "v")
    _, _, heads, d = q.shape
    o = _out(o, q, "o")
    rows = packed_lse_rows(bounds)
    if lse is None:
        lse = torch.empty((heads, rows), dtype=torch.float32, device=q.device)
    elif lse.dtype != torch.float32 or not lse.is_contiguous() or lse.numel() != heads * rows:
        raise ValueError(f"lse must be contiguous fp32 with {heads} x {rows} elements")
    _check("osp_attn_packed_train", library().osp_attn_packed_train(
        _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), b, len(b) - 1, heads, d, ctypes.c_float(scale),
        _stream_handle(q)))
    return o, lse


def attn_packed_backward(q, k, v, o, dout, lse, bounds, scale: float = 0.0, dq=None, dk=None, dv=None):
    """osp_attn_packed_backward: returns (dq, dk, dv)."""
    b = _packed_self(q, bounds)
    for t, n in ((k, "k"), (v, "v"), (o, "o"), (dout, "dout")):
        _same(t, q, n)
    _, _, heads, d = q.shape
    rows = packed_lse_rows(bounds)
    if lse.dtype != torch.float32 or not lse.is_contiguous() or lse.numel() != heads * rows:
        raise ValueError(f"lse must be contiguous fp32 with {heads} x {rows} elements")
    dq, dk, dv = _out(dq, q, "dq"), _out(dk, q, "dk"), _out(dv, q, "dv")
    _check("osp_attn_packed_backward", library().osp_attn_packed_backward(
        _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(dout), _ptr(lse), _ptr(dq), _ptr(dk), _ptr(dv), b, len(b) - 1,
        heads, d, ctypes.c_float(scale), _stream_handle(q)))
    return dq, dk, dv


def attn_full_noalloc(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, grid, text_len: int, scale: float = 0.0,
                      o: Optional[torch.Tensor] = None) -> torch.Tensor:
    """osp_attn_full_noalloc: dense attention whose call allocates no device memory (the
    library's scratch is a static device array).  `o` should be preallocated by such callers."""
    _bshd(q, "q"); _same(k, q, "k"); _same(v, q, "v")
    shp = _shape_of(q, grid, text_len)
    o = _out(o, q, "o")
    _check("osp_attn_full_noalloc",
           library().osp_attn_full_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(o), ctypes.byref(shp),
                                           ctypes.c_float(scale), _stream_handle(q)))
    return o


def skiparse_attn(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, grid, sparse_k: int, mode: int,
                  scale: float = 0.0, o: Optional[torch.Tensor] = None, text_len: int = 0) -> torch.Tensor:
    """osp_skiparse_attn: fused Skiparse attention in natural token order (text_len > 0: the text
    prefix is joined to every set as global tokens)."""
    _bshd(q, "q"); _same(k, q, "k"); _same(v, q, "v")
    shp = _shape_of(q, grid, text_len)
    o = _out(o, q, "o")
    _check("osp_skiparse_attn", library().osp_skiparse_attn(_ptr(q), _ptr(k), _ptr(v), _ptr(o), ctypes.byref(shp),
                                                            int(sparse_k), int(mode), ctypes.c_float(scale),
                                                            _stream_handle(q)))
    return o


def skiparse_gather(q: torch.Tensor, k: Optional[torch.Tensor], v: Optional[torch.Tensor], grid, sparse_k: int,
                    mode: int, split=None, theta: float = 10000.0):
    """osp_skiparse_gather: returns (q_out, k_out, v_out) in the k-fold batch layout; RoPE on q, k
    with the tokens' own positions when ``split`` is given."""
    _bshd(q, "q")
    for t, n in ((k, "k"), (v, "v")):
        if t is not None:
            _same(t, q, n)
    shp = _shape_of(q, grid, 0)
    if sparse_k < 1 or q.shape[1] % sparse_k:
        raise ValueError(f"sparse_k {sparse_k} must divide the {q.shape[1]} video tokens")
    B, N, heads, d = q.shape
    outs = []
    for t in (q, k, v):
        outs.append(None if t is None else torch.empty((B * sparse_k, N // sparse_k, heads, d), dtype=t.dtype,
                                                          device=t.device))
    rp = make_rope(split, theta) if split is not None else None
    _check("osp_skiparse_gather",
           library().osp_skiparse_gather(_ptr(q), _ptr(k), _ptr(v), _ptr(outs[0]), _ptr(outs[1]), _ptr(outs[2]),
                                         ctypes.byref(shp), int(sparse_k), int(mode),
                                         ctypes.byref(rp) if rp is not None else None, _stream_handle(q)))
    return tuple(outs)


def skiparse_scatter(o_perm: torch.Tensor, grid, sparse_k: int, mode: int,
                     o: Optional[torch.Tensor] = None) -> torch.Tensor:
    """osp_skiparse_scatter: inverse of the gather for one tensor."""
    _bshd(o_perm, "o_perm")
    Bk, n_set, heads, d = o_perm.shape
    T, H, W = (int(x) for x in grid)
    if sparse_k < 1 or Bk % sparse_k or n_set * sparse_k != T * H * W:
        raise ValueError(f"o_perm {tuple(o_perm.shape)} is not the k-fold batch of a {T}x{H}x{W} grid "
                         f"with sparse_k {sparse_k}")
    B, N = Bk // sparse_k, n_set * sparse_k
    if o is None:
        o = torch.empty((B, N, heads, d), dtype=o_perm.dtype, device=o_perm.device)
    elif tuple(o.shape) != (B, N, heads, d) or o.device != o_perm.device:
        raise ValueError(f"o must have shape {(B, N, heads, d)} on {o_perm.device} (got {tuple(o.shape)})")
    _bshd(o, "o")
    shp = make_shape(B, 0, grid, heads, d)
    _check("osp_skiparse_scatter", library().osp_skiparse_scatter(_ptr(o_perm), _ptr(o), ctypes.byref(shp),
                                                                  int(sparse_k), int(mode), _stream_handle(o)))
    return o


def skiparse_index_map(n_video: int, sparse_k: int, mode: int, device="cuda") -> torch.Tensor:
    """osp_skiparse_index_map: int32 [n_video] map, entry g*(n/k)+s = token of slot s of set g."""
    out = torch.empty(n_video, dtype=torch.int32, device=device)
    _check("osp_skiparse_index_map", library().osp_skiparse_index_map(int(n_video), int(sparse_k), int(mode),
                                                                      _ptr(out), _stream_handle(out)))
    return out


def check_status(device=None) -> None:
    """osp_check_status on the current stream: raises OspError on a device-side timeout."""
    dev = torch.device("cuda") if device is None else torch.device(device)
    _check("osp_check_status", library().osp_check_status(ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream)))
