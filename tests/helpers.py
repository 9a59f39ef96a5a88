"""Comparison helpers shared by the tests (no method arithmetic here)."""

import numpy as np
import torch

# Tolerances for attention outputs against the fp64 oracle (bf16 inputs): max-abs and relative-L2
ATTN_MAX_ABS = 2e-2
ATTN_REL_L2 = 5e-3


def to_f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float64).numpy()


def bf16_round(x: np.ndarray) -> torch.Tensor:
    """fp64 values -> bf16 tensor, correctly rounded (the oracle's storage rounding)."""
    from oracle import round_to_bf16
    return torch.from_numpy(round_to_bf16(x).astype(np.float32)).to(torch.bfloat16)


def assert_bf16_close(got: torch.Tensor, ref: torch.Tensor, what: str = ""):
    """Correctly rounded results: at most 1 ulp apart anywhere, and almost all identical."""
    dist = bf16_ulp_distance(got, ref)
    mx = int(dist.max()) if dist.numel() else 0
    frac = float((dist != 0).double().mean()) if dist.numel() else 0.0
    assert mx <= 1 and frac <= 1e-4, f"{what}: max ulp distance {mx}, mismatch fraction {frac:.2e}"


def bf16_ulp_distance(a: torch.Tensor, b: torch.Tensor) -> torch.Tensor:
    """|ordered(a) - ordered(b)| on the bf16 bit patterns (0 = identical, 1 = adjacent)."""
    def ordered(t):
        i = t.contiguous().view(torch.int16).to(torch.int32)
        return torch.where(i < 0, -32768 - i, i)
    return (ordered(a.cpu()) - ordered(b.cpu())).abs()


def attn_errors(gpu: torch.Tensor, ref: np.ndarray):
    g = to_f64(gpu)
    d = g - ref
    return float(np.abs(d).max()), float(np.linalg.norm(d) / max(np.linalg.norm(ref), 1e-300))


def assert_attn_close(gpu: torch.Tensor, ref: np.ndarray, what: str = ""):
    assert np.isfinite(to_f64(gpu)).all(), f"{what}: non-finite output"
    mx, rl = attn_errors(gpu, ref)
    assert mx <= ATTN_MAX_ABS and rl <= ATTN_REL_L2, f"{what}: max-abs {mx:.3e}, rel-L2 {rl:.3e}"
    return mx, rl
