"""Shared helpers of the GPU parity tests (comparison rules and case builders).

Tolerances: quantised codes and scales bit-exact; O within max-abs 1e-2 and
mean-abs 1e-3 of the oracle's float64 result, LSE within 1e-3 (natural log).
O is stored as bf16, whose own rounding moves a value of magnitude 2..4 by up
to 2^-7 and one of 4..8 by up to 2^-6, so the max-abs bound of each element is
1e-2 plus half a bf16 step at the oracle's value.
"""
from __future__ import annotations

import numpy as np
import torch

O_MAX_ABS = 1e-2
O_MEAN_ABS = 1e-3
LSE_MAX_ABS = 1e-3


def bf16_half_step(x: torch.Tensor) -> torch.Tensor:
    """Half the spacing of bf16 numbers at |x| (8 significant bits)."""
    e = torch.floor(torch.log2(x.abs().clamp_min(2.0 ** -126)))
    return 0.5 * torch.pow(2.0, e - 7)


# One record per O comparison: (tag, elements, elements beyond the plain 1e-2 that
# the added half bf16 step admitted, max-abs, mean-abs). The test session prints
# them at its end, so every run reports how often the bf16 output step was needed.
RECORDS: list[tuple[str, int, int, float, float]] = []


def compare_o(O_gpu: torch.Tensor, O_ref: np.ndarray, tag: str = ""):
    got = O_gpu.detach().to("cpu", torch.float64).reshape(O_ref.shape)
    ref = torch.from_numpy(np.ascontiguousarray(O_ref)).to(torch.float64)
    diff = (got - ref).abs()
    excess = diff - (O_MAX_ABS + bf16_half_step(ref))
    mx, mean = float(diff.max()), float(diff.mean())
    n_half_step = int((diff > O_MAX_ABS).sum())
    RECORDS.append((tag, int(diff.numel()), n_half_step, mx, mean))
    assert torch.isfinite(got).all(), f"{tag}: non-finite output"
    assert float(excess.max()) <= 0.0, f"{tag}: O error {mx:.3e} beyond 1e-2 + half a bf16 step"
    assert mean <= O_MEAN_ABS, f"{tag}: O mean-abs {mean:.3e}"
    return mx, mean


def compare_lse(L_gpu: torch.Tensor, L_ref: np.ndarray, tag: str = ""):
    got = L_gpu.detach().to("cpu", torch.float64).reshape(L_ref.shape).numpy()
    mx = float(np.abs(got - L_ref).max())
    assert np.isfinite(got).all(), f"{tag}: non-finite LSE"
    assert mx <= LSE_MAX_ABS, f"{tag}: LSE max-abs {mx:.3e}"
    return mx


def rows_of(B, Hq, S, picks):
    """Flat oracle row ids (b*Hq + h)*S + t for a list of (b, h, t)."""
    return np.array([(b * Hq + h) * S + t for b, h, t in picks], np.int64)
