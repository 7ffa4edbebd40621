"""Helpers shared by the GPU parity tests: host<->device marshalling of the seeded inputs
and the tolerance of the float outputs.

Tolerance (float outputs, against the fp64 oracle): max-abs-error <= 1e-5 * max|ref| for
fp32 outputs and <= 1e-2 * max|ref| for bf16 outputs.  bf16 outputs are additionally held
to the rounding they must show: |got - ref| <= 2^-8 |ref| + 1e-5 max|ref| element-wise
(RNE to bf16 costs at most 2^-9 relative; the rest is the fp32 arithmetic)."""

from __future__ import annotations

import numpy as np

import torch


def dev(x: np.ndarray, dtype: str) -> torch.Tensor:
    """Host fp32 array (bf16-representable when dtype == 'bf16') -> contiguous CUDA tensor."""
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).cuda()
    return t.to(torch.bfloat16) if dtype == "bf16" else t


def tdtype(dtype: str):
    return torch.bfloat16 if dtype == "bf16" else torch.float32


def host64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to(torch.float64).cpu().numpy()


def check_close(got: torch.Tensor, ref: np.ndarray, out_dtype: str, what: str = ""):
    g = host64(got).reshape(ref.shape)
    ref = np.asarray(ref, np.float64)
    assert np.all(np.isfinite(g)), f"{what}: non-finite output"
    scale = float(np.max(np.abs(ref))) if ref.size else 0.0
    err = np.abs(g - ref)
    worst = float(err.max()) if err.size else 0.0
    if out_dtype == "f32":
        assert worst <= 1e-5 * scale, f"{what}: max err {worst:.3e} > 1e-5 * {scale:.3e}"
    else:
        assert worst <= 1e-2 * scale, f"{what}: max err {worst:.3e} > 1e-2 * {scale:.3e}"
        bound = 2.0 ** -8 * np.abs(ref) + 1e-5 * scale
        bad = np.argwhere(err > bound)
        assert bad.size == 0, f"{what}: {len(bad)} elements beyond bf16 rounding, first {bad[:3]}"
    return worst, scale
