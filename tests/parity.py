"""Tolerances and comparison helpers of the GPU parity tests.

The bars (fp32 accumulation in every case):
  fp32 storage:  |gpu - ref| <= 1e-5 * (1 + |ref|)      element by element
  fp16 storage:  |gpu - ref| <= 2e-3 * max|ref|
  bf16 storage:  |gpu - ref| <= 8e-3 * max|ref|
  atomic backward, fp32:  |gpu - ref| <= 1e-4 * (|ref| + rms(ref))
The fp16/bf16 bars contain the final rounding of the output to the storage
type (half an ulp: 2^-11 and 2^-8 relative) plus fp32 summation error.  The
backward bar is relative to the tensor's own scale because an input
gradient is a sum of many atomically added contributions that can cancel.
NaN must match NaN exactly.
"""
from __future__ import annotations

import numpy as np
import torch

FWD_TOL = {torch.float32: ("elem", 1e-5), torch.float16: ("max", 2e-3), torch.bfloat16: ("max", 8e-3)}
# Backward in fp16/bf16 storage: the oracle's gradients are rounded once to the
# storage type by the GPU, and grad_x is summed by packed half-precision atomic
# adds (one rounding per addition, up to 4*K*ceil(max tap reach) additions).
BWD_TOL = {torch.float32: 1e-4, torch.float16: 2e-2, torch.bfloat16: 1e-1}


def to_np(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float64).numpy()


def assert_close_fwd(gpu: torch.Tensor, ref: np.ndarray, what: str = "out") -> float:
    """Assert the forward bar for gpu's storage dtype; returns the worst ratio err/bound."""
    g = to_np(gpu)
    nan_g, nan_r = np.isnan(g), np.isnan(ref)
    assert np.array_equal(nan_g, nan_r), f"{what}: NaN pattern differs ({nan_g.sum()} vs {nan_r.sum()})"
    g, r = g[~nan_r], ref[~nan_r]
    if r.size == 0:
        return 0.0
    kind, tol = FWD_TOL[gpu.dtype]
    err = np.abs(g - r)
    if kind == "elem":
        bound = tol * (1.0 + np.abs(r))
    else:
        bound = np.full_like(r, tol * max(np.abs(r).max(), 1e-30))
    ratio = err / bound
    worst = int(np.argmax(ratio))
    assert ratio[worst] <= 1.0, (f"{what}: |err| {err[worst]:.3e} > bound {bound[worst]:.3e} "
                                 f"at flat {worst} (gpu {g[worst]!r}, ref {r[worst]!r})")
    return float(ratio.max())


def assert_close_bwd(gpu: torch.Tensor, ref: np.ndarray, what: str) -> float:
    g = to_np(gpu)
    nan_g, nan_r = np.isnan(g), np.isnan(ref)
    assert np.array_equal(nan_g, nan_r), f"{what}: NaN pattern differs"
    g, r = g[~nan_r], ref[~nan_r]
    if r.size == 0:
        return 0.0
    tol = BWD_TOL[gpu.dtype]
    rms = float(np.sqrt(np.mean(r * r))) if r.size else 0.0
    bound = tol * (np.abs(r) + rms)
    err = np.abs(g - r)
    ratio = err / np.maximum(bound, 1e-300)
    worst = int(np.argmax(ratio))
    assert ratio[worst] <= 1.0, (f"{what}: |err| {err[worst]:.3e} > bound {bound[worst]:.3e} "
                                 f"at flat {worst} (gpu {g[worst]!r}, ref {r[worst]!r})")
    return float(ratio.max())
