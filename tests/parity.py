"""Tolerances and comparison helpers of the GPU parity tests.

The bars (fp32 accumulation in every case):
  fp32 storage:  |gpu - ref| <= 1e-5 * (1 + |ref|)      element by element
  fp16 storage:  |gpu - ref| <= 2e-3 * max|ref|
  bf16 storage:  |gpu - ref| <= 8e-3 * max|ref|
  backward, fp32 (every gradient):  |gpu - ref| <= 1e-4 * (|ref| + rms(ref))
  backward, fp16/bf16 grad_offset and grad_mask:
                 |gpu - ref| <= 2e-3 (fp16) / 8e-3 (bf16) * (|ref| + rms(ref))
  backward, fp16/bf16 grad_x (packed half-precision atomic adds):
                 |gpu - ref| <= 2e-2 (fp16) / 1e-1 (bf16) * (|ref| + rms(ref))
The fp16/bf16 forward bars contain the final rounding of the output to the
storage type (half an ulp: 2^-11 and 2^-8 relative) plus fp32 summation error.
"1e-4 relative" for the backward is read per element against the tensor's own
scale, |ref| + rms(ref): an input gradient is a sum of many atomically added
contributions that can cancel to far below the size of its terms, so a bar
on |ref| alone would be meaningless where the sum cancels.
grad_offset and grad_mask are reduced in fp32 (over the channels of one
item, by lane shuffles) and stored once: in 16-bit storage their only error
beyond fp32 summation is that one rounding (at most 2^-11 resp. 2^-8
relative), which the 2e-3 / 8e-3 bars cover with room to spare while a few
percent of error (a mis-scaled or dropped term) fails them.  grad_x in
16-bit storage is summed by packed half-precision atomic adds, each rounding
to the storage type, so it keeps the wider bars; where the oracle's error
budget is passed (`budget`: per element the absolute sum A of the n
contributions and n itself), an element may instead stay within the
recursive-summation bound gamma_(n+1) * A, gamma_m = m u / (1 - m u), u the
storage type's unit roundoff (2^-24, 2^-11, 2^-8): the bound that holds for
any order of the atomic additions, which matters where a sum cancels far
below its terms.  Where (n+1) u >= 1/2 (over 127 additions in bf16) no
useful bound exists and the element is checked for its NaN pattern only.
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
# grad_offset / grad_mask: fp32 lane reductions stored once (no atomics).
BWD_TOL_REDUCED = {torch.float32: 1e-4, torch.float16: 2e-3, torch.bfloat16: 8e-3}


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


# Unit roundoff of each storage type (round to nearest).
UNIT_ROUNDOFF = {torch.float32: 2.0 ** -24, torch.float16: 2.0 ** -11, torch.bfloat16: 2.0 ** -8}


def summation_bound(abs_sum: np.ndarray, terms: np.ndarray, dtype: torch.dtype) -> np.ndarray:
    """gamma_(n+1) * A: the error bound of n contributions with absolute sum A
    added one by one, each partial sum and each contribution rounded once.
    The bound holds while (n+1) u < 1; where (n+1) u >= 1/2 (more than 127
    additions in bf16, 1023 in fp16) it exceeds A itself and the element is
    left unbounded (infinite): a 16-bit running sum of that many terms can lose
    every significant bit, in any order of the additions."""
    mu = (terms + 1.0) * UNIT_ROUNDOFF[dtype]
    with np.errstate(divide="ignore"):
        return np.where(mu < 0.5, mu / (1.0 - np.minimum(mu, 0.5)) * abs_sum, np.inf)


def assert_close_bwd(gpu: torch.Tensor, ref: np.ndarray, what: str, atomic: bool = True, budget=None) -> float:
    """Backward bar: `atomic` for gradients summed by atomic adds (grad_x),
    else the tighter bar of gradients reduced in fp32 and stored once.
    `budget` (atomic only): the oracle's {"abs_sum", "terms"} for grad_x."""
    g = to_np(gpu)
    nan_g, nan_r = np.isnan(g), np.isnan(ref)
    assert np.array_equal(nan_g, nan_r), f"{what}: NaN pattern differs"
    keep = ~nan_r
    g, r = g[keep], ref[keep]
    if r.size == 0:
        return 0.0
    tol = (BWD_TOL if atomic else BWD_TOL_REDUCED)[gpu.dtype]
    rms = float(np.sqrt(np.mean(r * r))) if r.size else 0.0
    bound = tol * (np.abs(r) + rms)
    if budget is not None:
        assert atomic, "an error budget applies to atomically summed gradients"
        C = ref.shape[-1] // budget["terms"].shape[-1]
        terms = np.repeat(budget["terms"], C, axis=-1)
        bound = np.maximum(bound, summation_bound(budget["abs_sum"], terms, gpu.dtype)[keep])
    err = np.abs(g - r)
    ratio = err / np.maximum(bound, 1e-300)
    worst = int(np.argmax(ratio))
    assert ratio[worst] <= 1.0, (f"{what}: |err| {err[worst]:.3e} > bound {bound[worst]:.3e} "
                                 f"at flat {worst} (gpu {g[worst]!r}, ref {r[worst]!r})")
    return float(ratio.max())
