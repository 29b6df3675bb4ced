"""The parity bars themselves, on the CPU: a gradient that is right up to its
one storage rounding passes, and a few percent of planted error fails.

The planted mistake is made on the oracle's own output (rounded to the
storage type as the GPU stores it), so no GPU is needed."""
import numpy as np
import pytest
import torch

import oracle
import synthetic_inputs as si
from parity import assert_close_bwd


def _bf16_backward():
    shape = si.CoreShape(B=1, H=10, W=11, G=2, C=32, softmax=True, dtype="bf16")
    inp = si.core_inputs(shape, 31, offset_std=2.0, oob_fraction=0.03, with_grad_out=True)
    return oracle.dcn_backward(inp["x"], inp["offset"], inp["mask"], inp["grad_out"], G=shape.G,
                               softmax=True)


@pytest.mark.parametrize("key", ["grad_offset", "grad_mask"])
def test_rounded_reduced_gradient_passes(key):
    ref = _bf16_backward()[key]
    stored = torch.from_numpy(ref).to(torch.bfloat16)  # one nearest-even rounding
    assert assert_close_bwd(stored, ref, key, atomic=False) <= 1.0


@pytest.mark.parametrize("key", ["grad_offset", "grad_mask"])
def test_five_percent_error_fails_reduced_bar(key):
    ref = _bf16_backward()[key]
    planted = torch.from_numpy(ref * 1.05).to(torch.bfloat16)  # e.g. a mis-applied scale
    with pytest.raises(AssertionError):
        assert_close_bwd(planted, ref, key, atomic=False)


def test_dropped_corner_term_fails_reduced_bar():
    """grad_offset with a quarter of its entries off by one corner's share
    (modelled as 10 % of the value on a random quarter of the elements)."""
    ref = _bf16_backward()["grad_offset"]
    rng = np.random.default_rng(0)
    bad = ref.copy()
    sel = rng.random(ref.shape) < 0.25
    bad[sel] *= 0.9
    with pytest.raises(AssertionError):
        assert_close_bwd(torch.from_numpy(bad).to(torch.bfloat16), ref, "grad_offset", atomic=False)


def test_fp16_reduced_bar_is_tighter_than_atomic_bar():
    ref = _bf16_backward()["grad_mask"]
    planted = torch.from_numpy(ref * 1.01).to(torch.float16)  # 1 %: far above fp16 rounding
    with pytest.raises(AssertionError):
        assert_close_bwd(planted, ref, "grad_mask", atomic=False)
    assert_close_bwd(planted, ref, "grad_mask", atomic=True)  # the grad_x bar would let it through


def test_summation_bound_values():
    """gamma_(n+1) * A for small n, no bound once (n+1) u >= 1/2."""
    from parity import summation_bound

    u = 2.0 ** -8
    b = summation_bound(np.array([2.0, 2.0, 2.0]), np.array([3.0, 126.0, 127.0]), torch.bfloat16)
    assert b[0] == pytest.approx(4 * u / (1 - 4 * u) * 2.0)
    assert b[1] == pytest.approx(127 * u / (1 - 127 * u) * 2.0)
    assert np.isinf(b[2])
    assert summation_bound(np.array([1.0]), np.array([1000.0]), torch.float32)[0] == pytest.approx(
        1001 * 2.0 ** -24 / (1 - 1001 * 2.0 ** -24))


def test_budget_admits_rounding_and_rejects_a_mis_scaled_gradient():
    """Errors within half the worst-case summation bound pass (including
    elements whose contributions cancel, where the bar on |ref| + rms alone
    fails); a grad_x off by 20 % (a modulation applied twice, a mis-scaled
    kernel weight) fails, since where nothing cancels the bound is about
    (n + 1) u |ref|, about 10 % of the value for 25 bf16 additions."""
    shape = si.CoreShape(B=1, H=10, W=11, G=2, C=32, dtype="bf16")
    inp = si.core_inputs(shape, 32, offset_std=2.0, with_grad_out=True)
    ref = oracle.dcn_backward(inp["x"], inp["offset"], inp["mask"], inp["grad_out"], G=shape.G)["grad_x"]
    bud = oracle.dcn_grad_x_budget(inp["offset"], inp["mask"], inp["grad_out"], x_shape=tuple(inp["x"].shape),
                                   G=shape.G)
    from parity import summation_bound

    terms = np.repeat(bud["terms"], shape.C, axis=-1)
    bound = summation_bound(bud["abs_sum"], terms, torch.bfloat16)
    near = torch.from_numpy(ref + 0.5 * np.where(np.isfinite(bound), bound, 0.0)).to(torch.bfloat16)
    with pytest.raises(AssertionError):
        assert_close_bwd(near, ref, "near, no budget")
    assert assert_close_bwd(near, ref, "near", budget=bud) <= 1.0
    scaled = torch.from_numpy(ref * 1.2).to(torch.bfloat16)
    with pytest.raises(AssertionError):
        assert_close_bwd(scaled, ref, "scaled", budget=bud)
