"""Host check of the division by an invariant divisor used in the fused kernel's
item decode (dcn_forward_proj.cu): q = mulhi(n, floor((2^32 - 1) / d)) is low by
at most one for every n < 2^31, so one remainder correction gives the exact
quotient and remainder (Granlund and Montgomery, "Division by invariant integers
using multiplication", 1994, round-down reciprocal)."""
import numpy as np


def _fastdiv(n: np.ndarray, d: int):
    m = np.uint64(0xFFFFFFFF // d)
    q = (n.astype(np.uint64) * m) >> np.uint64(32)
    r = n.astype(np.uint64) - q * np.uint64(d)
    fix = r >= np.uint64(d)
    return q + fix, r - np.where(fix, np.uint64(d), np.uint64(0))


def test_fastdiv_exact_below_2_31():
    rng = np.random.default_rng(0)
    divisors = [1, 2, 3, 5, 7, 8, 9, 25, 63, 64, 87, 100, 127, 128, 200, 1600, 4095, 12800,
                65536, 123457, 1000003, (1 << 30) + 7, (1 << 31) - 1]
    edge = np.arange((1 << 31) - 4096, 1 << 31, dtype=np.uint64)
    small = np.arange(0, 1 << 16, dtype=np.uint64)
    for d in divisors:
        n = np.concatenate([small, edge, rng.integers(0, 1 << 31, 1 << 18, dtype=np.uint64),
                            np.arange(0, 1 << 31, max(d, 1) * 997, dtype=np.uint64)[: 1 << 16] + np.uint64(d - 1)])
        n = n[n < (1 << 31)]
        q, r = _fastdiv(n, d)
        np.testing.assert_array_equal(q, n // np.uint64(d))
        np.testing.assert_array_equal(r, n % np.uint64(d))


def test_fastdiv_one_correction_needed():
    # the estimate alone is not exact: the correction step is exercised
    n = np.arange(0, 1 << 16, dtype=np.uint64)
    m = np.uint64(0xFFFFFFFF // 3)
    q0 = (n * m) >> np.uint64(32)
    assert (q0 != n // np.uint64(3)).any()
