"""Host check of the work-list invariant that the fused kernel's hand-over relies
on (dcn_forward_proj.cu): a gather step never spans more K-blocks than the
sample ring holds (four), for every chunk size the launcher can produce.  The
launcher's choices are restated here: a persistent grid of min(SMs, ceil(P/16))
CTAs, contiguous pixel ranges cut into chunks of at most 128 pixels, steps of
32 / LPI items (LPI = 16-byte lanes per item), or 32 items with per-point
records, which are chosen only when every chunk has at least 11 items per
K-block."""
import math

SMS = 148
RING = 4


def ranges(P, n_cta):
    return [(P * c // n_cta, P * (c + 1) // n_cta) for c in range(n_cta)]


def chunks(r0, r1):
    n = max(1, math.ceil((r1 - r0) / 128))
    return [(r0 + (r1 - r0) * c // n, r0 + (r1 - r0) * (c + 1) // n) for c in range(n)]


def max_span(n_items, step, per_kb):
    span = 0
    for first in range(0, n_items, step):
        last = min(first + step, n_items) - 1
        span = max(span, last // per_kb - first // per_kb + 1)
    return span


def launcher(P):
    n_cta = max(1, min(SMS, math.ceil(P / 16)))
    return n_cta, [c for r in ranges(P, n_cta) for c in chunks(*r) if c[1] > c[0]]


def test_chunk_sizes():
    for P in list(range(1, 700)) + [12800, 18944, 19600, 40000, 102400]:
        n_cta, ch = launcher(P)
        assert all(b - a <= 128 for a, b in ch)
        min_range = P // n_cta
        floor_px = 64 if min_range > 128 else min_range
        assert all(b - a >= floor_px for a, b in ch), P


def test_steps_span_at_most_the_ring():
    for C in (8, 16, 32, 64):           # 16-bit storage: LPI = C / 8, groups per K-block 64 / C
        lpi, gpb = C // 8, 64 // C
        for P in list(range(1, 400)) + [12800, 19600, 40000]:
            n_cta, ch = launcher(P)
            min_range = P // n_cta
            min_px = 64 if min_range > 128 else min_range
            pp = min_px * gpb >= 11
            for KB in (1, 3, 8):
                for a, b in {(0, b - a) for a, b in ch}:
                    per_kb = (b - a) * gpb
                    n_items = per_kb * KB
                    assert max_span(n_items, 32 // lpi, per_kb) <= RING, (C, P, b - a)
                    if pp:
                        assert max_span(n_items, 32, per_kb) <= RING, (C, P, b - a)
