"""The bench's host-side summaries of device records, on hand-built inputs
whose figures are worked out by hand: the per-unit trace summary (CTA
balance, FA/SA concurrency, time per tile, unit phases) and the interval
union of the host-path timeline."""
import numpy as np
import pytest

import bench


def _records():
    # columns: start, first S ready, last P handed over, end (ns), CTA, rank,
    # sparse, KV tiles
    return np.array([
        [0, 1000, 9000, 10000, 0, 0, 0, 4],          # CTA 0: FA unit, 0-10 us
        [10000, 10500, 14000, 15000, 0, 2, 1, 2],    # CTA 0: SA unit, 10-15 us (touches the FA unit)
        [0, 2000, 6000, 8000, 1, 1, 1, 2],           # CTA 1: SA unit, 0-8 us
    ], dtype=np.int64)


def test_unit_trace_summary_by_hand():
    s = bench.summarize_unit_trace(_records(), total=3)
    assert s["units"] == 3 and s["ctas"] == 2
    assert s["fa_units"] == 1 and s["sa_units"] == 2
    assert s["span_us"] == 15.0
    # CTA 1 finishes at 8 us, CTA 0 at 15 us; the median of two is 11.5
    assert s["cta_finish_us"] == {"min": 8.0, "median": 11.5, "max": 15.0}
    assert s["tail_us"] == 3.5
    # busy: CTA 0 15 us, CTA 1 8 us, over 2 CTAs x 15 us
    assert s["busy_fraction"] == pytest.approx(23 / 30, abs=1e-4)
    # FA [0, 10) and SA [0, 8) overlap for 8 us; the SA unit starting at the
    # FA unit's end does not overlap it
    assert s["fa_sa_concurrent_fraction"] == pytest.approx(8 / 15, abs=1e-4)
    assert s["fa_us_per_tile"] == 2.5            # 10 us over 4 tiles
    assert s["sa_us_per_tile"] == 3.25           # 13 us over 4 tiles
    assert s["unit_ramp_us"] == pytest.approx(3.5 / 3, abs=1e-3)    # 1, 0.5, 2 us
    assert s["unit_body_us"] == pytest.approx(15.5 / 3, abs=1e-3)   # 8, 3.5, 4 us
    assert s["unit_drain_us"] == pytest.approx(4.0 / 3, abs=1e-3)   # 1, 1, 2 us
    assert s["unit_tiles_mean"] == pytest.approx(8 / 3, abs=1e-2)


def test_unit_trace_summary_one_mode_only():
    rec = _records()[1:]                     # the two SA units
    s = bench.summarize_unit_trace(rec, total=2)
    assert s["fa_units"] == 0 and "fa_us_per_tile" not in s
    assert s["fa_sa_concurrent_fraction"] == 0.0
    # the span runs from the first start (CTA 1, 0 us) to the last end (CTA 0,
    # 15 us); CTA 0 is busy 10-15 us, CTA 1 0-8 us
    assert s["span_us"] == 15.0
    assert s["busy_fraction"] == pytest.approx((5 + 8) / 30, abs=1e-4)


def test_union_of_intervals():
    assert bench._union_ms([]) == 0.0
    assert bench._union_ms([(0, 10), (5, 20), (30, 40)]) == pytest.approx(0.030)
    assert bench._union_ms([(10, 20), (0, 10)]) == pytest.approx(0.020)    # touching, unsorted
    assert bench._union_ms([(0, 100), (10, 20), (30, 40)]) == pytest.approx(0.100)  # nested
