"""The benchmark's timed window (CPU only): it starts on a refresh step, so a
window of K = R steps holds exactly one refresh step, and the per-kind means
amortize over one refresh period."""
import os
import sys

import pytest

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
import bench  # noqa: E402


@pytest.mark.parametrize("warmup", [3, 4, 7, 31, 40])
@pytest.mark.parametrize("refresh", [1, 2, 16, 32, 64])
def test_window_starts_on_refresh(warmup, refresh):
    a = bench.alignment_steps(warmup, refresh)
    assert 0 <= a < refresh or (refresh == 1 and a == 0)
    first_timed = 1 + warmup + a  # step 0 runs eagerly before the warm-up
    assert first_timed % refresh == 0
    kinds = [(first_timed + i) % refresh == 0 for i in range(refresh)]
    assert sum(kinds) == 1 and kinds[0]


def test_no_alignment_without_refresh():
    assert bench.alignment_steps(3, 1 << 30) == 0


def test_step_means_amortize():
    # R = 4: one refresh step of 10 ms and three reuse steps of 2 ms
    st = bench.step_means([10.0, 2.0, 2.0, 2.0], [True, False, False, False], 4)
    assert st["refresh_mean_us"] == pytest.approx(10000.0)
    assert st["reuse_mean_us"] == pytest.approx(2000.0)
    assert st["amortized_us"] == pytest.approx(4000.0)  # equals the window mean when K = R
    only = bench.step_means([3.0, 5.0], [True, True], 1)
    assert only["reuse_mean_us"] is None and "amortized_us" not in only
