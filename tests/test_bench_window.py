"""The benchmark's timed window (CPU only): it holds refresh and reuse steps
in the proportion of the refresh schedule (the nearest whole number of
refresh steps to K / R; exactly K / R when R divides K), and the per-kind
means amortize over one refresh period.  Also the key of the recorded
DRAM-traffic figure (the kernels' code without comments)."""
import os
import sys

import pytest

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
import bench  # noqa: E402


@pytest.mark.parametrize("warmup", [3, 4, 7, 31, 40])
@pytest.mark.parametrize("refresh", [1, 2, 16, 32, 64])
@pytest.mark.parametrize("steps", [1, 5, 8, 16, 20, 32, 40, 64, 100])
def test_window_holds_proportional_refreshes(warmup, refresh, steps):
    a = bench.alignment_steps(warmup, refresh, steps)
    assert 0 <= a < max(refresh, 1)
    first = 1 + warmup + a  # step 0 runs eagerly before the warm-up
    n = sum(1 for t in range(first, first + steps) if t % refresh == 0)
    assert n == int(steps / refresh + 0.5)
    if steps % refresh == 0:
        assert n == steps // refresh


def test_no_alignment_without_refresh():
    assert bench.alignment_steps(3, 1 << 30, 32) == 0


def test_step_means_amortize():
    # R = 4: one refresh step of 10 ms and three reuse steps of 2 ms
    st = bench.step_means([10.0, 2.0, 2.0, 2.0], [True, False, False, False], 4)
    assert st["refresh_mean_us"] == pytest.approx(10000.0)
    assert st["reuse_mean_us"] == pytest.approx(2000.0)
    assert st["amortized_us"] == pytest.approx(4000.0)  # equals the window mean when K = R
    only = bench.step_means([3.0, 5.0], [True, True], 1)
    assert only["reuse_mean_us"] is None and "amortized_us" not in only


@pytest.mark.parametrize("first", [0, 1, 5, 36, 77])
@pytest.mark.parametrize("refresh,steps", [(32, 32), (32, 16), (16, 64), (64, 32), (1, 7)])
def test_any_window_start(first, refresh, steps):
    a = bench.alignment_from(first, refresh, steps)
    assert bench.refresh_count(first + a, steps, refresh) == int(steps / refresh + 0.5)


@pytest.mark.parametrize("warmup,steps,refresh,e2e", [(3, 32, 32, True), (3, 16, 16, True), (3, 16, 64, True),
                                                      (5, 100, 64, True), (3, 10, 1, False), (3, 32, 1 << 30, True)])
def test_step_plan(warmup, steps, refresh, e2e):
    p = bench.step_plan(warmup, steps, refresh, e2e)
    assert p["total"] == 1 + warmup + p["A"] + steps + p["A2"] + p["E"] + p["T"]
    assert p["timed_first"] == 1 + warmup + p["A"]
    assert p["e2e_first"] == p["timed_first"] + steps + p["A2"]
    if refresh <= 1024:
        want = int(steps / refresh + 0.5)
        assert bench.refresh_count(p["timed_first"], steps, refresh) == want
        if e2e:
            assert bench.refresh_count(p["e2e_first"], p["E"], refresh) == int(p["E"] / refresh + 0.5)
    assert (p["E"] == 0) == (not e2e)


def test_traffic_key_ignores_comments_only():
    """The recorded DRAM-traffic figure is keyed by the kernels' code: comment and whitespace edits keep the
    key, any code edit (a string literal's text included) changes it."""
    src = 'int a = 1; // count\n/* two\n lines */ asm volatile("mov.u32 %0, 1; // x" : "=r"(a));\nchar c = \'/\';'
    same = 'int a = 1;   /* another comment */\nasm volatile("mov.u32 %0, 1; // x" : "=r"(a)); // trailing\nchar c = \'/\';'
    assert bench.code_tokens(src) == bench.code_tokens(same)
    assert bench.code_tokens(src) != bench.code_tokens(src.replace("a = 1", "a = 2"))
    assert bench.code_tokens(src) != bench.code_tokens(src.replace("// x", "// y"))
    assert "//" in bench.code_tokens(src) and "count" not in bench.code_tokens(src)
