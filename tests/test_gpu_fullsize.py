"""Full-size parity in the benchmark's launch configuration (needs a B200).

Llama-SAGA 32K (16 layers x 64 steps), Qwen-SAGA 128K (28 layers x 32 steps)
and dense GQA 128K (16 layers x 32 steps) run with every layer per step,
through CUDA-graph replays that read the length from the device, exactly as
the benchmark times them, and every layer of every step is compared with the
stepping oracle: outputs (max-abs 1e-2), thresholds (within 1e-3) and, for
the sparse configurations, the kept index sets (band rule).  The oracle runs
one layer per worker process.  A first run without index tracking (the timed
configuration) gives the outputs; a second run with tracking must give the
same bits, and its index lists are checked.

Llama-SAGA 32K and Qwen-SAGA 128K also run with every layer of a step in one call (batch = layers x B)
and are checked the same way.

The sweep (Llama-3.2-1B shapes) covers every (h_k, N, R) triple at 128K
context with batch 1, and mixed points at every context length and batch,
each on two of its 16 layers (the layers are drawn independently, so any two
stand for the rest) and on sampled steps: a refresh step, stale-threshold
steps and the next refresh.
"""
import numpy as np
import pytest
import torch

from long_context_decoding_saga_b200 import saga, workload
from tests import gpu_harness

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from long_context_decoding_saga_b200 import build
    build.build()
    saga.load()


FULL = [workload.LLAMA_SAGA_32K, workload.QWEN_SAGA_128K, workload.DENSE_GQA_128K]


@pytest.mark.parametrize("wl", FULL, ids=lambda w: w.name)
def test_every_layer_and_step_matches_oracle(wl):
    steps = wl.steps
    inputs = gpu_harness.layer_inputs_on_gpu(wl, steps)
    plain, n_top, l_cap = gpu_harness.run_full_all(wl, inputs, steps, track=False)
    # index lists of every row: the sparse configurations (the dense one keeps every token: counts only)
    tracked, _, _ = gpu_harness.run_full_all(wl, inputs, steps, track=True, record_idx=not wl.dense)
    del inputs
    torch.cuda.empty_cache()
    for i in range(wl.layers):
        for t in range(steps):
            assert np.array_equal(plain[i][t]["out"], tracked[i][t]["out"]), f"layer {i} step {t}: tracking changed O"
            if wl.dense:
                assert (tracked[i][t]["count"] == wl.l_kv + t + 1).all(), f"layer {i} step {t}: dense count"
                del tracked[i][t]["count"]
    summaries = gpu_harness.check_full_all(wl, tracked, n_top, l_cap, steps)
    assert len(summaries) == wl.layers
    assert all(s["steps"] == steps for s in summaries)
    if not wl.dense:
        assert sum(s["index_sets_checked"] for s in summaries) == wl.layers * steps * wl.batch * wl.h_q
        assert all(s["refresh_steps"] == (steps + wl.refresh - 1) // wl.refresh for s in summaries)


@pytest.mark.parametrize("wl", [workload.LLAMA_SAGA_32K, workload.QWEN_SAGA_128K], ids=lambda w: w.name)
def test_layers_in_one_call_match_oracle(wl):
    """The same steps with every layer of a step in one call (batch = layers x B): every layer of every step
    against the stepping oracle, index sets included."""
    steps = wl.steps
    inputs = gpu_harness.layer_inputs_on_gpu(wl, steps)
    tracked, n_top, l_cap = gpu_harness.run_full_all(wl, inputs, steps, track=True, record_idx=True,
                                                    layer_batched=True)
    del inputs
    torch.cuda.empty_cache()
    summaries = gpu_harness.check_full_all(wl, tracked, n_top, l_cap, steps)
    assert len(summaries) == wl.layers
    assert sum(s["index_sets_checked"] for s in summaries) == wl.layers * steps * wl.batch * wl.h_q


# Every (h_k, N, R) triple at 128K with batch 1, plus points that bring in every context length and batch.
SWEEP = [workload.sweep_point(131072, 1, hk, n, r) for hk in workload.SWEEP_H_K for n in workload.SWEEP_N
         for r in workload.SWEEP_R]
SWEEP += [
    workload.sweep_point(4096, 1, 1, 64, 1),
    workload.sweep_point(4096, 16, 8, 1024, 16),
    workload.sweep_point(16384, 4, 2, 256, 64),
    workload.sweep_point(16384, 16, 1, 64, 16),
    workload.sweep_point(65536, 1, 4, 1024, 1),
    workload.sweep_point(65536, 4, 8, 64, 64),
    workload.sweep_point(131072, 4, 4, 256, 1),
    workload.sweep_point(131072, 16, 8, 256, 16),
]


@pytest.mark.parametrize("wl", SWEEP, ids=lambda w: w.name)
def test_sweep_sampled_parity(wl):
    R = wl.refresh
    steps = (0, 1, 2) if R == 1 else (0, 3, R) if R <= 16 else (0, 5)
    groups = ((0, 0), (wl.batch - 1, wl.h_k - 1))
    got, inputs, n_top = gpu_harness.run_full_sampled(wl, (0, 1), steps, groups, layers=2, track=True)
    gpu_harness.check_full_sampled(wl, got, inputs, n_top, track=True)
