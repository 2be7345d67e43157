"""Full-size parity in the benchmark's launch configuration (needs a B200).

The Llama-SAGA 32K, Qwen-SAGA 128K and dense-GQA 128K configurations run
with every layer per step, through CUDA-graph replays that read the length
from the device, exactly as the benchmark times them.  The oracle recomputes
sampled (layer, step, batch, key-head group) rows one at a time: a refresh
step, stale-threshold steps after it, and the next refresh where the step
count reaches it.  Outputs are checked in the untracked configuration (the
one timed); a second run with index tracking checks the selected index sets
and that tracking leaves the outputs bit-identical.
"""
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


# (workload, checked layers, checked steps, checked (batch, key head) groups)
FULL = [
    (workload.LLAMA_SAGA_32K, (0, 7, 15), (0, 9, 16), ((0, 0), (0, 1))),
    (workload.QWEN_SAGA_128K, (0, 13, 27), (0, 5, 31), ((0, 0),)),
    (workload.DENSE_GQA_128K, (0, 15), (0, 3), ((0, 0), (0, 5))),
]


@pytest.mark.parametrize("case", FULL, ids=lambda c: c[0].name)
def test_full_size_sampled_parity(case):
    wl, layers, steps, groups = case
    got, inputs, n_top = gpu_harness.run_full_sampled(wl, layers, steps, groups, track=False)
    gpu_harness.check_full_sampled(wl, got, inputs, n_top, track=False)
    got_t, _, _ = gpu_harness.run_full_sampled(wl, layers, steps, groups, track=True)
    for key, row in got.items():
        assert (row["out"] == got_t[key]["out"]).all(), f"{key}: index tracking changed the output"
    gpu_harness.check_full_sampled(wl, got_t, inputs, n_top, track=True)


# Sweep points (Llama-3.2-1B shapes, h_q=32, h_v=8, d=64) chosen so that every value of every axis
# appears: l_kv {4K,16K,64K,128K}, batch {1,4,16}, h_k {1,2,4,8}, N {64,256,1024}, R {1,16,64}.  Two
# of the 16 layers each (the layers are drawn independently, so any two stand for the rest).
SWEEP = [
    workload.sweep_point(4096, 1, 1, 64, 1),
    workload.sweep_point(4096, 16, 8, 1024, 16),
    workload.sweep_point(16384, 4, 2, 256, 64),
    workload.sweep_point(16384, 16, 1, 64, 16),
    workload.sweep_point(65536, 1, 4, 1024, 1),
    workload.sweep_point(65536, 4, 8, 64, 64),
    workload.sweep_point(131072, 1, 2, 1024, 64),
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
