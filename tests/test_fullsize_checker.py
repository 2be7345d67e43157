"""The full-size parity checker on the CPU: fed the stepping oracle's own
results it passes, through the spawned process pool too; a planted output
error, a threshold error, a dropped kept position or an unsorted list makes
it fail.  (The mistakes are planted in the recorded results, on the CPU.)"""
import copy

import numpy as np
import pytest

from long_context_decoding_saga_b200 import workload
from oracle import saga_oracle
from tests import fullsize_oracle, gpu_harness

WL = workload.Workload("checker", 2, 8, 2, 4, 64, 700, 2, 6, 40, 3, 0.02, "planted_mean", 21)


def _recorded(wl, layer):
    """What a GPU run would record for one layer, taken from the oracle itself."""
    steps = wl.steps
    l_cap = wl.l_kv + steps
    inp = workload.make_layer(wl, layer, device="cpu", steps=steps)
    orc = saga_oracle.OracleLayer(inp["K0"].float().numpy(), inp["V0"].float().numpy(), wl.h_q, wl.n_top,
                                  wl.refresh, l_cap=l_cap)
    rows = []
    for t in range(steps):
        res = orc.step(inp["q"][t].float().numpy(), inp["k_new"][t].float().numpy(),
                       inp["v_new"][t].float().numpy())
        keep = res["keep"]
        rows.append({"out": res["out"].astype(np.float32), "tau": res["tau"].copy(),
                     "count": keep.sum(-1).astype(np.int32),
                     "idx": [np.nonzero(keep[b, j])[0].astype(np.int32) for b in range(wl.batch)
                             for j in range(wl.h_q)]})
    return rows, wl.n_top, l_cap


def _task(rows, n_top, l_cap, layer=0):
    return {"wl": WL, "layer": layer, "steps": WL.steps, "n_top": n_top, "l_cap": l_cap, "gpu": rows, "threads": 1}


def test_checker_accepts_the_oracle_itself():
    rows, n_top, l_cap = _recorded(WL, 0)
    summary = fullsize_oracle.check_layer(_task(rows, n_top, l_cap))
    assert summary["max_out_err"] < 1e-6 and summary["max_tau_err"] == 0.0
    assert summary["index_sets_checked"] == WL.steps * WL.batch * WL.h_q
    assert summary["refresh_steps"] == 2


def test_checker_pool_over_layers():
    per_layer, n_top, l_cap = [], None, None
    for i in range(WL.layers):
        rows, n_top, l_cap = _recorded(WL, i)
        per_layer.append(rows)
    out = gpu_harness.check_full_all(WL, per_layer, n_top, l_cap, WL.steps, workers=2)
    assert [s["layer"] for s in out] == list(range(WL.layers))


@pytest.mark.parametrize("plant", ["out", "tau", "drop_index", "unsorted"])
def test_checker_catches_planted_mistakes(plant):
    rows, n_top, l_cap = _recorded(WL, 1)
    bad = copy.deepcopy(rows)
    t = 4
    if plant == "out":
        bad[t]["out"][1, 3, 5] += 0.05
    elif plant == "tau":
        bad[t]["tau"][0, 2] += 0.01
    elif plant == "drop_index":
        r = int(np.argmax([len(x) for x in bad[t]["idx"]]))
        bad[t]["idx"][r] = bad[t]["idx"][r][1:]  # one kept position lost (this seeded case: outside the band)
        bad[t]["count"].reshape(-1)[r] -= 1
    else:
        r = int(np.argmax([len(x) for x in bad[t]["idx"]]))
        bad[t]["idx"][r] = bad[t]["idx"][r][::-1].copy()
    with pytest.raises(AssertionError):
        fullsize_oracle.check_layer(_task(bad, n_top, l_cap, layer=1))
