"""The row-at-a-time oracle used by the full-size parity tests agrees with the
stepping oracle (OracleLayer) on small inputs: same thresholds (including the
stale reuse between refreshes), same kept sets, same outputs."""
import numpy as np
import pytest

from long_context_decoding_saga_b200 import workload
from oracle import saga_oracle
from tests import gpu_harness


@pytest.mark.parametrize("wl", [
    workload.Workload("s1", 2, 8, 2, 4, 64, 300, 1, 7, 20, 3, 0.05, "planted_mean", 11),
    workload.Workload("s2", 1, 6, 3, 6, 64, 90, 1, 5, 7, 1, 0.0, "gaussian", 12),
    workload.Workload("s3", 1, 4, 1, 2, 64, 50, 1, 4, workload.DENSE, 1 << 30, 0.0, "gaussian", 13),
], ids=lambda w: w.name)
def test_rows_match_stepping_oracle(wl):
    inp = {k: v.float().numpy() for k, v in workload.make_layer(wl, 0, device="cpu", steps=wl.steps).items()}
    l_cap = wl.l_kv + wl.steps
    n_top = wl.n_for_kernel(l_cap)
    orc = saga_oracle.OracleLayer(inp["K0"], inp["V0"], wl.h_q, n_top, wl.refresh, l_cap=l_cap)
    G = wl.h_q // wl.h_k
    rows = {"K": {}, "V": {}, "q": inp["q"], "k_new": inp["k_new"], "v_new": inp["v_new"]}
    for b in range(wl.batch):
        for h in range(wl.h_k):
            rows["K"][(b, h)] = inp["K0"][b, h]
        for u in range(wl.h_v):
            rows["V"][(b, u)] = inp["V0"][b, u]
    for t in range(wl.steps):
        res = orc.step(inp["q"][t], inp["k_new"][t], inp["v_new"][t])
        for b in range(wl.batch):
            for h in range(wl.h_k):
                js = slice(h * G, (h + 1) * G)
                r = gpu_harness.oracle_rows(rows, wl.h_q, wl.h_k, wl.h_v, n_top, wl.refresh, t, b, h)
                np.testing.assert_array_equal(r["tau"], res["tau"][b, js])
                np.testing.assert_array_equal(r["keep"], res["keep"][b, js])
                np.testing.assert_array_equal(r["scores"], res["scores"][b, js])
                np.testing.assert_allclose(r["out"], res["out"][b, js], rtol=0, atol=1e-12)
