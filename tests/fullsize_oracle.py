"""Worker side of the full-size parity tests: one layer of a configuration,
every decode step, through the stepping oracle, compared with what the GPU
recorded for that layer.

Runs in a process of its own (started with `spawn`, after the parent has
initialised CUDA), so it imports no CUDA code: it regenerates the layer's
inputs with the seeded generator on the CPU, which gives the same bytes the
GPU run was fed (the GPU run draws them on the CPU too and copies them over).
"""
from __future__ import annotations

import numpy as np

BAND = 1e-3     # |score - threshold| band inside which membership may differ
OUT_TOL = 1e-2  # max |O_gpu - O_oracle|


def check_layer(task):
    """task: dict(wl, layer, steps, n_top, l_cap, gpu) with gpu[t] = dict(out [B, h_q, d], tau [B, h_q],
    and, when index lists were recorded, count [B, h_q] and idx: list over (b, j) of kept positions).
    Returns a summary; raises AssertionError on the first mismatch."""
    import torch
    from threadpoolctl import threadpool_limits

    threads = max(1, task.get("threads", 1))
    torch.set_num_threads(threads)
    with threadpool_limits(limits=threads):  # the workers share the cores: no BLAS oversubscription
        return _check_layer(task)


def _check_layer(task):
    from long_context_decoding_saga_b200 import workload
    from oracle import saga_oracle

    wl, layer, steps = task["wl"], task["layer"], task["steps"]
    inp = workload.make_layer(wl, layer, device="cpu", steps=steps)
    orc = saga_oracle.OracleLayer(inp["K0"].float().numpy(), inp["V0"].float().numpy(), wl.h_q, task["n_top"],
                                  wl.refresh, l_cap=task["l_cap"])
    q, kn, vn = (inp[k].float().numpy() for k in ("q", "k_new", "v_new"))
    del inp
    worst_out, worst_tau, band_tokens, checked_sets, refreshes = 0.0, 0.0, 0, 0, 0
    for t in range(steps):
        res = orc.step(q[t], kn[t], vn[t])
        g = task["gpu"][t]
        where = f"{wl.name} layer {layer} step {t}"
        err = float(np.max(np.abs(g["out"].astype(np.float64) - res["out"])))
        assert err <= OUT_TOL, f"{where}: max |out diff| {err}"
        worst_out = max(worst_out, err)
        with np.errstate(invalid="ignore"):
            both = np.isneginf(res["tau"]) & np.isneginf(g["tau"])
            terr = np.where(both, 0.0, np.abs(g["tau"].astype(np.float64) - res["tau"].astype(np.float64)))
        assert float(np.max(terr)) <= BAND, f"{where}: threshold differs by {float(np.max(terr))}"
        worst_tau = max(worst_tau, float(np.max(terr)))
        refreshes += int(res["refreshed"])
        if "idx" in g:
            A, tau, keep = res["scores"], res["tau"], res["keep"]
            B, H = tau.shape
            for b in range(B):
                for j in range(H):
                    sel = g["idx"][b * H + j]
                    assert len(sel) == int(g["count"][b, j]), f"{where} b {b} head {j}: count / list length"
                    assert (np.diff(sel) > 0).all(), f"{where} b {b} head {j}: list not strictly ascending"
                    mine = np.zeros(A.shape[2], dtype=bool)
                    mine[sel] = True
                    far = np.abs(A[b, j].astype(np.float64) - np.float64(tau[b, j])) > BAND
                    bad = (mine != keep[b, j]) & far
                    assert not bad.any(), f"{where} b {b} head {j}: {int(bad.sum())} index mismatches outside the band"
                    band_tokens += int((~far).sum())
                    checked_sets += 1
    return {"layer": layer, "steps": steps, "max_out_err": worst_out, "max_tau_err": worst_tau,
            "band_tokens": band_tokens, "index_sets_checked": checked_sets, "refresh_steps": refreshes}
